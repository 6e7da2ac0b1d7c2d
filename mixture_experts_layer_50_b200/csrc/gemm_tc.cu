// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by TMA.
//
// It computes, for every expert group g of variable size (read on the device from
// offsets[], so no group size ever travels to the host):
//     out[row0_g + i][n] = epilogue( sum_k A[arow0_g + i][k] * B[g][n][k] )
// with both operands K-major bf16 and fp32 accumulation in tensor memory.  The same kernel
// serves the three tensor-core steps of the layer:
//   * the router projection z = x . W_g (one group, fp32 store, plus a per-expert offset);
//   * the expert gate/up projection with SiLU(gate) * up (optionally clamped, "SwiGLU,
//     écrêtée à 10" in the DeepSeek-V4.1-Flash table) or ReLU fused in the epilogue
//     ("Le compte des paramètres": W_gate, W_up, W_down per expert; dataistudio listing:
//     max(x W1, 0) W2);
//   * the expert down projection (plain bf16 store).
// The shared expert ("Des experts partagés") is one more group whose rows are all tokens.
//
// Design (one CTA per SM, persistent over a static round-robin of output tiles):
//   warp 0      one thread issues TMA loads of 128x64 A tiles and BNx64 B tiles (128-byte
//               swizzle) into a STAGES-deep ring of shared-memory stages;
//   warp 1      allocates 2*BN TMEM columns (two accumulators) and one thread issues
//               tcgen05.mma (M=128, N=BN, K=16) and tcgen05.commit;
//   warps 2-5   drain an accumulator with tcgen05.ld while the next tile accumulates in
//               the other one, apply the epilogue, stage rows in shared memory and write
//               them with coalesced 16-byte stores, masking rows beyond the group and
//               columns beyond n_out.
// Tiles are numbered group by group, N-block outer and M-block inner, so the CTAs working
// at the same time share B panels (weights) and A panels (tokens) through L2.
// Tall tiles (AM = 256, BN = 256): a tile is 256 rows, two M = 128 MMAs per k-step on one
// B stage, their accumulators in TMEM columns [0, 256) and [256, 512); half the shared-memory
// operand bytes per MMA of the 128-row tile, and each stage holds twice the MMA time.
// Every wait is bounded (globaltimer); on expiry the kernel records MOE_ERR_TIMEOUT in
// the status word, lets the other roles stop, drains what it issued and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kStageA = BM * BK * 2;   // 16 KB
constexpr int kStagingPerWarp = 32 * 128;   // 32 rows of 128 B, 16-byte pieces XOR-swizzled
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// ---- mbarrier ------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Polls after which a wait gives up even if the global timer did not advance (a backstop:
// each poll takes well over 20 ns, so this is more than a second).
constexpr uint64_t kWaitMaxPolls = 50000000ull;

// Wait for the phase of `parity` to complete.  Gives up (false) when another role of the
// CTA has given up, or after limit_ns, recording a timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort_flag, int* status,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint64_t polls = 0;; ++polls) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns || polls > kWaitMaxPolls) {
      *abort_flag = 1;
      report_status(status, kStatusTimeout);
      return false;
    }
  }
}

// Wait, after an abort, for copies or MMAs this thread already issued (their barrier phase
// completes when they land); bounded by the same time limit and poll backstop as mbar_wait,
// and records nothing: the abort is reported already.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  for (uint64_t polls = 0; polls <= kWaitMaxPolls; ++polls)
    if (mbar_try_wait(bar, parity) || global_timer_ns() - t0 >= kWaitLimitNs) return;
}

// ---- TMA -----------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ---- tcgen05 -------------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor of a K-major tile written by TMA with the 128-byte
// swizzle: rows of 128 bytes, 8-row (1024-byte) swizzle atoms stacked at a 1024-byte
// stride (SBO); the leading-dimension offset is unused for this layout (set to 1).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// TMEM columns the 1-SM kernel allocates: two BN-column accumulators, rounded up to the
// power of two the allocator requires (BN = 192 -> 512).
template <int BN>
__host__ __device__ constexpr int tmem_cols() {
  return 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
}
// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both K-major.
template <int BN>
__device__ __forceinline__ constexpr uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// Thread i of the warp receives TMEM lane (taddr.lane + i), 32 consecutive columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- clusters and the 2-SM (cta_group::2) forms ----------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// The same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA load into this CTA's shared memory whose byte count completes on the barrier of the
// pair's first CTA (`bar` is a shared::cluster address there).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// Arrive on the barrier at this offset in both CTAs of the pair once the issued MMAs finish.
__device__ __forceinline__ void mma_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], m;\n\t}\n" ::"r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mma_commit_pair_local(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

struct Args {
  const int32_t* offsets;
  int n_routed;
  int has_shared;
  int shared_rows;
  int shared_a_row0;
  int shared_out_row0;
  int K;
  int n_out;
  int up_row0;       // SwiGLU: first W_up row inside a group's B slice
  float clamp;
  const float* col_bias;
  void* out;
  void* out_shared;   // non-null: the shared group's row r goes to row r here, not into out
  int64_t ld_out;
  int* status;
  int k_splits;       // > 1: split K; split s writes rows [s * split_rows, ...) of out
  int64_t split_rows;
  int m64_tails;      // 1-SM kernel: a tile with at most 64 valid rows issues M = 64 MMAs
  int half_tails;     // 2-SM kernel: a tile with at most 128 valid rows issues M = 128 MMAs
  int band;           // > 0: M blocks of a large group run in bands of this many (decode_tile)
};

// AM: A rows a stage holds (128; 64 for a batch whose groups all fit 64 rows, which leaves
// room for more stages of weights; 256 for tall tiles).
template <int BN, int STAGES, int AM = BM>
struct Layout {
  static constexpr int kStageA = AM * BK * 2;
  static constexpr int kStageB = BN * BK * 2;
  static constexpr int kOffB = STAGES * kStageA;
  static constexpr int kOffStaging = kOffB + STAGES * kStageB;
  static constexpr int kOffBar = kOffStaging + 4 * kStagingPerWarp;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;       // tmem base, abort flag
  static constexpr int kOffStart = kOffMisc + 16;               // tile prefix [G + 1]
  static size_t bytes(int groups) { return 1024 + kOffStart + 4 * (size_t)(groups + 1); }
};

// Tile -> (group, M block, N block).  Tiles are numbered group by group; inside a group the
// operand with the smaller total panel is kept resident in L2 while the other streams: if the
// group's A rows outnumber its B rows, M blocks are outer and N blocks inner, else the reverse.
// band > 0 (a group whose A panel outgrows L2): the group's M blocks run in bands of `band`;
// inside a band, N blocks outer and the band's M blocks inner, so the band's A rows stay in
// L2 while the weights stream once per band.
template <int BMT, int BN>
__device__ __forceinline__ void decode_tile(int tile, const int* s_start, int G, int nt,
                                            int& g, int& m_blk, int& n_blk, int band = 0) {
  int lo = 0, hi = G;  // largest g with s_start[g] <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_start[mid] <= tile) lo = mid; else hi = mid;
  }
  g = lo;
  const int r = tile - s_start[g];
  const int mt = (s_start[g + 1] - s_start[g]) / nt;
  if (band > 0 && mt > band && mt * BMT <= nt * BN) {
    const int per_band = band * nt;
    const int b = r / per_band;
    const int rr = r - b * per_band;
    const int mb = min(band, mt - b * band);
    n_blk = rr / mb;
    m_blk = b * band + (rr - n_blk * mb);
  } else if (mt * BMT > nt * BN) {
    m_blk = r / nt;
    n_blk = r - m_blk * nt;
  } else {
    n_blk = r / mt;
    m_blk = r - n_blk * mt;
  }
}

// SiLU(a) = a * sigmoid(a) with the fast exponential and division (the result is rounded to
// bf16 right after); for a below about -88 the denominator overflows and the result is 0.
__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

// One epilogue warp drains its 32 TMEM lanes (rows row_base + lane of the output tile) of an
// accumulator: activation, packing, per-warp staging in shared memory, then coalesced 16-byte
// stores with row and column masks.  `release` runs right after the last TMEM read.
// `chunks` (default: the whole tile) chunks of output columns are drained, starting at TMEM
// column 0 of the accumulator and at output column n_blk * kOutPerTile + col_extra.
template <int BN, int EPI, typename Release>
__device__ __forceinline__ void epilogue_warp(const Args& p, void* out, uint32_t t_row,
                                              uint8_t* stg, int lane, int n_blk,
                                              int64_t out_row0, int row_base, int rows_valid,
                                              Release&& release, int chunks = -1,
                                              int col_extra = 0) {
  constexpr int kOutPerTile = (EPI == kEpiSwiglu) ? BN / 2 : BN;
  constexpr int kColsPerChunk = (EPI == kEpiStoreF32) ? 32 : 64;
  constexpr int kChunks = kOutPerTile / kColsPerChunk;
  const int n_chunks = chunks < 0 ? kChunks : chunks;
#pragma unroll 1
  for (int c = 0; c < n_chunks; ++c) {
    uint32_t packed[32];
    if constexpr (EPI == kEpiSwiglu) {
      float gv[32], uv[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tmem_ld32(t_row + c * 64 + h * 32, gv);
        tmem_ld32(t_row + BN / 2 + c * 64 + h * 32, uv);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float g0 = gv[2 * i], g1 = gv[2 * i + 1], u0 = uv[2 * i], u1 = uv[2 * i + 1];
          if (p.clamp > 0.f) {
            g0 = fminf(fmaxf(g0, -p.clamp), p.clamp);
            g1 = fminf(fmaxf(g1, -p.clamp), p.clamp);
            u0 = fminf(fmaxf(u0, -p.clamp), p.clamp);
            u1 = fminf(fmaxf(u1, -p.clamp), p.clamp);
          }
          __nv_bfloat162 hv = __floats2bfloat162_rn(silu_f(g0) * u0, silu_f(g1) * u1);
          packed[h * 16 + i] = *reinterpret_cast<uint32_t*>(&hv);
        }
      }
    } else if constexpr (EPI == kEpiStoreF32) {
      float v[32];
      tmem_ld32(t_row + c * 32, v);
      tmem_ld_wait();
      const int col0 = n_blk * BN + c * 32;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float o = v[i];
        if (p.col_bias != nullptr && col0 + i < p.n_out) o += p.col_bias[col0 + i];
        packed[i] = __float_as_uint(o);
      }
    } else {
      float v[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tmem_ld32(t_row + c * 64 + h * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float a = v[2 * i], b = v[2 * i + 1];
          if (EPI == kEpiRelu) {
            a = fmaxf(a, 0.f);
            b = fmaxf(b, 0.f);
          }
          __nv_bfloat162 hv = __floats2bfloat162_rn(a, b);
          packed[h * 16 + i] = *reinterpret_cast<uint32_t*>(&hv);
        }
      }
    }
    if (c == n_chunks - 1) release();
    // stage this thread's 128-byte row piece: piece i of row r at 16 * (i ^ (r & 7)), so the
    // eight threads of each quarter-warp access hit eight different bank groups, in the
    // row-wise writes here and in the piece-wise reads below
    uint8_t* my = stg + lane * 128;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint4*>(my + 16 * (i ^ (lane & 7))) =
          make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
    __syncwarp();
    // coalesced copy-out: 4 rows x 128 bytes per instruction
    constexpr int kElPerPiece = (EPI == kEpiStoreF32) ? 4 : 8;
    const int col_base = n_blk * kOutPerTile + col_extra + c * kColsPerChunk;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int rr = i * 4 + (lane >> 3);
      const int pc = lane & 7;
      const int row_in_tile = row_base + rr;
      const int col = col_base + pc * kElPerPiece;
      if (row_in_tile < rows_valid && col < p.n_out) {
        const uint4 val = *reinterpret_cast<const uint4*>(stg + rr * 128 + 16 * (pc ^ (rr & 7)));
        const int64_t orow = out_row0 + row_in_tile;
        if constexpr (EPI == kEpiStoreF32) {
          // fp32 rows of n_out = E columns: a 16-byte store only where the row stride and the
          // base keep it 16-byte aligned (E a multiple of 4), else element by element
          float* o = reinterpret_cast<float*>(out) + orow * p.ld_out + col;
          const bool vec = (p.ld_out & 3) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0;
          if (vec && col + 4 <= p.n_out) {
            *reinterpret_cast<uint4*>(o) = val;
          } else {
            const float* f = reinterpret_cast<const float*>(&val);
            const int n = min(4, p.n_out - col);
            for (int e = 0; e < n; ++e) o[e] = f[e];
          }
        } else {
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + orow * p.ld_out + col;
          *reinterpret_cast<uint4*>(o) = val;  // n_out % 8 == 0 (checked on the host)
        }
      }
    }
    __syncwarp();
  }
}

template <int BN, int EPI, int STAGES, int AM = BM>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmAs,
                        const __grid_constant__ CUtensorMap tmB, const Args p) {
  pdl_wait();
  using L = Layout<BN, STAGES, AM>;
  // AM = 64: groups are cut into 64-row tiles, each running M = 64 MMAs
  constexpr bool kAll64 = AM < BM;
  // AM = 256: tall tiles, one accumulator in two halves of BN columns (rows 0-127, 128-255)
  constexpr bool kTall = AM > BM;
  static_assert(!kTall || (AM == 2 * BM && 2 * BN <= 512), "tall tiles: 256 rows, 2 BN <= 512");
  constexpr int TM = AM;  // rows of an output tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + L::kOffB;
  uint8_t* staging = smem + L::kOffStaging;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  int* s_start = reinterpret_cast<int*>(smem + L::kOffStart);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.n_routed + p.has_shared;
  constexpr int kOutPerTile = (EPI == kEpiSwiglu) ? BN / 2 : BN;
  const int nt = (p.n_out + kOutPerTile - 1) / kOutPerTile;
  const int nk = (p.K + BK - 1) / BK;

  // ---- tile schedule: per-group tile counts and their prefix, from device offsets ----
  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int g0 = min(lane * per, G), g1 = min(g0 + per, G);
    int local = 0;
    for (int g = g0; g < g1; ++g) {
      const int cnt = g < p.n_routed ? p.offsets[g + 1] - p.offsets[g] : p.shared_rows;
      local += ((cnt + TM - 1) / TM) * nt;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int g = g0; g < g1; ++g) {
      s_start[g] = run;
      const int cnt = g < p.n_routed ? p.offsets[g + 1] - p.offsets[g] : p.shared_rows;
      run += ((cnt + TM - 1) / TM) * nt;
    }
    if (lane == 31) s_start[G] = incl;
    if (lane == 0) {
      for (int i = 0; i < STAGES; ++i) {
        mbar_init(&full[i], 1);
        mbar_init(&empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&tfull[i], 1);
        mbar_init(&tempty[i], 128);
      }
      mbar_init(drain, 1);
      *s_abort = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(s_tmem)),
                 "r"(tmem_cols<BN>()));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  // with a split K, work item = (output tile, K slice); slices of a tile are adjacent
  const int ks_n = p.k_splits > 1 ? p.k_splits : 1;
  const int kper = (nk + ks_n - 1) / ks_n;
  const int total = s_start[G] * ks_n;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      int stage = 0;

      uint32_t phase = 0;
      int armed = 0;  // stages armed so far (for the drain on abort)
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        int g, m_blk, n_blk;
        decode_tile<TM, BN>(tile / ks_n, s_start, G, nt, g, m_blk, n_blk, p.band);
        const int kb0 = (tile % ks_n) * kper, kb1 = min(nk, kb0 + kper);
        const bool sh = g >= p.n_routed;
        const int a_row = (sh ? p.shared_a_row0 : p.offsets[g]) + m_blk * TM;
        const CUtensorMap* mA = sh ? &tmAs : &tmA;
        // tall tiles: the second 128-row A box only when the tile has rows past 128
        bool a_hi = false;
        if constexpr (kTall) {
          const int cnt = sh ? p.shared_rows : p.offsets[g + 1] - p.offsets[g];
          a_hi = cnt - m_blk * TM > BM;
        }
        constexpr int kBoxA = kTall ? BM * BK * 2 : L::kStageA;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, p.status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[stage], (a_hi ? 2 : 1) * kBoxA + L::kStageB);
          tma_load_2d(sA + stage * L::kStageA, mA, &full[stage], kb * BK, a_row);
          if (a_hi)
            tma_load_2d(sA + stage * L::kStageA + kBoxA, mA, &full[stage], kb * BK, a_row + BM);
          uint8_t* b_dst = sB + stage * L::kStageB;
          if (EPI == kEpiSwiglu) {
            tma_load_3d(b_dst, &tmB, &full[stage], kb * BK, n_blk * (BN / 2), g);
            tma_load_3d(b_dst + (BN / 2) * BK * 2, &tmB, &full[stage], kb * BK,
                        p.up_row0 + n_blk * (BN / 2), g);
          } else {
            tma_load_3d(b_dst, &tmB, &full[stage], kb * BK, n_blk * BN, g);
          }
          ++armed;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every load of this CTA is issued: the next kernel on the stream may be scheduled
      pdl_release();
      if (!ok) {
        // let the loads already issued land before the CTA leaves
        for (int i = 0; i < STAGES && i < armed; ++i) {
          stage = (stage + STAGES - 1) % STAGES;
          if (stage == STAGES - 1) phase ^= 1;
          mbar_drain(&full[stage], phase);
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16<BN>();
      // M = 64: the same descriptor with the M field halved
      constexpr uint32_t kIdesc64 = (kIdesc & ~(0x1Fu << 24)) | ((uint32_t)(64 >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        int g, m_blk, n_blk;
        decode_tile<TM, BN>(tile / ks_n, s_start, G, nt, g, m_blk, n_blk, p.band);
        const int cnt = g < p.n_routed ? p.offsets[g + 1] - p.offsets[g] : p.shared_rows;
        if constexpr (kTall) {
          // One accumulator in two halves.  The epilogue hands back half 0 (tempty[0]) and
          // then half 1 (tempty[1]) of the previous tile; this tile starts its half-0 MMAs
          // as soon as half 0 is free and defers the half-1 MMAs of up to STAGES - 1 stages
          // (their stages stay held) until half 1 is free.  Both barriers are waited once
          // per tile, so their phases stay in step with the tile count.
          const uint32_t ph = (uint32_t)(it & 1);
          const int rows = cnt - m_blk * TM;
          const bool two = rows > BM;
          const uint32_t id0 = (p.m64_tails && rows <= 64) ? kIdesc64 : kIdesc;
          const uint32_t id1 = (p.m64_tails && rows - BM <= 64) ? kIdesc64 : kIdesc;
          if (!mbar_wait(&tempty[0], ph ^ 1, s_abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int kb0 = (tile % ks_n) * kper, kb1 = min(nk, kb0 + kper);
          bool h1 = false;              // half 1 of the accumulator is free
          int pend = 0, pend_stage = 0, pend_kb = 0;  // deferred half-1 k-blocks
          auto half1 = [&](int st, int kb) {
            const uint32_t a1 = smem_u32(sA + st * L::kStageA + BM * BK * 2);
            const uint32_t b1 = smem_u32(sB + st * L::kStageB);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_bf16(tmem_base + (uint32_t)BN, sw128_desc(a1 + kk * 32),
                       sw128_desc(b1 + kk * 32), id1, (kb > kb0 || kk > 0) ? 1u : 0u);
          };
          auto flush = [&]() {
            int st = pend_stage;
            for (int i = 0; i < pend; ++i) {
              half1(st, pend_kb + i);
              mma_commit(&empty[st]);
              st = st + 1 == STAGES ? 0 : st + 1;
            }
            pend = 0;
          };
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(&full[stage], phase, s_abort, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(sA + stage * L::kStageA);
            const uint32_t b0 = smem_u32(sB + stage * L::kStageB);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_bf16(tmem_base, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), id0,
                       (kb > kb0 || kk > 0) ? 1u : 0u);
            bool commit = true;
            if (two) {
              if (!h1) h1 = mbar_try_wait(&tempty[1], ph ^ 1);
              if (!h1 && pend < STAGES - 1) {
                if (pend == 0) {
                  pend_stage = stage;
                  pend_kb = kb;
                }
                ++pend;
                commit = false;
              } else {
                if (!h1) {
                  if (!mbar_wait(&tempty[1], ph ^ 1, s_abort, p.status)) {
                    ok = false;
                    break;
                  }
                  h1 = true;
                }
                tc_fence_after();
                flush();
                half1(stage, kb);
              }
            }
            if (commit) mma_commit(&empty[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          if (!h1) {
            // a one-half tile, or a K loop shorter than the deferral: wait for half 1 here
            if (!mbar_wait(&tempty[1], ph ^ 1, s_abort, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            flush();
          }
          mma_commit(&tfull[0]);
          continue;
        }
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        const uint32_t idesc =
            (kAll64 || (p.m64_tails && cnt - m_blk * TM <= 64)) ? kIdesc64 : kIdesc;
        if (!mbar_wait(&tempty[acc], aph ^ 1, s_abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        const int kb0 = (tile % ks_n) * kper, kb1 = min(nk, kb0 + kper);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, s_abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * L::kStageA);
          const uint32_t b0 = smem_u32(sB + stage * L::kStageB);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            mma_bf16(d_tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                     (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) mma_commit(&tfull[acc]);
      }
      if (!ok) {
        // wait for the MMAs already issued before TMEM is released
        mma_commit(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // ================= epilogue (warps 2..5) =================
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    uint8_t* stg = staging + (warp - 2) * kStagingPerWarp;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      int g, m_blk, n_blk;
      decode_tile<TM, BN>(tile / ks_n, s_start, G, nt, g, m_blk, n_blk, p.band);
      const int acc = kTall ? 0 : it & 1;
      const uint32_t aph = kTall ? (uint32_t)(it & 1) : (uint32_t)((it >> 1) & 1);
      // warp-uniform decision: tcgen05.ld below needs all 32 lanes
      const bool ready = mbar_wait(&tfull[acc], aph, s_abort, p.status);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const bool sh = g >= p.n_routed;
      const int cnt = sh ? p.shared_rows : p.offsets[g + 1] - p.offsets[g];
      const int64_t out_row0 = (int64_t)(sh ? p.shared_out_row0 : p.offsets[g]) + m_blk * TM +
                               (int64_t)(tile % ks_n) * p.split_rows;
      const int rows_valid = min(TM, cnt - m_blk * TM);
      void* out = (sh && p.out_shared != nullptr) ? p.out_shared : p.out;
      if constexpr (kTall) {
        // half h: rows 128 h .. 128 h + 127 of the tile, TMEM columns [BN h, BN h + BN);
        // each half is handed back to the MMA warp as soon as it is read
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const int rows_h = min(BM, rows_valid - h * BM);
          if (rows_h <= 0) {
            tc_fence_before();
            mbar_arrive(&tempty[h]);
            continue;
          }
          const uint32_t t_row =
              tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * BN);
          const bool m64 = p.m64_tails && rows_h <= 64;
          const int row_base = m64 ? q * 16 : q * 32;
          const int rows_w = m64 ? min(rows_h, q * 16 + 16) : rows_h;
          epilogue_warp<BN, EPI>(p, out, t_row, stg, lane, n_blk, out_row0 + h * BM, row_base,
                                 rows_w, [&] {
                                   tc_fence_before();
                                   mbar_arrive(&tempty[h]);
                                 });
        }
        continue;
      }
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      // an M = 64 accumulator holds rows 16q .. 16q + 15 in lanes 32q .. 32q + 15
      const bool m64 = kAll64 || (p.m64_tails && rows_valid <= 64);
      const int row_base = m64 ? q * 16 : q * 32;
      const int rows_w = m64 ? min(rows_valid, q * 16 + 16) : rows_valid;

      epilogue_warp<BN, EPI>(p, out, t_row, stg, lane, n_blk, out_row0, row_base, rows_w, [&] {
        // all TMEM reads of this accumulator are done: hand it back to the MMA warp
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
      });
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(tmem_cols<BN>()));
  }
}

// ---- 2-SM variant ------------------------------------------------------------------------
// A cluster of two CTAs on neighbouring SMs computes 256x256 tiles with tcgen05.mma
// cta_group::2 (M = 256): CTA r stages rows [128 r, 128 r + 128) of the A tile and half of the
// B tile (the gate box or the up box for SwiGLU; B rows [128 r, 128 r + 128) otherwise), so
// each SM moves half the B bytes of the 1-SM kernel per MMA.  Both CTAs' TMA loads complete on
// the first CTA's barrier; the first CTA issues the MMAs; commits arrive on both CTAs'
// barriers; each CTA drains its own 128 accumulator rows from its own TMEM.
template <int STAGES>
struct Layout2 {
  static constexpr int kStageA = tc::kStageA;          // 128 rows x 64 (16 KB)
  static constexpr int kStageB = 128 * BK * 2;         // 128 rows x 64 (16 KB)
  static constexpr int kOffB = STAGES * kStageA;
  static constexpr int kOffStaging = kOffB + STAGES * kStageB;
  static constexpr int kOffBar = kOffStaging + 4 * kStagingPerWarp;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffStart = kOffMisc + 16;
  static size_t bytes(int groups) { return 1024 + kOffStart + 4 * (size_t)(groups + 1); }
};

template <int EPI, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmAs,
                            const __grid_constant__ CUtensorMap tmB, const Args p) {
  pdl_wait();
  constexpr int BN = 256;   // MMA N
  constexpr int BMT = 256;  // tile rows (128 per CTA)
  // half tiles for group tails: an elementwise epilogue only (SwiGLU pairs columns c and
  // c + 128, which a half tile's accumulator keeps in different warps' lanes)
  constexpr bool kHalfTiles = EPI != kEpiSwiglu;
  using L = Layout2<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + L::kOffB;
  uint8_t* staging = smem + L::kOffStaging;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  int* s_start = reinterpret_cast<int*>(smem + L::kOffStart);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int G = p.n_routed + p.has_shared;
  constexpr int kOutPerTile = (EPI == kEpiSwiglu) ? BN / 2 : BN;
  const int nt = (p.n_out + kOutPerTile - 1) / kOutPerTile;
  const int nk = (p.K + BK - 1) / BK;

  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int g0 = min(lane * per, G), g1 = min(g0 + per, G);
    int local = 0;
    for (int g = g0; g < g1; ++g) {
      const int cnt = g < p.n_routed ? p.offsets[g + 1] - p.offsets[g] : p.shared_rows;
      local += ((cnt + BMT - 1) / BMT) * nt;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int g = g0; g < g1; ++g) {
      s_start[g] = run;
      const int cnt = g < p.n_routed ? p.offsets[g + 1] - p.offsets[g] : p.shared_rows;
      run += ((cnt + BMT - 1) / BMT) * nt;
    }
    if (lane == 31) s_start[G] = incl;
    if (lane == 0) {
      for (int i = 0; i < STAGES; ++i) {
        mbar_init(&full[i], 1);
        mbar_init(&empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&tfull[i], 1);
        mbar_init(&tempty[i], 8);  // one arrive per epilogue warp of both CTAs
      }
      mbar_init(drain, 1);
      *s_abort = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(s_tmem)),
                 "r"(2 * BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = s_start[G];

  if (warp == 0) {
    // ================= TMA producer (both CTAs) =================
    if (lane == 0) {
      const uint32_t full0 = map_to_cta(smem_u32(&full[0]), 0);  // the first CTA's barriers
      int stage = 0;
      uint32_t phase = 0;
      int armed = 0;
      bool ok = true;
      // a half tile (at most 128 valid rows) gives each CTA 64 rows: CTA 1's start at 64
      auto a_row_of = [&](int g, int m_blk) {
        const bool sh = g >= p.n_routed;
        const int cnt = sh ? p.shared_rows : p.offsets[g + 1] - p.offsets[g];
        const bool half = kHalfTiles && p.half_tails && cnt - m_blk * BMT <= BMT / 2;
        return (sh ? p.shared_a_row0 : p.offsets[g]) + m_blk * BMT + (int)rank * (half ? 64 : 128);
      };
      auto b_row_of = [&](int n_blk) {
        if (EPI == kEpiSwiglu) return rank == 0 ? n_blk * 128 : p.up_row0 + n_blk * 128;
        return n_blk * BN + (int)rank * 128;
      };
      for (int tile = pair; ok && tile < total; tile += npairs) {
        int g, m_blk, n_blk;
        decode_tile<BMT, BN>(tile, s_start, G, nt, g, m_blk, n_blk, p.band);
        const CUtensorMap* mA = g >= p.n_routed ? &tmAs : &tmA;
        const int a_row = a_row_of(g, m_blk);
        const int b_row = b_row_of(n_blk);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, p.status)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_expect_tx(&full[stage], 2 * (L::kStageA + L::kStageB));
          const uint32_t bar = full0 + 8u * (uint32_t)stage;
          tma_load_2d_pair(sA + stage * L::kStageA, mA, bar, kb * BK, a_row);
          tma_load_3d_pair(sB + stage * L::kStageB, &tmB, bar, kb * BK, b_row, g);
          ++armed;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      pdl_release();
      if (!ok && rank == 0) {
        for (int i = 0; i < STAGES && i < armed; ++i) {
          stage = (stage + STAGES - 1) % STAGES;
          if (stage == STAGES - 1) phase ^= 1;
          mbar_drain(&full[stage], phase);
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (first CTA of the pair) =================
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                  ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BMT >> 4) << 24);
      // M = 128 across the pair (64 rows per CTA): the same descriptor with the M field halved
      constexpr uint32_t kIdescHalf = (kIdesc & ~(0x1Fu << 24)) | ((uint32_t)(128 >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        int g, m_blk, n_blk;
        decode_tile<BMT, BN>(tile, s_start, G, nt, g, m_blk, n_blk, p.band);
        const int cnt = g < p.n_routed ? p.offsets[g + 1] - p.offsets[g] : p.shared_rows;
        const uint32_t idesc =
            (kHalfTiles && p.half_tails && cnt - m_blk * BMT <= BMT / 2) ? kIdescHalf : kIdesc;
        if (!mbar_wait(&tempty[acc], aph ^ 1, s_abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, s_abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * L::kStageA);
          const uint32_t b0 = smem_u32(sB + stage * L::kStageB);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            mma_bf16_pair(d_tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                          (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit_pair_both(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) mma_commit_pair_both(&tfull[acc]);
      }
      if (!ok) {
        mma_commit_pair_local(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // ================= epilogue (warps 2..5 of both CTAs) =================
    const int q = warp & 3;
    uint8_t* stg = staging + (warp - 2) * kStagingPerWarp;
    const uint32_t tempty_first = map_to_cta(smem_u32(&tempty[0]), 0);
    int it = 0;
    for (int tile = pair; tile < total; tile += npairs, ++it) {
      int g, m_blk, n_blk;
      decode_tile<BMT, BN>(tile, s_start, G, nt, g, m_blk, n_blk, p.band);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const bool ready = mbar_wait(&tfull[acc], aph, s_abort, p.status);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const bool sh = g >= p.n_routed;
      const int cnt = sh ? p.shared_rows : p.offsets[g + 1] - p.offsets[g];
      const int64_t out_row0 = (int64_t)(sh ? p.shared_out_row0 : p.offsets[g]) + m_blk * BMT;
      const int rows_valid = min(BMT, cnt - m_blk * BMT);
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      // a half tile's accumulator (M = 128 across the pair) holds CTA r's 64 rows twice over
      // the lanes: lane m has row 64 r + m for output columns 0..127, lane 64 + m the same row
      // for columns 128..255, both at TMEM columns 0..127.  Warp q drains lanes 32 q .. + 31:
      // rows 64 r + 32 (q & 1) + lane, output columns 128 (q >> 1) .. + 127 (two chunks).
      const bool half = kHalfTiles && p.half_tails && rows_valid <= BMT / 2;
      const int row_base = half ? (int)rank * 64 + (q & 1) * 32 : (int)rank * 128 + q * 32;
      void* out = (sh && p.out_shared != nullptr) ? p.out_shared : p.out;
      epilogue_warp<BN, EPI>(p, out, t_row, stg, lane, n_blk, out_row0, row_base, rows_valid, [&] {
                               tc_fence_before();
                               __syncwarp();
                               if (lane == 0) mbar_arrive_cluster(tempty_first + 8u * (uint32_t)acc);
                             },
                             half ? 2 : -1, half ? (q >> 1) * 128 : 0);
    }
  }

  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still signal its barriers
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(2 * BN));
  }
}

// ---- token-in-N ("swapped") variant ---------------------------------------------------------
// Groups of a few hundred rows leave most of a 128-row M tile idle in their last tile.  This
// variant puts the weights in the MMA's M dimension and the group's rows in N, which tcgen05
// takes in steps of 16:  D[w][t] = sum_k W[w][k] X[t][k].  A tile is (group, weight block,
// up to 256 of the group's rows).  The weight block is one 128-row M operand built from two
// 64-row TMA boxes: the gate rows f0..f0+63 and the up rows F+f0..F+f0+63 for SwiGLU, or
// output columns o0..o0+127 otherwise.  Per MMA the tensor core reads the same operand bytes
// as the 128x256 tile of the 1-SM kernel.  For SwiGLU the up warps (TMEM lanes 64-127) pass
// their values through shared memory to the gate warps (lanes 0-63), which apply the
// activation.  The epilogue transposes 32x32 blocks through shared memory so that
// out[row][feature] is written with coalesced 16-byte stores.  Tiles inside a group run
// weight block outer, row block inner.
constexpr int kSwapRows = 256;      // group rows per tile (MMA N <= 256)
constexpr int kSwapBox = 128;       // rows per TMA box of the N operand
constexpr int kSwapWBox = 64;       // rows per TMA box of the weight operand
constexpr int kSwapStageW = 128 * BK * 2;          // the 128-row weight operand (16 KB)
constexpr int kSwapStageX = kSwapRows * BK * 2;    // up to 256 group rows (32 KB)
constexpr int kSwapStagingPerWarp = 32 * 64;       // 32 rows x 32 bf16 features
// SwiGLU exchange, per chunk of 32 rows and per gate/up warp pair: the gate warp's values of
// rows 16..31 and the up warp's values of rows 0..15 (fp32), double-buffered over chunks
constexpr int kSwapXchg = 2 * 2 * 2 * 16 * 32 * 4;

template <int STAGES>
struct LayoutSwap {
  static constexpr int kStage = kSwapStageW + kSwapStageX;
  static constexpr int kOffStaging = STAGES * kStage;
  static constexpr int kOffXchg = kOffStaging + 4 * kSwapStagingPerWarp;
  static constexpr int kOffBar = kOffXchg + kSwapXchg;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffStart = kOffMisc + 16;
  static size_t bytes(int groups) { return 1024 + kOffStart + 4 * (size_t)(groups + 1); }
};

// Tile -> (group, weight block, row block).  Inside a group the smaller panel stays resident
// in L2 while the other streams: a group with more rows than weight rows (w_rows) runs row
// blocks outer and weight blocks inner, any other group the reverse.
__device__ __forceinline__ void decode_tile_swap(int tile, const int* s_start, int G, int nw,
                                                 int w_rows, int& g, int& w_blk, int& r_blk) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_start[mid] <= tile) lo = mid; else hi = mid;
  }
  g = lo;
  const int r = tile - s_start[g];
  const int rt = (s_start[g + 1] - s_start[g]) / nw;
  if (rt * kSwapRows > w_rows) {
    r_blk = r / nw;
    w_blk = r - r_blk * nw;
  } else {
    w_blk = r / rt;
    r_blk = r - w_blk * rt;
  }
}

// Named barrier over the four epilogue warps (id 1; id 0 is __syncthreads).
__device__ __forceinline__ void epilogue_bar() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// The same barrier, returning whether any of the 128 threads passed true: the four warps
// take the same exit decision before they meet at epilogue_bar().
__device__ __forceinline__ bool epilogue_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

template <int EPI, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmX,
                             const __grid_constant__ CUtensorMap tmXs,
                             const __grid_constant__ CUtensorMap tmW, const Args p) {
  pdl_wait();
  using L = LayoutSwap<STAGES>;
  constexpr int kOutPerTile = (EPI == kEpiSwiglu) ? 64 : 128;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* staging = smem + L::kOffStaging;
  float* xchg = reinterpret_cast<float*>(smem + L::kOffXchg);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  int* s_start = reinterpret_cast<int*>(smem + L::kOffStart);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.n_routed + p.has_shared;
  const int nw = (p.n_out + kOutPerTile - 1) / kOutPerTile;
  const int w_rows = EPI == kEpiSwiglu ? 2 * p.n_out : p.n_out;
  const int nk = (p.K + BK - 1) / BK;
  auto group_rows = [&](int g) {
    return g < p.n_routed ? p.offsets[g + 1] - p.offsets[g] : p.shared_rows;
  };

  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int g0 = min(lane * per, G), g1 = min(g0 + per, G);
    int local = 0;
    for (int g = g0; g < g1; ++g) local += ((group_rows(g) + kSwapRows - 1) / kSwapRows) * nw;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int g = g0; g < g1; ++g) {
      s_start[g] = run;
      run += ((group_rows(g) + kSwapRows - 1) / kSwapRows) * nw;
    }
    if (lane == 31) s_start[G] = incl;
    if (lane == 0) {
      for (int i = 0; i < STAGES; ++i) {
        mbar_init(&full[i], 1);
        mbar_init(&empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&tfull[i], 1);
        mbar_init(&tempty[i], 128);
      }
      mbar_init(drain, 1);
      *s_abort = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  } else if (warp == 1) {
    // two accumulator buffers of up to 256 columns: 512 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(s_tmem)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = s_start[G];

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int armed = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        int g, w_blk, r_blk;
        decode_tile_swap(tile, s_start, G, nw, w_rows, g, w_blk, r_blk);
        const bool sh = g >= p.n_routed;
        const int rows = min(kSwapRows, group_rows(g) - r_blk * kSwapRows);
        const int boxes = (rows + kSwapBox - 1) / kSwapBox;
        const int x_row = (sh ? p.shared_a_row0 : p.offsets[g]) + r_blk * kSwapRows;
        const CUtensorMap* mX = sh ? &tmXs : &tmX;
        const int w_row0 = w_blk * kOutPerTile;
        const int w_row1 = EPI == kEpiSwiglu ? p.up_row0 + w_blk * 64 : w_row0 + 64;
        const uint32_t bytes = (uint32_t)(kSwapStageW + boxes * kSwapBox * BK * 2);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, p.status)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * L::kStage;
          mbar_expect_tx(&full[stage], bytes);
          tma_load_3d(st, &tmW, &full[stage], kb * BK, w_row0, g);
          tma_load_3d(st + kSwapWBox * BK * 2, &tmW, &full[stage], kb * BK, w_row1, g);
          for (int b = 0; b < boxes; ++b)
            tma_load_2d(st + kSwapStageW + b * kSwapBox * BK * 2, mX, &full[stage], kb * BK,
                        x_row + b * kSwapBox);
          ++armed;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      pdl_release();
      if (!ok) {
        for (int i = 0; i < STAGES && i < armed; ++i) {
          stage = (stage + STAGES - 1) % STAGES;
          if (stage == STAGES - 1) phase ^= 1;
          mbar_drain(&full[stage], phase);
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        int g, w_blk, r_blk;
        decode_tile_swap(tile, s_start, G, nw, w_rows, g, w_blk, r_blk);
        const int rows = min(kSwapRows, group_rows(g) - r_blk * kSwapRows);
        const int n_mma = (rows + 15) & ~15;
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                               ((uint32_t)(n_mma >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1, s_abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, s_abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t s0 = smem_u32(smem + stage * L::kStage);
          const uint32_t x0 = s0 + kSwapStageW;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16(d0, sw128_desc(s0 + kk * 32), sw128_desc(x0 + kk * 32), idesc,
                     (kb | kk) != 0 ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) mma_commit(&tfull[acc]);
      }
      if (!ok) {
        mma_commit(drain);
        mbar_drain(drain, 0);
      }
    }
  } else {
    // ================= epilogue (warps 2..5) =================
    const int q = warp & 3;  // TMEM lanes 32q..32q+31 = weight rows 32q + lane of the operand
    uint8_t* stg = staging + (warp - 2) * kSwapStagingPerWarp;
    __nv_bfloat16* stg_h = reinterpret_cast<__nv_bfloat16*>(stg);
    // SwiGLU: warp q = 0, 1 holds the gate rows of features f0 + 32q + lane, warp q + 2 their up
    // rows.  Per chunk of 32 group rows the gate warp computes rows 0..15 and the up warp rows
    // 16..31; each passes the other the half it needs through xchg.
    const bool up_warp = EPI == kEpiSwiglu && q >= 2;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      int g, w_blk, r_blk;
      decode_tile_swap(tile, s_start, G, nw, w_rows, g, w_blk, r_blk);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const bool ready = mbar_wait(&tfull[acc], aph, s_abort, p.status);
      // the four warps take the same exit decision (they meet at named barriers below), and
      // this barrier also separates the previous tile's exchange reads from this tile's writes
      if (epilogue_any(!ready)) break;
      tc_fence_after();
      const bool sh = g >= p.n_routed;
      const int rows = min(kSwapRows, group_rows(g) - r_blk * kSwapRows);
      const int64_t out_row0 =
          (int64_t)(sh ? p.shared_out_row0 : p.offsets[g]) + (int64_t)r_blk * kSwapRows;
      __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(
          (sh && p.out_shared != nullptr) ? p.out_shared : p.out);
      const int chunks = (rows + 31) / 32;
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
      for (int c = 0; c < chunks; ++c) {
        float v[32];
        tmem_ld32(t_row + c * 32, v);
        tmem_ld_wait();
        if (c == chunks - 1) {
          // every TMEM read of this accumulator is done: hand it back to the MMA warp
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
        }
        int r0 = 0, nr = 32;  // this warp's rows of the chunk
        if constexpr (EPI == kEpiSwiglu) {
          float* xb = xchg + ((c & 1) * 2 + (q & 1)) * 1024;  // [gate 16..31 | up 0..15]
          if (!up_warp) {
#pragma unroll
            for (int i = 0; i < 16; ++i) xb[i * 32 + lane] = v[16 + i];
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) xb[512 + i * 32 + lane] = v[i];
          }
          epilogue_bar();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float gg = up_warp ? xb[i * 32 + lane] : v[i];
            float uu = up_warp ? v[16 + i] : xb[512 + i * 32 + lane];
            if (p.clamp > 0.f) {
              gg = fminf(fmaxf(gg, -p.clamp), p.clamp);
              uu = fminf(fmaxf(uu, -p.clamp), p.clamp);
            }
            v[i] = silu_f(gg) * uu;
          }
          r0 = up_warp ? 16 : 0;
          nr = 16;
        } else if (EPI == kEpiRelu) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = fmaxf(v[i], 0.f);
        }
        // transpose: staging row r holds the warp's 32 features of group row c*32 + r0 + r
        // (64-byte rows: the stores below and the 16-byte reads are conflict-free)
#pragma unroll
        for (int r = 0; r < 32; ++r)
          if (r < nr) stg_h[r * 32 + lane] = __float2bfloat16_rn(v[r]);
        __syncwarp();
        const int feat0 = w_blk * kOutPerTile + (q & (EPI == kEpiSwiglu ? 1 : 3)) * 32;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = i * 8 + (lane >> 2);
          const int piece = lane & 3;
          const int col = feat0 + piece * 8;
          const int grow = c * 32 + r0 + r;
          if (r < nr && grow < rows && col < p.n_out) {
            const uint4 val = *reinterpret_cast<const uint4*>(stg + r * 64 + piece * 16);
            *reinterpret_cast<uint4*>(outp + (out_row0 + grow) * p.ld_out + col) = val;
          }
        }
        __syncwarp();
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(512));
  }
}

// ---- failure-detection self-test --------------------------------------------------------
// One thread waits, with the GEMMs' bounded wait, on an mbarrier that nothing ever completes:
// the wait runs out after limit_ns and records MOE_ERR_TIMEOUT in the status word, as a
// stalled GEMM pipeline would.  out[0] = 1 if the wait (wrongly) succeeded, else 0.
__global__ void wait_selftest_kernel(int* status, uint64_t limit_ns, int* out) {
  pdl_wait();
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const bool ok = mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
  if (out != nullptr) out[0] = ok ? 1 : 0;
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(&bar)) : "memory");
}

// ---- host side -------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor [outer][rows][K] (outer == 0: 2-D [rows][K]); box [box_rows][64], 128B swizzle.
bool make_map(CUtensorMap* m, const void* ptr, int64_t K, int64_t rows, int64_t outer,
              int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)(outer > 0 ? outer : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)(K * rows * 2)};
  cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const cuuint32_t rank = outer > 0 ? 3 : 2;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMaxDev = 64;

int num_sms() {
  static int cached[kMaxDev] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDev) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

int64_t l2_bytes() {
  static int64_t cached[kMaxDev] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDev) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrL2CacheSize, dev);
    cached[dev] = n > 0 ? n : (126LL << 20);
  }
  return cached[dev];
}

// Opt a kernel into the largest dynamic shared memory once per device (the per-launch size is
// always below it), so launches do not repeat the attribute call.  `done` must be distinct
// for every kernel: each launch_* instantiation passes its own.
template <typename Kernel>
cudaError_t allow_max_smem(Kernel kern, bool (&done)[kMaxDev]) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kMaxDev && done[dev]) return cudaSuccess;
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDev) done[dev] = true;
  return e;
}

// 2-SM kernel: half-height tiles for group tails (MOE_B200_2SM_HALF_TAILS=0 turns them off).
bool half_tails_enabled() {
  const char* v = std::getenv("MOE_B200_2SM_HALF_TAILS");
  return !(v != nullptr && std::strcmp(v, "0") == 0);
}

Args make_args(const GroupedGemm& g) {
  Args a;
  a.offsets = g.offsets;
  a.n_routed = g.n_routed;
  a.has_shared = g.has_shared;
  a.shared_rows = (int)g.shared_rows;
  a.shared_a_row0 = (int)g.shared_a_row0;
  a.shared_out_row0 = (int)g.shared_out_row0;
  a.K = g.K;
  a.n_out = g.n_out;
  a.up_row0 = g.n_out;
  a.clamp = g.clamp;
  a.col_bias = g.col_bias;
  a.out = g.out;
  a.out_shared = g.out_shared;
  a.ld_out = g.ld_out;
  a.status = g.status;
  a.k_splits = g.k_splits > 1 ? g.k_splits : 1;
  a.split_rows = g.split_rows;
  const char* m64 = std::getenv("MOE_B200_M64_TAILS");
  a.m64_tails = (m64 != nullptr && std::strcmp(m64, "0") == 0) ? 0 : 1;
  a.half_tails = half_tails_enabled() ? 1 : 0;
  a.band = 0;
  return a;
}

// Bands of M blocks for groups whose A panel outgrows L2 (MOE_B200_BAND: unset or 0 = off,
// 1 = bands of about a third of L2 of A rows, n > 1 = bands of n M blocks).  Only groups
// that run N blocks outer (their B panel at least as large as their A panel) are banded.
int band_for(const GroupedGemm& g, int bmt) {
  const char* v = std::getenv("MOE_B200_BAND");
  if (v == nullptr) return 0;
  const int n = std::atoi(v);
  if (n <= 0) return 0;
  if (n > 1) return n;
  const int64_t tile_bytes = (int64_t)bmt * g.K * 2;
  return (int)std::max<int64_t>(1, l2_bytes() / 3 / tile_bytes);
}

template <int BN, int EPI, int STAGES, int AM = BM>
cudaError_t launch_t(const GroupedGemm& g, const CUtensorMap& mA, const CUtensorMap& mAs,
                     const CUtensorMap& mB, cudaStream_t stream, int grid) {
  auto kern = grouped_gemm_kernel<BN, EPI, STAGES, AM>;
  const size_t smem = Layout<BN, STAGES, AM>::bytes(g.n_routed + g.has_shared);
  static bool done[kMaxDev] = {};
  const cudaError_t e = allow_max_smem(kern, done);
  if (e != cudaSuccess) return e;
  Args a = make_args(g);
  a.band = band_for(g, AM > BM ? AM : BM);
  launch_pdl(kern, grid, kThreads, smem, stream, mA, mAs, mB, a);
  return cudaGetLastError();
}

template <int EPI, int STAGES>
cudaError_t launch_2sm(const GroupedGemm& g, const CUtensorMap& mA, const CUtensorMap& mAs,
                       const CUtensorMap& mB, cudaStream_t stream, int pairs) {
  auto kern = grouped_gemm_2sm_kernel<EPI, STAGES>;
  const size_t smem = Layout2<STAGES>::bytes(g.n_routed + g.has_shared);
  static bool done[kMaxDev] = {};
  const cudaError_t e = allow_max_smem(kern, done);
  if (e != cudaSuccess) return e;
  Args a = make_args(g);
  a.band = band_for(g, 256);
  launch_pdl(kern, 2 * pairs, kThreads, smem, stream, mA, mAs, mB, a);
  return cudaGetLastError();
}

template <int EPI, int STAGES>
cudaError_t launch_swap(const GroupedGemm& g, const CUtensorMap& mX, const CUtensorMap& mXs,
                        const CUtensorMap& mW, cudaStream_t stream, int grid) {
  auto kern = grouped_gemm_swap_kernel<EPI, STAGES>;
  const size_t smem = LayoutSwap<STAGES>::bytes(g.n_routed + g.has_shared);
  static bool done[kMaxDev] = {};
  const cudaError_t e = allow_max_smem(kern, done);
  if (e != cudaSuccess) return e;
  launch_pdl(kern, grid, kThreads, smem, stream, mX, mXs, mW, make_args(g));
  return cudaGetLastError();
}

// Which kernel a bf16 grouped GEMM uses.  The 2-SM kernel tiles 256 rows per group, so it
// pays off only when groups are large, and there only for the down projection: for gate/up it
// ran no faster than the 1-SM kernel while reading its operands from DRAM 2.6x over (5.75 GB vs
// 2.20 GB on the 16384-token Mixtral-shaped layer), where the 1-SM kernel reads each byte once.
// Small groups keep the 1-SM kernel's 128-row tiles.
// MOE_B200_GEMM_PATH=1sm|1sm128|2sm|swap overrides the choice (the tests cover every kernel).
const char* path_override() { return std::getenv("MOE_B200_GEMM_PATH"); }

// Average rows of a routed group, as the caller estimates it (the true sizes stay on the
// device).  The token-in-N kernel is taken only on request (MOE_B200_GEMM_PATH=swap): it
// pads a DeepSeek-V3-shaped prefill to 1.02x the MMA rows where 128-row tiles pad to 1.20x,
// yet measured 17-20 % slower there (and 6 % slower on the capacity configs), so the
// automatic choice keeps the 1-SM and 2-SM kernels.
constexpr int64_t kSwapMaxRows = 0;

int64_t avg_group_rows(const GroupedGemm& g) {
  if (g.rows_per_group_hint >= 0) return g.rows_per_group_hint;
  return g.n_routed > 0 ? g.max_rows_routed / g.n_routed : g.shared_rows;
}

bool use_swap(const GroupedGemm& g) {
  if (g.epilogue == kEpiStoreF32 || g.k_splits > 1) return false;
  if (const char* env = path_override()) {
    if (std::strcmp(env, "swap") == 0) return true;
    if (std::strncmp(env, "1sm", 3) == 0 || std::strcmp(env, "2sm") == 0) return false;
  }
  return g.n_routed > 0 && avg_group_rows(g) < kSwapMaxRows;
}

// Rows of a group as the 1-SM kernel computes them: 128-row tiles, the last one an M = 64
// tile when it holds at most 64 rows.
int64_t one_sm_rows(int64_t r) {
  const int64_t full = r / BM * BM, rem = r - full;
  return full + (rem == 0 ? 0 : rem <= 64 ? 64 : BM);
}

// The 2-SM kernel (256-row tiles, each SM staging half of B) moves two thirds of the 1-SM
// kernel's operand bytes from L2 to the SMs per FLOP, and L2-to-SM bandwidth is what keeps
// the 1-SM kernel's tensor pipe from running full (its 128x256 tile needs about 96 B per
// clock per SM, the 2-SM tile 64), but it computes more padding rows: a routed group of r
// rows takes ceil(r / 256) tiles of 256 rows there, against 128-row tiles with an M = 64 last
// tile on the 1-SM kernel, 96 more rows on average when r is spread evenly modulo 256.  It is taken when that padding is at most a quarter of the
// rows, estimated from the caller's rows per group.  Measured on one B200: the capacity and
// Switch layers (padding estimate 1/8 and 3/16) gain 2-6 % per step, the Mixtral-shaped down
// projection (1/64 to 3/32) gains, and the V3/V4.1-shaped prefill (1/3) loses.  For gate/up
// the weight panel of one expert must also fit in a quarter of L2: with the Mixtral-shaped
// 235 MB panels the 2-SM kernel missed L2 more (2.99 vs 1.95 GB from DRAM at 4096 tokens)
// and was 0-9 % slower, while the 1-SM kernel reads each weight byte once.
bool use_two_sm(const GroupedGemm& g) {
  if (g.epilogue == kEpiStoreF32 || g.k_splits > 1) return false;
  if (const char* env = path_override()) {
    if (std::strncmp(env, "1sm", 3) == 0 || std::strcmp(env, "tall") == 0) return false;
    if (std::strcmp(env, "2sm") == 0) return true;
  }
  const int64_t routed = g.n_routed > 0 ? avg_group_rows(g) * g.n_routed : 0;
  const int64_t shared = g.has_shared ? g.shared_rows : 0;
  if (routed + shared <= 0) return false;
  // a group's last tile pads to 256 rows against 128 (64 with an M = 64 tile) on the 1-SM
  // kernel: on average 96 more rows per group.  (Half tiles, where the 2-SM kernel runs an
  // elementwise epilogue, cut that to 32, but at the ridge-point layers the 1-SM kernel still
  // won with them -- V4.1-shaped prefill 9.47 vs 9.71-9.86 ms -- so the estimate keeps 96.)
  int64_t extra = 96LL * g.n_routed;
  if (shared > 0) extra += (shared + 255) / 256 * 256 - one_sm_rows(shared);
  if (4 * extra > routed + shared) return false;
  if (g.epilogue == kEpiStoreBf16) return true;
  return (int64_t)g.rows_b * g.K * 2 <= l2_bytes() / 4;
}

// Tall tiles (1-SM kernel, 256x256), on request only (MOE_B200_GEMM_PATH=tall): two M = 128
// MMAs per k-step share one B stage, so a stage of 64 KB feeds 1024 MMA cycles where a 48 KB
// stage of the 128x256 tile feeds 512, and the operands cross from shared memory at 64 B per
// clock instead of 96.  A tile with at most 128 rows issues only the first MMA (and loads
// only the first A box), so groups pad exactly as on the 128-row tiles.  Measured slower or
// level everywhere: the V3/V4.1-shaped prefill gate/up 4.53 -> 5.91 ms and 5.85 -> 7.86 ms
// (its many short groups get 3 stages of weights in flight instead of 4), the Mixtral-shaped
// 16384-token step 9.45 ms either way (9.66 with tall gate/up and the 2-SM down).
bool use_tall(const GroupedGemm& g) {
  if (g.epilogue == kEpiStoreF32 || g.k_splits > 1) return false;
  const char* env = path_override();
  return env != nullptr && std::strcmp(env, "tall") == 0;
}

// N width of the 1-SM kernel's tiles.  256 keeps the tensor pipe busiest; when nearly every
// group fits one 128-row tile the launch streams weights (memory-bound) and the tile count
// is small, so 128-wide tiles are taken when they leave a clearly smaller idle tail on the
// last wave.  MOE_B200_GEMM_PATH=1sm128 forces 128.
int pick_bn_1sm(const GroupedGemm& g) {
  if (const char* env = path_override())
    if (std::strcmp(env, "1sm128") == 0) return 128;
  const int groups = g.n_routed + g.has_shared;
  const int64_t rows = (g.n_routed > 0 ? g.max_rows_routed : 0) + (g.has_shared ? g.shared_rows : 0);
  if (rows >= 128LL * groups) return 256;
  int64_t mtiles = std::min<int64_t>(g.n_routed, g.max_rows_routed);
  if (g.has_shared) mtiles += (g.shared_rows + BM - 1) / BM;
  auto tail_eff = [&](int bn) {
    const int out = g.epilogue == kEpiSwiglu ? bn / 2 : bn;
    const double waves = (double)(mtiles * ((g.n_out + out - 1) / out)) / num_sms();
    return waves / std::ceil(waves);
  };
  return tail_eff(128) > tail_eff(256) + 0.02 ? 128 : 256;
}

// 64-row tiles: groups are cut into 64-row output tiles, each running M = 64 MMAs, so a stage
// holds 64 A rows and the freed shared memory holds more stages of weights (more weight bytes
// in flight per SM).  Taken when every group fits one such tile (the caller's bound on a
// routed group, and the shared group): decode-sized batches.  With larger groups it lost
// badly (Mixtral-shaped, 256 tokens, about 64 rows per expert: 0.503 -> 0.587 ms per step;
// 4096 tokens: 2.36 -> 3.09 ms): the weights of a group are then read by two M tiles and the
// M = 64 MMAs halve the rows per instruction.
// MOE_B200_DECODE_A64=0 turns it off; =2 forces it on any group sizes (tests).
bool use_a64(const GroupedGemm& g) {
  if (g.epilogue == kEpiStoreF32 || g.k_splits > 1 || use_swap(g) || use_two_sm(g) ||
      use_tall(g))
    return false;
  const char* v = std::getenv("MOE_B200_DECODE_A64");
  if (v != nullptr && v[0] == '0') return false;
  if (v != nullptr && v[0] == '2') return true;
  if (g.has_shared && g.shared_rows > 64) return false;
  if (g.n_routed > 0 && (g.max_group_rows <= 0 || g.max_group_rows > 64)) return false;
  return true;
}

}  // namespace tc

cudaError_t launch_wait_selftest(int* status, uint64_t limit_ns, int* out, cudaStream_t stream,
                                 int* launches) {
  ++*launches;
  launch_pdl(tc::wait_selftest_kernel, 1, 32, 0, stream, status, limit_ns, out);
  return cudaGetLastError();
}

// N width of the fp32-store (router) tiles: the fewest padded columns, then the wider tile.
int router_tile_n(int n_out) {
  if (n_out <= 32) return 32;
  if (n_out <= 64) return 64;
  if (n_out <= 128) return 128;
  if (n_out <= 192) return 192;
  int best = 256;
  int64_t best_cols = (n_out + 255) / 256 * 256;
  for (int bn : {192, 128}) {
    const int64_t cols = (int64_t)(n_out + bn - 1) / bn * bn;
    if (cols < best_cols) {
      best = bn;
      best_cols = cols;
    }
  }
  return best;
}

// The kernel launch_grouped_gemm takes for g, by the same host-side decisions in the same
// order (device attributes only; no device memory is touched).
const char* grouped_gemm_kernel_name(const GroupedGemm& g) {
  using namespace tc;
  if (g.n_routed + g.has_shared == 0) return "none";
  if (use_swap(g)) return "grouped_gemm_swap_kernel (token-in-N)";
  if (g.epilogue == kEpiStoreF32) {
    switch (router_tile_n(g.n_out)) {
      case 32: return "grouped_gemm_kernel (1-SM, 128x32 fp32 tiles)";
      case 64: return "grouped_gemm_kernel (1-SM, 128x64 fp32 tiles)";
      case 128: return "grouped_gemm_kernel (1-SM, 128x128 fp32 tiles)";
      case 192: return "grouped_gemm_kernel (1-SM, 128x192 fp32 tiles)";
      default: return "grouped_gemm_kernel (1-SM, 128x256 fp32 tiles)";
    }
  }
  if (use_two_sm(g)) return "grouped_gemm_2sm_kernel (2-SM, 256x256 tiles)";
  if (use_tall(g)) return "grouped_gemm_kernel (1-SM, 256x256 tiles)";
  if (use_a64(g))
    return pick_bn_1sm(g) == 128 ? "grouped_gemm_kernel (1-SM, 64x128 tiles)"
                                 : "grouped_gemm_kernel (1-SM, 64x256 tiles)";
  return pick_bn_1sm(g) == 128 ? "grouped_gemm_kernel (1-SM, 128x128 tiles)"
                               : "grouped_gemm_kernel (1-SM, 128x256 tiles)";
}

cudaError_t launch_grouped_gemm(const GroupedGemm& g, cudaStream_t stream, int* launches,
                                const char** why) {
  using namespace tc;
  const int groups = g.n_routed + g.has_shared;
  if (groups == 0) return cudaSuccess;
  if (use_swap(g)) {
    CUtensorMap mX, mXs, mW;
    const void* x_ptr = g.a != nullptr ? g.a : g.a_shared;
    const int64_t x_rows = g.a != nullptr ? g.rows_a : g.rows_a_shared;
    if (!make_map(&mX, x_ptr, g.K, std::max<int64_t>(x_rows, 1), 0, kSwapBox) ||
        !make_map(&mXs, g.a_shared != nullptr ? g.a_shared : x_ptr, g.K,
                  std::max<int64_t>(g.a_shared != nullptr ? g.rows_a_shared : x_rows, 1), 0,
                  kSwapBox) ||
        !make_map(&mW, g.b, g.K, g.rows_b, g.groups_b, kSwapWBox)) {
      *why = "cuTensorMapEncodeTiled failed (pointer alignment, strides or driver entry point)";
      return cudaErrorInvalidValue;
    }
    const int out_per_tile = g.epilogue == kEpiSwiglu ? 64 : 128;
    const int64_t nw = (g.n_out + out_per_tile - 1) / out_per_tile;
    int64_t rtiles = 0;
    if (g.n_routed > 0) rtiles += (g.max_rows_routed + kSwapRows - 1) / kSwapRows + g.n_routed;
    if (g.has_shared) rtiles += (g.shared_rows + kSwapRows - 1) / kSwapRows;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), rtiles * nw));
    ++*launches;
    switch (g.epilogue) {
      case kEpiSwiglu: return launch_swap<kEpiSwiglu, 4>(g, mX, mXs, mW, stream, grid);
      case kEpiRelu: return launch_swap<kEpiRelu, 4>(g, mX, mXs, mW, stream, grid);
      default: return launch_swap<kEpiStoreBf16, 4>(g, mX, mXs, mW, stream, grid);
    }
  }
  int BN;
  const bool two_sm = use_two_sm(g);
  const bool tall = !two_sm && use_tall(g);
  if (g.epilogue == kEpiStoreF32) {
    BN = router_tile_n(g.n_out);
  } else {
    BN = (two_sm || tall) ? 256 : pick_bn_1sm(g);
  }
  const int box_b = two_sm ? 128 : (g.epilogue == kEpiSwiglu) ? BN / 2 : BN;
  const bool a64 = use_a64(g);
  const int box_a = a64 ? 64 : BM;
  CUtensorMap mA, mAs, mB;
  const void* a_ptr = g.a != nullptr ? g.a : g.a_shared;
  const int64_t a_rows = g.a != nullptr ? g.rows_a : g.rows_a_shared;
  if (!make_map(&mA, a_ptr, g.K, std::max<int64_t>(a_rows, 1), 0, box_a) ||
      !make_map(&mAs, g.a_shared != nullptr ? g.a_shared : a_ptr, g.K,
                std::max<int64_t>(g.a_shared != nullptr ? g.rows_a_shared : a_rows, 1), 0, box_a) ||
      !make_map(&mB, g.b, g.K, g.rows_b, g.groups_b, box_b)) {
    *why = "cuTensorMapEncodeTiled failed (pointer alignment, strides or driver entry point)";
    return cudaErrorInvalidValue;
  }
  // grid: at most one CTA per SM, no more than an upper bound of the tile count
  const int out_per_tile = (g.epilogue == kEpiSwiglu) ? BN / 2 : BN;
  const int64_t nt = (g.n_out + out_per_tile - 1) / out_per_tile;
  const int tm = a64 ? 64 : tall ? 256 : BM;  // rows of an output tile
  int64_t mtiles = 0;
  if (g.n_routed > 0) mtiles += (g.max_rows_routed + tm - 1) / tm + g.n_routed;
  if (g.has_shared) mtiles += (g.shared_rows + tm - 1) / tm;
  const int64_t bound = mtiles * nt * std::max(1, g.k_splits);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), bound));
  ++*launches;
  if (two_sm) {
    int64_t mt2 = 0;
    if (g.n_routed > 0) mt2 += (g.max_rows_routed + 255) / 256 + g.n_routed;
    if (g.has_shared) mt2 += (g.shared_rows + 255) / 256;
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms() / 2, mt2 * nt));
    switch (g.epilogue) {
      case kEpiSwiglu: return launch_2sm<kEpiSwiglu, 6>(g, mA, mAs, mB, stream, pairs);
      case kEpiRelu: return launch_2sm<kEpiRelu, 6>(g, mA, mAs, mB, stream, pairs);
      default: return launch_2sm<kEpiStoreBf16, 6>(g, mA, mAs, mB, stream, pairs);
    }
  }
  if (tall) {
    // 256-row tiles: 3 stages of 64 KB
    switch (g.epilogue) {
      case kEpiSwiglu: return launch_t<256, kEpiSwiglu, 3, 256>(g, mA, mAs, mB, stream, grid);
      case kEpiRelu: return launch_t<256, kEpiRelu, 3, 256>(g, mA, mAs, mB, stream, grid);
      default: return launch_t<256, kEpiStoreBf16, 3, 256>(g, mA, mAs, mB, stream, grid);
    }
  }
  if (a64) {
    // 64-row A stages: 8 stages of 24 KB (128-wide tiles) or 5 of 40 KB (256-wide)
    if (BN == 128) {
      switch (g.epilogue) {
        case kEpiSwiglu: return launch_t<128, kEpiSwiglu, 8, 64>(g, mA, mAs, mB, stream, grid);
        case kEpiRelu: return launch_t<128, kEpiRelu, 8, 64>(g, mA, mAs, mB, stream, grid);
        default: return launch_t<128, kEpiStoreBf16, 8, 64>(g, mA, mAs, mB, stream, grid);
      }
    }
    switch (g.epilogue) {
      case kEpiSwiglu: return launch_t<256, kEpiSwiglu, 5, 64>(g, mA, mAs, mB, stream, grid);
      case kEpiRelu: return launch_t<256, kEpiRelu, 5, 64>(g, mA, mAs, mB, stream, grid);
      default: return launch_t<256, kEpiStoreBf16, 5, 64>(g, mA, mAs, mB, stream, grid);
    }
  }
  if (BN == 128 && g.epilogue != kEpiStoreF32) {
    switch (g.epilogue) {
      case kEpiSwiglu: return launch_t<128, kEpiSwiglu, 6>(g, mA, mAs, mB, stream, grid);
      case kEpiRelu: return launch_t<128, kEpiRelu, 6>(g, mA, mAs, mB, stream, grid);
      default: return launch_t<128, kEpiStoreBf16, 6>(g, mA, mAs, mB, stream, grid);
    }
  }
  switch (g.epilogue) {
    case kEpiSwiglu: return launch_t<256, kEpiSwiglu, 4>(g, mA, mAs, mB, stream, grid);
    case kEpiRelu: return launch_t<256, kEpiRelu, 4>(g, mA, mAs, mB, stream, grid);
    case kEpiStoreBf16: return launch_t<256, kEpiStoreBf16, 4>(g, mA, mAs, mB, stream, grid);
    case kEpiStoreF32:
      switch (BN) {
        case 32: return launch_t<32, kEpiStoreF32, 8>(g, mA, mAs, mB, stream, grid);
        case 64: return launch_t<64, kEpiStoreF32, 8>(g, mA, mAs, mB, stream, grid);
        case 128: return launch_t<128, kEpiStoreF32, 6>(g, mA, mAs, mB, stream, grid);
        case 192: return launch_t<192, kEpiStoreF32, 5>(g, mA, mAs, mB, stream, grid);
        default: return launch_t<256, kEpiStoreF32, 4>(g, mA, mAs, mB, stream, grid);
      }
  }
  *why = "unknown epilogue";
  return cudaErrorInvalidValue;
}

}  // namespace moe
