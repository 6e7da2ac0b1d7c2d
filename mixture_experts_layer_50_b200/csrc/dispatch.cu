// Capacity, token dropping and the permutation into per-expert contiguous groups.
//
// "Mixture-of-Experts : routage et capacité" slides, "L'idée — Capacité" and "Cas guidé —
// trace complète": an expert serves its assignments in arrival (token) order, keeps the
// first C and drops the rest; "Support visuel — Capacité" lays the kept tokens of each
// expert out in that order.  "Основы MoE", "Эксперимент на PyTorch": the per-expert
// gather x[rows] that feeds each expert.
//
// rank(t, e) = #{t' < t : e in ids[t']} is computed without atomics in three passes, so
// every output is a deterministic function of ids:
//   1. one warp per tile of kRankTile tokens walks its tokens in order with per-expert
//      counters in shared memory (local rank) and writes the tile's histogram;
//   2. one block per 32 experts scans the histograms over tiles (tile_base) and applies the
//      capacity to the per-expert totals; the last block to finish scans the capped totals
//      over the experts (offsets);
//   3. one block (or one warp) per token: rank = tile_base + local rank, keep iff rank < C,
//      row = offsets[e] + rank; the token's x row is copied to each kept row (the gather).
#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// Where the gather writes the kept row `row` (compact per-expert layout, `off` = its
// expert's first row): into xp, or with kRemote straight into the destination of its expert
// e -- row rem.row0[e] + (row - off) of the buffer at rem.base[e] (another device's receive
// buffer reached through peer memory, or a local one); null (reported) past that buffer.
template <bool kRemote, typename V>
__device__ __forceinline__ V* gather_dst(V* xp, const RemoteRows& rem, int e, int32_t row,
                                         int32_t off, int row_vecs) {
  if constexpr (kRemote) {
    const int64_t d = (int64_t)rem.row0[e] + (row - off);
    if (d < 0 || d >= rem.rows[e]) {
      if (rem.status != nullptr) report_status(rem.status, kStatusInvalidInput);
      return nullptr;
    }
    return reinterpret_cast<V*>(rem.base[e]) + d * row_vecs;
  } else {
    return xp + (int64_t)row * row_vecs;
  }
}

__global__ void __launch_bounds__(32) rank_local_kernel(
    const int32_t* __restrict__ ids, const uint8_t* __restrict__ drop_mask, int64_t N, int k,
    int E, int32_t* __restrict__ local_rank, int32_t* __restrict__ tile_hist, int* status) {
  pdl_wait();
  extern __shared__ int32_t smem[];
  int32_t* cnt = smem;       // [E]
  int32_t* sid = smem + E;   // [kRankTile * k]
  const int lane = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * kRankTile;
  const int ntok = (int)min((int64_t)kRankTile, N - t0);
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  bool bad = false;
  for (int i = lane; i < ntok * k; i += 32) {
    int v = ids[t0 * k + i];
    if (v < 0 || v >= E) {
      bad = true;
      v = -1;
    } else if (drop_mask != nullptr && drop_mask[t0 * k + i]) {
      v = -1;
    }
    sid[i] = v;
  }
  __syncwarp();
  bad |= warp_rank_walk(sid, ntok, k, cnt, lane,
                        [&](int t, int j, int r) { local_rank[(t0 + t) * k + j] = r; });
  if (bad) report_status(status, kStatusInvalidInput);
  for (int e = lane; e < E; e += 32) tile_hist[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// Block b scans the tile histograms of experts [32 b, 32 b + 32): lane = expert, warp w = a
// contiguous chunk of tiles.  The per-expert totals give demand and the capped counts; the
// block that arrives last (a ticket taken after its counts are visible) scans the counts over
// the experts into offsets and puts the ticket counter back to 0.  Every output is a fixed
// function of the histograms: only which block does the final scan varies.
__global__ void __launch_bounds__(1024) dispatch_scan_kernel(
    const int32_t* __restrict__ tile_hist, int n_tiles, int E, int64_t C,
    int32_t* __restrict__ tile_base, int32_t* __restrict__ demand,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* arrive,
    const int32_t* __restrict__ cap_e) {
  pdl_wait();
  __shared__ int32_t part[32][33];  // chunk sums [warp][lane]
  __shared__ int32_t warp_tot[32];
  __shared__ bool s_last;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  const bool has_e = e < E;
  const int per = (n_tiles + 31) / 32;
  const int c0 = min(w * per, n_tiles), c1 = min(c0 + per, n_tiles);
  int32_t s = 0;
  if (has_e) {
#pragma unroll 8
    for (int c = c0; c < c1; ++c) s += tile_hist[(int64_t)c * E + e];
  }
  part[w][lane] = s;
  __syncthreads();
  int32_t run = 0, total = 0;
  for (int j = 0; j < 32; ++j) {
    const int32_t v = part[j][lane];
    run += j < w ? v : 0;
    total += v;
  }
  if (has_e) {
#pragma unroll 8
    for (int c = c0; c < c1; ++c) {
      const int32_t v = tile_hist[(int64_t)c * E + e];
      tile_base[(int64_t)c * E + e] = run;
      run += v;
    }
    if (w == 0) {
      demand[e] = total;
      if (cap_e != nullptr)
        counts[e] = min(total, max(cap_e[e], 0));
      else
        counts[e] = (C > 0 && total > C) ? (int32_t)C : total;
      __threadfence();
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int32_t ticket = atomicAdd(arrive, 1);
    s_last = ticket == (int32_t)gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // exclusive scan of counts over the experts (E <= 1024: one expert per thread)
  const int e_me = threadIdx.x;
  const int32_t my_count = e_me < E ? *((volatile const int32_t*)counts + e_me) : 0;
  int32_t incl = my_count;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    int32_t v = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    warp_tot[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  const int32_t excl = incl - my_count + (w > 0 ? warp_tot[w - 1] : 0);
  if (e_me < E) offsets[e_me] = excl;
  if (e_me == E - 1) offsets[E] = excl + my_count;
  if (threadIdx.x == 0) *arrive = 0;
}

// One block per token.  Thread j < k resolves slot j's row with two rounds of loads (local
// rank and expert together, then the expert's tile base and offset together: a local rank
// >= 0 implies a valid expert, set by the rank pass), then the block copies the token's row
// to each kept slot, two vectors in flight per thread.
template <typename V, bool kRemote>
__global__ void __launch_bounds__(128) dispatch_scatter_kernel(
    const int32_t* __restrict__ ids, const int32_t* __restrict__ local_rank,
    const int32_t* __restrict__ tile_base, const int32_t* __restrict__ offsets, int k, int E,
    int64_t C, int32_t* __restrict__ slot_row, int32_t* __restrict__ row_token,
    uint8_t* __restrict__ drop_mask_out, const V* __restrict__ x, V* __restrict__ xp,
    int row_vecs, const int32_t* __restrict__ cap_e, RemoteRows rem) {
  pdl_wait();
  __shared__ int32_t s_row[32];
  __shared__ V* s_dst[32];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    const int j = threadIdx.x;
    const int lr = local_rank[t * k + j];
    const int e_raw = ids[t * k + j];
    const int e = lr >= 0 ? e_raw : 0;
    const int64_t base = tile_base[(t / kRankTile) * E + e];
    const int32_t off = offsets[e];
    int32_t row = -1;
    if (lr >= 0) {
      const int64_t r = base + lr;
      const bool keep = cap_e != nullptr ? r < (int64_t)cap_e[e] : (C <= 0 || r < C);
      if (keep) row = off + (int32_t)r;
    }
    if (slot_row != nullptr) slot_row[t * k + j] = row;
    if (drop_mask_out != nullptr) drop_mask_out[t * k + j] = row < 0 ? 1 : 0;
    if (row >= 0 && row_token != nullptr) row_token[row] = (int32_t)t;
    s_row[j] = row;
    s_dst[j] = row < 0 ? nullptr : gather_dst<kRemote>(xp, rem, e, row, off, row_vecs);
  }
  if (!kRemote && xp == nullptr) return;
  __syncthreads();
  // a token whose slots were all dropped is not read at all
  bool any = false;
  for (int j = 0; j < k; ++j) any |= s_row[j] >= 0;
  if (!any) return;
  const V* src = x + t * row_vecs;
  const int step = blockDim.x;
  for (int v = threadIdx.x; v < row_vecs; v += 2 * step) {
    const bool two = v + step < row_vecs;
    const V a = src[v];
    V b{};
    if (two) b = src[v + step];
    for (int j = 0; j < k; ++j) {
      V* dst = s_dst[j];
      if (dst == nullptr) continue;
      dst[v] = a;
      if (two) dst[v + step] = b;
    }
  }
}

// The same work with one warp per token and kScatterWarps tokens per block: for many tokens
// with small rows it launches 8x fewer blocks and keeps 64 tokens in flight per SM instead of
// 16 (the capacity layer, 16384 tokens of 4 KB rows: 16.5 -> 10.6 us); with few tokens or
// large rows the block-per-token kernel spreads the copies over more SMs and warps.
constexpr int kScatterWarps = 8;
constexpr int kScatterUnroll = 4;

template <typename V, bool kRemote>
__global__ void __launch_bounds__(32 * kScatterWarps, 8) dispatch_scatter_warp_kernel(
    const int32_t* __restrict__ ids, const int32_t* __restrict__ local_rank,
    const int32_t* __restrict__ tile_base, const int32_t* __restrict__ offsets, int64_t N,
    int k, int E, int64_t C, int32_t* __restrict__ slot_row, int32_t* __restrict__ row_token,
    uint8_t* __restrict__ drop_mask_out, const V* __restrict__ x, V* __restrict__ xp,
    int row_vecs, const int32_t* __restrict__ cap_e, RemoteRows rem) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kScatterWarps + (threadIdx.x >> 5);
  if (t >= N) return;  // warp-uniform
  int32_t row = -1;
  V* my_dst = nullptr;
  if (lane < k) {
    const int lr = local_rank[t * k + lane];
    const int e_raw = ids[t * k + lane];
    const int e = lr >= 0 ? e_raw : 0;
    const int64_t base = tile_base[(t / kRankTile) * E + e];
    const int32_t off = offsets[e];
    if (lr >= 0) {
      const int64_t r = base + lr;
      const bool keep = cap_e != nullptr ? r < (int64_t)cap_e[e] : (C <= 0 || r < C);
      if (keep) row = off + (int32_t)r;
    }
    if (slot_row != nullptr) slot_row[t * k + lane] = row;
    if (drop_mask_out != nullptr) drop_mask_out[t * k + lane] = row < 0 ? 1 : 0;
    if (row >= 0 && row_token != nullptr) row_token[row] = (int32_t)t;
    if (row >= 0) my_dst = gather_dst<kRemote>(xp, rem, e, row, off, row_vecs);
  }
  if (!kRemote && xp == nullptr) return;
  if (__ballot_sync(0xffffffffu, row >= 0) == 0u) return;
  const V* src = x + t * row_vecs;
  for (int v0 = 0; v0 < row_vecs; v0 += 32 * kScatterUnroll) {
    V val[kScatterUnroll];
#pragma unroll
    for (int u = 0; u < kScatterUnroll; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < row_vecs) val[u] = src[v];
    }
    for (int j = 0; j < k; ++j) {
      V* dst = reinterpret_cast<V*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_dst), j));
      if (dst == nullptr) continue;
#pragma unroll
      for (int u = 0; u < kScatterUnroll; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < row_vecs) dst[v] = val[u];
      }
    }
  }
}

// The three passes in one launch for a small batch (decode): every block ranks all N*k
// assignments itself (warp 0 walks the tokens in order, as a rank-pass warp walks its tile),
// scans the capped counts over the experts and resolves every slot's row, so that no block
// waits for another; block 0 writes the routing outputs and each block gathers its share of
// the kept rows (slots b, b + gridDim.x, ...).  The results are those of the three passes.
template <typename V, bool kRemote>
__global__ void __launch_bounds__(kSmallDispatchThreads) dispatch_small_kernel(
    const int32_t* __restrict__ ids, const uint8_t* __restrict__ drop_in, int N, int k, int E,
    int64_t C, const int32_t* __restrict__ cap_e, int32_t* __restrict__ demand,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ slot_row,
    int32_t* __restrict__ row_token, uint8_t* __restrict__ drop_mask_out,
    const V* __restrict__ x, V* __restrict__ xp, int row_vecs, int* status, RemoteRows rem) {
  pdl_wait();
  extern __shared__ int32_t sm[];
  int32_t* cnt = sm;                 // [E]
  int32_t* offs = cnt + E;           // [E + 1]
  int32_t* s_id = offs + E + 1;      // [N * k]
  int32_t* s_rank = s_id + N * k;    // [N * k], then the slot's row
  __shared__ int32_t warp_tot[32];
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nk = N * k;
  const bool writer = blockIdx.x == 0;
  if (tid == 0) s_bad = 0;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  for (int i = tid; i < nk; i += blockDim.x) {
    int v = ids[i];
    if (v < 0 || v >= E) {
      s_bad = 1;
      v = -1;
    } else if (drop_in != nullptr && drop_in[i]) {
      v = -1;
    }
    s_id[i] = v;
  }
  __syncthreads();
  if (w == 0) {
    const bool bad = warp_rank_walk(s_id, N, k, cnt, lane,
                                    [&](int t, int j, int r) { s_rank[t * k + j] = r; });
    if (bad && lane == 0) s_bad = 1;
  }
  __syncthreads();
  // capped counts and their exclusive scan over the experts (E <= blockDim.x)
  const int e_me = tid;
  const int32_t dem = e_me < E ? cnt[e_me] : 0;
  int32_t kept = dem;
  if (e_me < E) {
    if (cap_e != nullptr) kept = min(dem, max(cap_e[e_me], 0));
    else if (C > 0 && dem > C) kept = (int32_t)C;
  }
  int32_t incl = kept;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    int32_t v = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    warp_tot[lane] = v;
  }
  __syncthreads();
  const int32_t excl = incl - kept + (w > 0 ? warp_tot[w - 1] : 0);
  if (e_me < E) {
    offs[e_me] = excl;
    if (writer) {
      demand[e_me] = dem;
      counts[e_me] = kept;
      offsets[e_me] = excl;
    }
    if (e_me == E - 1) {
      offs[E] = excl + kept;
      if (writer) offsets[E] = excl + kept;
    }
  }
  __syncthreads();
  for (int i = tid; i < nk; i += blockDim.x) {
    const int r = s_rank[i];
    const int e = s_id[i];
    int32_t row = -1;
    if (r >= 0) {
      const bool keep = cap_e != nullptr ? r < cap_e[e] : (C <= 0 || r < C);
      if (keep) row = offs[e] + r;
    }
    s_rank[i] = row;
    if (writer) {
      if (slot_row != nullptr) slot_row[i] = row;
      if (drop_mask_out != nullptr) drop_mask_out[i] = row < 0 ? 1 : 0;
      if (row >= 0 && row_token != nullptr) row_token[row] = i / k;
    }
  }
  if (writer && tid == 0 && s_bad) report_status(status, kStatusInvalidInput);
  if (!kRemote && xp == nullptr) return;
  __syncthreads();
  for (int i = blockIdx.x; i < nk; i += gridDim.x) {
    const int32_t row = s_rank[i];
    if (row < 0) continue;
    const V* src = x + (int64_t)(i / k) * row_vecs;
    V* dst = gather_dst<kRemote>(xp, rem, s_id[i], row, offs[s_id[i]], row_vecs);
    if (dst == nullptr) continue;
    for (int v = tid; v < row_vecs; v += blockDim.x) dst[v] = src[v];
  }
}

__global__ void pad_offsets_kernel(int E, int64_t C, int32_t* __restrict__ offsets_pad) {
  pdl_wait();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e <= E) offsets_pad[e] = (int32_t)(e * C);
}

// One block per padded row.
__global__ void __launch_bounds__(128) zero_padding_kernel(
    const int32_t* __restrict__ counts, int64_t C, uint4* __restrict__ xp_pad, int row_vecs,
    int32_t* __restrict__ row_token_pad) {
  pdl_wait();
  const int64_t r = blockIdx.x;
  const int e = (int)(r / C);
  if (r - (int64_t)e * C < counts[e]) return;
  if (threadIdx.x == 0 && row_token_pad != nullptr) row_token_pad[r] = -1;
  for (int v = threadIdx.x; v < row_vecs; v += blockDim.x) xp_pad[r * row_vecs + v] = make_uint4(0, 0, 0, 0);
}

}  // namespace

bool use_small_dispatch(int64_t N, int k, int E) {
  if (N <= 0 || N > kSmallDispatchMaxTokens || N * k > kSmallDispatchMaxSlots) return false;
  const char* v = std::getenv("MOE_B200_SMALL_DISPATCH");
  (void)E;
  return !(v != nullptr && v[0] == '0');
}

cudaError_t launch_dispatch_small(const int32_t* ids, const uint8_t* drop_in, int64_t N, int k,
                                  int E, int64_t C, const int32_t* cap_e, int32_t* demand,
                                  int32_t* counts, int32_t* offsets, int32_t* slot_row,
                                  int32_t* row_token, uint8_t* drop_mask_out, const void* x,
                                  void* xp, int row_bytes, int* status, cudaStream_t stream,
                                  int* launches, const RemoteRows* rem) {
  if (rem != nullptr && row_bytes % 16 != 0) return cudaErrorInvalidValue;
  ++*launches;
  const int nk = (int)(N * k);
  const size_t smem = sizeof(int32_t) * ((size_t)E + (size_t)E + 1 + 2 * (size_t)nk);
  const bool gather = xp != nullptr || rem != nullptr;
  const int grid = gather ? std::max(1, std::min(nk, tc::num_sms())) : 1;
  const RemoteRows none{};
  if (rem != nullptr) {
    launch_pdl(dispatch_small_kernel<uint4, true>, grid, kSmallDispatchThreads, smem, stream,
               ids, drop_in, (int)N, k, E, C, cap_e, demand, counts, offsets, slot_row,
               row_token, drop_mask_out, (const uint4*)x, (uint4*)nullptr, row_bytes / 16,
               status, *rem);
  } else if (xp != nullptr && row_bytes % 16 == 0) {
    launch_pdl(dispatch_small_kernel<uint4, false>, grid, kSmallDispatchThreads, smem, stream,
               ids, drop_in, (int)N, k, E, C, cap_e, demand, counts, offsets, slot_row,
               row_token, drop_mask_out, (const uint4*)x, (uint4*)xp, row_bytes / 16, status,
               none);
  } else {
    launch_pdl(dispatch_small_kernel<uint32_t, false>, grid, kSmallDispatchThreads, smem,
               stream, ids, drop_in, (int)N, k, E, C, cap_e, demand, counts, offsets, slot_row,
               row_token, drop_mask_out, (const uint32_t*)x, (uint32_t*)xp, row_bytes / 4,
               status, none);
  }
  return cudaGetLastError();
}

cudaError_t launch_pad_offsets(int E, int64_t C, int32_t* offsets_pad, cudaStream_t stream,
                               int* launches) {
  ++*launches;
  launch_pdl(pad_offsets_kernel, (E + 1 + 255) / 256, 256, 0, stream, E, C, offsets_pad);
  return cudaGetLastError();
}

cudaError_t launch_zero_padding(const int32_t* counts, int E, int64_t C, void* xp_pad,
                                int row_bytes, int32_t* row_token_pad, cudaStream_t stream,
                                int* launches) {
  const int64_t rows = (int64_t)E * C;
  if (rows == 0) return cudaSuccess;
  ++*launches;
  launch_pdl(zero_padding_kernel, (unsigned)rows, 128, 0, stream, counts, C, (uint4*)xp_pad,
                                                         row_bytes / 16, row_token_pad);
  return cudaGetLastError();
}

cudaError_t launch_rank_local(const int32_t* ids, const uint8_t* drop_mask, int64_t N, int k,
                              int E, int32_t* local_rank, int32_t* tile_hist, int* status,
                              cudaStream_t stream, int* launches) {
  if (N == 0) return cudaSuccess;
  const int64_t tiles = (N + kRankTile - 1) / kRankTile;
  const size_t smem = sizeof(int32_t) * ((size_t)E + (size_t)kRankTile * k);
  ++*launches;  // at most (1024 + kRankTile * 32) ints of shared memory: below the 48 KB default
  launch_pdl(rank_local_kernel, (unsigned)tiles, 32, smem, stream, ids, drop_mask, N, k, E, local_rank,
                                                           tile_hist, status);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_scan(const int32_t* tile_hist, int64_t N, int E, int64_t C,
                                 int32_t* tile_base, int32_t* demand, int32_t* counts,
                                 int32_t* offsets, int32_t* arrive, cudaStream_t stream,
                                 int* launches, const int32_t* cap_e) {
  const int tiles = (int)((N + kRankTile - 1) / kRankTile);
  ++*launches;
  launch_pdl(dispatch_scan_kernel, (E + 31) / 32, 1024, 0, stream, tile_hist, tiles, E, C, tile_base,
                                                           demand, counts, offsets, arrive, cap_e);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_scatter(const int32_t* ids, const int32_t* local_rank,
                                    const int32_t* tile_base, const int32_t* offsets,
                                    int64_t N, int k, int E, int64_t C, int32_t* slot_row,
                                    int32_t* row_token, uint8_t* drop_mask_out,
                                    const void* x, void* xp, int row_bytes,
                                    cudaStream_t stream, int* launches, const int32_t* cap_e,
                                    const RemoteRows* rem) {
  if (N == 0) return cudaSuccess;
  if (rem != nullptr && row_bytes % 16 != 0) return cudaErrorInvalidValue;
  ++*launches;
  const RemoteRows none{};
  // warp per token when the warps fill every SM several times over and a token moves at
  // most 16 KB; else block per token
  const bool per_warp = N >= (int64_t)tc::num_sms() * 64 && (int64_t)k * row_bytes <= 16384;
  if (per_warp) {
    const unsigned grid = (unsigned)((N + kScatterWarps - 1) / kScatterWarps);
    const unsigned block = 32 * kScatterWarps;
    if (rem != nullptr) {
      launch_pdl(dispatch_scatter_warp_kernel<uint4, true>, grid, block, 0, stream, ids,
                 local_rank, tile_base, offsets, N, k, E, C, slot_row, row_token,
                 drop_mask_out, (const uint4*)x, (uint4*)nullptr, row_bytes / 16, cap_e, *rem);
    } else if (xp != nullptr && row_bytes % 16 == 0) {
      launch_pdl(dispatch_scatter_warp_kernel<uint4, false>, grid, block, 0, stream, ids,
                 local_rank, tile_base, offsets, N, k, E, C, slot_row, row_token,
                 drop_mask_out, (const uint4*)x, (uint4*)xp, row_bytes / 16, cap_e, none);
    } else if (xp != nullptr) {
      launch_pdl(dispatch_scatter_warp_kernel<uint32_t, false>, grid, block, 0, stream, ids,
                 local_rank, tile_base, offsets, N, k, E, C, slot_row, row_token,
                 drop_mask_out, (const uint32_t*)x, (uint32_t*)xp, row_bytes / 4, cap_e, none);
    } else {
      launch_pdl(dispatch_scatter_warp_kernel<uint4, false>, grid, block, 0, stream, ids,
                 local_rank, tile_base, offsets, N, k, E, C, slot_row, row_token,
                 drop_mask_out, nullptr, nullptr, 0, cap_e, none);
    }
    return cudaGetLastError();
  }
  if (rem != nullptr) {
    launch_pdl(dispatch_scatter_kernel<uint4, true>, (unsigned)N, 128, 0, stream, ids,
               local_rank, tile_base, offsets, k, E, C, slot_row, row_token, drop_mask_out,
               (const uint4*)x, (uint4*)nullptr, row_bytes / 16, cap_e, *rem);
  } else if (xp != nullptr && row_bytes % 16 == 0) {
    launch_pdl(dispatch_scatter_kernel<uint4, false>, (unsigned)N, 128, 0, stream, ids,
               local_rank, tile_base, offsets, k, E, C, slot_row, row_token, drop_mask_out,
               (const uint4*)x, (uint4*)xp, row_bytes / 16, cap_e, none);
  } else if (xp != nullptr) {
    launch_pdl(dispatch_scatter_kernel<uint32_t, false>, (unsigned)N, 128, 0, stream, ids,
               local_rank, tile_base, offsets, k, E, C, slot_row, row_token, drop_mask_out,
               (const uint32_t*)x, (uint32_t*)xp, row_bytes / 4, cap_e, none);
  } else {
    launch_pdl(dispatch_scatter_kernel<uint4, false>, (unsigned)N, 128, 0, stream, ids,
               local_rank, tile_base, offsets, k, E, C, slot_row, row_token, drop_mask_out,
               nullptr, nullptr, 0, cap_e, none);
  }
  return cudaGetLastError();
}

}  // namespace moe
