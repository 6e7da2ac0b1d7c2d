// Gate-weighted combine back to token order, with the shared expert added.
//
// "Основы MoE", "Как устроен MoE-слой", step 4: y = sum_{i in T} g_i FFN_i(x); the slides
// ("L'idée — Top-k et mélange") add the always-on shared expert with weight 1, outside
// the renormalisation; a slot dropped by the capacity contributes nothing ("Cas guidé").
//
// One block per token; each thread owns 16-byte column vectors, reads the k expert rows
// (and the shared row) with 16-byte loads, sums in fp32 and rounds once to the output type.
// In the fused layer the down GEMM writes the shared expert's rows straight into y; the
// combine then reads y[t] as the shared row, adds the kept slots to it in place, and leaves a
// token with no kept slot as the GEMM wrote it.
//
// Expert parallelism over peer memory ("Support visuel — Communication"): the remote variants
// read each kept slot's expert output where its owner wrote it -- row row0[e] + (r - offsets[e])
// of the owner's output buffer, e = ids[t, j], r the slot's row in the send layout -- so the
// return trip of the rows and the combine are one pass.
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

__device__ __forceinline__ void accum_bf16x8(float (&acc)[8], const uint4& v, float g) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(p[i]);
    acc[2 * i] = fmaf(g, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(g, f.y, acc[2 * i + 1]);
  }
}

// The first 16-byte vector of slot (t, j)'s expert output row, or null when the slot was
// dropped (r < 0) or, for the remote variant, its expert or row falls outside the tables
// (reported in rem.status; the slot then contributes nothing).
template <bool kRemote>
__device__ __forceinline__ const uint4* slot_src(const uint4* ye, const RemoteSrc& rem,
                                                 int64_t slot, int32_t r, int vecs) {
  if (r < 0) return nullptr;
  if constexpr (!kRemote) {
    return ye + (int64_t)r * vecs;
  } else {
    const int32_t e = rem.ids[slot];
    if (e >= 0 && e < rem.E) {
      const int64_t lo = rem.offsets[e], hi = rem.offsets[e + 1];
      const int64_t row = (int64_t)rem.row0[e] + (r - lo);
      if (r >= lo && r < hi && row >= 0 && row < rem.rows[e])
        return reinterpret_cast<const uint4*>(rem.base[e]) + row * vecs;
    }
    if (rem.status != nullptr) report_status(rem.status, kStatusInvalidInput);
    return nullptr;
  }
}

// Local rows come through the read-only path (they were written by an earlier kernel and
// this one does not write them); remote rows are read at L2, bypassing L1.
template <bool kRemote>
__device__ __forceinline__ uint4 load_row_vec(const uint4* p) {
  if constexpr (kRemote) return __ldcg(p);
  else return __ldg(p);
}

// KMAX >= k bounds the slots so that the k row loads of a vector are issued together
// before the sums (KMAX = 0: any k, one load after the other).  Either way the sum runs in
// slot order and then adds the shared row, so every KMAX gives the same bits.  The shared row
// is ye[shared_row0 + t] (shared_row0 >= 0), y[t] itself (shared_in_y), or absent.
template <int KMAX, bool kRemote>
__global__ void __launch_bounds__(128) combine_bf16_kernel(
    const uint4* __restrict__ ye, const int32_t* __restrict__ slot_row,
    const float* __restrict__ gates, int k, int vecs, int64_t shared_row0, int shared_in_y,
    RemoteSrc rem, uint4* __restrict__ y) {
  pdl_wait();
  __shared__ int32_t s_row[33];        // local: the slot's row of ye, -1 when dropped
  __shared__ const uint4* s_src[33];   // remote: the slot's row address, null when dropped
  __shared__ float s_g[33];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    const int64_t slot = t * k + threadIdx.x;
    const int32_t r = slot_row[slot];
    if constexpr (kRemote) {
      const uint4* p = slot_src<true>(ye, rem, slot, r, vecs);
      s_src[threadIdx.x] = p;
      s_row[threadIdx.x] = p != nullptr ? 0 : -1;
    } else {
      s_row[threadIdx.x] = r;
    }
    s_g[threadIdx.x] = gates[slot];
  }
  __syncthreads();
  if (shared_in_y) {
    bool any = false;
    for (int j = 0; j < k; ++j) any |= s_row[j] >= 0;
    if (!any) return;  // y[t] is the shared row already
  }
  auto row_vec = [&](int j, int v) {
    return load_row_vec<kRemote>(kRemote ? s_src[j] + v : ye + (int64_t)s_row[j] * vecs + v);
  };
  const uint4* shp = shared_in_y ? y + t * vecs
                                 : (shared_row0 >= 0 ? ye + (shared_row0 + t) * vecs : nullptr);
  for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if constexpr (KMAX > 0) {
      uint4 rows[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && s_row[j] >= 0) rows[j] = row_vec(j, v);
      uint4 sh = make_uint4(0u, 0u, 0u, 0u);
      if (shp != nullptr) sh = shp[v];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && s_row[j] >= 0) accum_bf16x8(acc, rows[j], s_g[j]);
      if (shp != nullptr) accum_bf16x8(acc, sh, 1.0f);
    } else {
      for (int j = 0; j < k; ++j)
        if (s_row[j] >= 0) accum_bf16x8(acc, row_vec(j, v), s_g[j]);
      if (shp != nullptr) accum_bf16x8(acc, shp[v], 1.0f);
    }
    uint4 o;
    __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) po[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    y[t * vecs + v] = o;
  }
}

// The same sums with one warp per token and kCombineWarps tokens per block: a token's
// slots and gates sit in lanes 0..k-1 and are broadcast with shuffles, a token with no kept
// slot costs one ballot.  Used where tokens are many and rows small (8x fewer blocks than
// the block-per-token kernel); the summation order is the same, so the bits are.
constexpr int kCombineWarps = 8;

template <int KMAX, bool kRemote>
__global__ void __launch_bounds__(32 * kCombineWarps) combine_bf16_warp_kernel(
    const uint4* __restrict__ ye, const int32_t* __restrict__ slot_row,
    const float* __restrict__ gates, int64_t N, int k, int vecs, int64_t shared_row0,
    int shared_in_y, RemoteSrc rem, uint4* __restrict__ y) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  if (t >= N) return;  // warp-uniform
  // lane j < k holds slot j: its row index (local) or its row's address (remote; the 64-bit
  // broadcast is kept out of the local variant, where the extra registers cost occupancy)
  int32_t my_row = -1;
  const uint4* my_src = nullptr;
  float my_g = 0.f;
  if (lane < k) {
    const int64_t slot = t * k + lane;
    my_row = slot_row[slot];
    if constexpr (kRemote) my_src = slot_src<true>(ye, rem, slot, my_row, vecs);
    my_g = gates[slot];
  }
  const unsigned kept = __ballot_sync(0xffffffffu, kRemote ? my_src != nullptr : my_row >= 0);
  if (shared_in_y && kept == 0u) return;  // y[t] is the shared row already
  int32_t rj[KMAX];
  const uint4* pj[KMAX];
  float gj[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if constexpr (kRemote) {
      pj[j] = reinterpret_cast<const uint4*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_src), j));
      rj[j] = pj[j] != nullptr ? 0 : -1;
    } else {
      rj[j] = __shfl_sync(0xffffffffu, my_row, j);
      pj[j] = nullptr;
    }
    gj[j] = __shfl_sync(0xffffffffu, my_g, j);
  }
  const uint4* shp = shared_in_y ? y + t * vecs
                                 : (shared_row0 >= 0 ? ye + (shared_row0 + t) * vecs : nullptr);
  for (int v = lane; v < vecs; v += 32) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint4 rows[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k && rj[j] >= 0)
        rows[j] = load_row_vec<kRemote>(kRemote ? pj[j] + v : ye + (int64_t)rj[j] * vecs + v);
    uint4 sh = make_uint4(0u, 0u, 0u, 0u);
    if (shp != nullptr) sh = shp[v];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k && rj[j] >= 0) accum_bf16x8(acc, rows[j], gj[j]);
    if (shp != nullptr) accum_bf16x8(acc, sh, 1.0f);
    uint4 o;
    __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) po[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    y[t * vecs + v] = o;
  }
}

__global__ void __launch_bounds__(128) combine_f32_kernel(
    const float4* __restrict__ ye, const int32_t* __restrict__ slot_row,
    const float* __restrict__ gates, int k, int vecs, int64_t shared_row0,
    float4* __restrict__ y) {
  pdl_wait();
  __shared__ int32_t s_row[33];
  __shared__ float s_g[33];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    s_row[threadIdx.x] = slot_row[t * k + threadIdx.x];
    s_g[threadIdx.x] = gates[t * k + threadIdx.x];
  }
  __syncthreads();
  for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int32_t r = s_row[j];
      if (r >= 0) {
        const float4 a = ye[(int64_t)r * vecs + v];
        const float g = s_g[j];
        acc.x = fmaf(g, a.x, acc.x);
        acc.y = fmaf(g, a.y, acc.y);
        acc.z = fmaf(g, a.z, acc.z);
        acc.w = fmaf(g, a.w, acc.w);
      }
    }
    if (shared_row0 >= 0) {
      const float4 a = ye[(shared_row0 + t) * vecs + v];
      acc.x += a.x;
      acc.y += a.y;
      acc.z += a.z;
      acc.w += a.w;
    }
    y[t * vecs + v] = acc;
  }
}

// MOE_B200_COMBINE_WARP=0 keeps the block-per-token kernel everywhere (A/B measurements).
bool combine_warp_enabled() {
  const char* v = std::getenv("MOE_B200_COMBINE_WARP");
  return !(v != nullptr && v[0] == '0');
}

}  // namespace

namespace {

template <bool kRemote>
void launch_combine_bf16(const uint4* src, const int32_t* slot_row, const float* gates,
                         int64_t N, int k, int d, int64_t shared_row0, int shared_in_y,
                         const RemoteSrc& rem, uint4* dst, cudaStream_t stream) {
  // warp per token when the warps fill every SM several times over and a token reads at
  // most 8 KB of expert rows; else block per token.  Measured: the capacity and Switch
  // layers (8 and 4 KB per token) 19.7 -> 16.4 and 16.6 -> 14.2 us; the Mixtral-shaped
  // prefill (16 KB per token) 72.5 -> 77.4 us, so it keeps a block per token.
  const int row_bytes = d * 2;
  const int vecs = d / 8;
  if (k <= 8 && N >= (int64_t)tc::num_sms() * 64 && (int64_t)k * row_bytes <= 8192 &&
      combine_warp_enabled()) {
    const unsigned wblocks = (unsigned)((N + kCombineWarps - 1) / kCombineWarps);
    const unsigned th = 32 * kCombineWarps;
    if (k <= 2)
      launch_pdl(combine_bf16_warp_kernel<2, kRemote>, wblocks, th, 0, stream, src, slot_row, gates, N, k, vecs, shared_row0, shared_in_y, rem, dst);
    else if (k <= 4)
      launch_pdl(combine_bf16_warp_kernel<4, kRemote>, wblocks, th, 0, stream, src, slot_row, gates, N, k, vecs, shared_row0, shared_in_y, rem, dst);
    else
      launch_pdl(combine_bf16_warp_kernel<8, kRemote>, wblocks, th, 0, stream, src, slot_row, gates, N, k, vecs, shared_row0, shared_in_y, rem, dst);
    return;
  }
  const unsigned blocks = (unsigned)N;
  if (k <= 2)
    launch_pdl(combine_bf16_kernel<2, kRemote>, blocks, 128, 0, stream, src, slot_row, gates, k, vecs, shared_row0, shared_in_y, rem, dst);
  else if (k <= 4)
    launch_pdl(combine_bf16_kernel<4, kRemote>, blocks, 128, 0, stream, src, slot_row, gates, k, vecs, shared_row0, shared_in_y, rem, dst);
  else if (k <= 8)
    launch_pdl(combine_bf16_kernel<8, kRemote>, blocks, 128, 0, stream, src, slot_row, gates, k, vecs, shared_row0, shared_in_y, rem, dst);
  else
    launch_pdl(combine_bf16_kernel<0, kRemote>, blocks, 128, 0, stream, src, slot_row, gates, k, vecs, shared_row0, shared_in_y, rem, dst);
}

}  // namespace

cudaError_t launch_combine(const void* ye, const int32_t* slot_row, const float* gates,
                           int64_t N, int k, int d, int64_t shared_row0, int shared_in_y,
                           int is_f32, void* y, cudaStream_t stream, int* launches,
                           const RemoteSrc* rem) {
  if (N == 0) return cudaSuccess;
  ++*launches;
  if (is_f32) {
    launch_pdl(combine_f32_kernel, (unsigned)N, 128, 0, stream, (const float4*)ye, slot_row, gates, k,
                                                        d / 4, shared_row0, (float4*)y);
  } else if (rem != nullptr) {
    launch_combine_bf16<true>((const uint4*)ye, slot_row, gates, N, k, d, shared_row0,
                              shared_in_y, *rem, (uint4*)y, stream);
  } else {
    launch_combine_bf16<false>((const uint4*)ye, slot_row, gates, N, k, d, shared_row0,
                               shared_in_y, RemoteSrc{}, (uint4*)y, stream);
  }
  return cudaGetLastError();
}

}  // namespace moe
