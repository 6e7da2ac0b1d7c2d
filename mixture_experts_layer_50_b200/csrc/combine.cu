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

// KMAX >= k bounds the slots so that the k row loads of a vector are issued together
// before the sums (KMAX = 0: any k, one load after the other).  Either way the sum runs in
// slot order and then adds the shared row, so every KMAX gives the same bits.  The shared row
// is ye[shared_row0 + t] (shared_row0 >= 0), y[t] itself (shared_in_y), or absent.
template <int KMAX>
__global__ void __launch_bounds__(128) combine_bf16_kernel(
    const uint4* __restrict__ ye, const int32_t* __restrict__ slot_row,
    const float* __restrict__ gates, int k, int vecs, int64_t shared_row0, int shared_in_y,
    uint4* __restrict__ y) {
  pdl_wait();
  __shared__ int32_t s_row[33];
  __shared__ float s_g[33];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    s_row[threadIdx.x] = slot_row[t * k + threadIdx.x];
    s_g[threadIdx.x] = gates[t * k + threadIdx.x];
  }
  __syncthreads();
  if (shared_in_y) {
    bool any = false;
    for (int j = 0; j < k; ++j) any |= s_row[j] >= 0;
    if (!any) return;  // y[t] is the shared row already
  }
  const uint4* shp = shared_in_y ? y + t * vecs
                                 : (shared_row0 >= 0 ? ye + (shared_row0 + t) * vecs : nullptr);
  for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if constexpr (KMAX > 0) {
      uint4 rows[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && s_row[j] >= 0) rows[j] = ye[(int64_t)s_row[j] * vecs + v];
      uint4 sh = make_uint4(0u, 0u, 0u, 0u);
      if (shp != nullptr) sh = shp[v];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && s_row[j] >= 0) accum_bf16x8(acc, rows[j], s_g[j]);
      if (shp != nullptr) accum_bf16x8(acc, sh, 1.0f);
    } else {
      for (int j = 0; j < k; ++j) {
        const int32_t r = s_row[j];
        if (r >= 0) accum_bf16x8(acc, ye[(int64_t)r * vecs + v], s_g[j]);
      }
      if (shp != nullptr) accum_bf16x8(acc, shp[v], 1.0f);
    }
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

}  // namespace

cudaError_t launch_combine(const void* ye, const int32_t* slot_row, const float* gates,
                           int64_t N, int k, int d, int64_t shared_row0, int shared_in_y,
                           int is_f32, void* y, cudaStream_t stream, int* launches) {
  if (N == 0) return cudaSuccess;
  ++*launches;
  if (is_f32) {
    launch_pdl(combine_f32_kernel, (unsigned)N, 128, 0, stream, (const float4*)ye, slot_row, gates, k,
                                                        d / 4, shared_row0, (float4*)y);
  } else {
    const uint4* src = (const uint4*)ye;
    uint4* dst = (uint4*)y;
    const unsigned blocks = (unsigned)N;
    if (k <= 2)
      launch_pdl(combine_bf16_kernel<2>, blocks, 128, 0, stream, src, slot_row, gates, k, d / 8, shared_row0, shared_in_y, dst);
    else if (k <= 4)
      launch_pdl(combine_bf16_kernel<4>, blocks, 128, 0, stream, src, slot_row, gates, k, d / 8, shared_row0, shared_in_y, dst);
    else if (k <= 8)
      launch_pdl(combine_bf16_kernel<8>, blocks, 128, 0, stream, src, slot_row, gates, k, d / 8, shared_row0, shared_in_y, dst);
    else
      launch_pdl(combine_bf16_kernel<0>, blocks, 128, 0, stream, src, slot_row, gates, k, d / 8, shared_row0, shared_in_y, dst);
  }
  return cudaGetLastError();
}

}  // namespace moe
