// float32 path of the layer: the router projection and the two-layer experts in plain
// fp32 FMAs (d and F at most 4096).  It serves the fp32 toy layer of the dataistudio "Mixture of Experts" page
// (1000 tokens, d = 64, eight 64 -> 256 -> 64 ReLU experts, top-2); tf32 tensor cores
// would not meet a 1e-4 absolute bound there, and the work is a few hundred MFLOP.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// logits[t][e] = sum_i x[t][i] W_g[e][i] (+ offset[e]); one thread per (token, expert).
__global__ void __launch_bounds__(256) router_f32_kernel(const float* __restrict__ x,
                                                         const float* __restrict__ W_g,
                                                         const float* __restrict__ off,
                                                         int64_t N, int d, int E,
                                                         float* __restrict__ logits) {
  pdl_wait();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * E) return;
  const int64_t t = idx / E;
  const int e = (int)(idx % E);
  const float* xr = x + t * d;
  const float* wr = W_g + (int64_t)e * d;
  float acc = 0.f;
  for (int i = 0; i < d; ++i) acc = fmaf(xr[i], wr[i], acc);
  if (off != nullptr) acc += off[e];
  logits[idx] = acc;
}

// Largest e with offsets[e] <= r (r < offsets[E]): the expert owning row r.
__device__ __forceinline__ int owner_group(const int32_t* offsets, int E, int64_t r) {
  int lo = 0, hi = E;  // offsets[lo] <= r < offsets[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

// Resolve row r of the (routed + shared) layout: expert index and source row, or -1.
__device__ __forceinline__ int resolve_row(const int32_t* offsets, int E, int64_t Nk,
                                           int64_t N, int n_shared, int64_t r,
                                           const float* xp, const float* x, int d,
                                           const float** src) {
  if (r < Nk) {
    if (r >= offsets[E]) return -1;
    *src = xp + r * d;
    return owner_group(offsets, E, r);
  }
  if (n_shared && r < Nk + N) {
    *src = x + (r - Nk) * d;
    return E;
  }
  return -1;
}

// One warp per (row, 32 consecutive outputs): the row stays in registers (NV floats per
// lane, element i on lane i % 32), the lanes split each dot product over the input dimension
// (coalesced weight rows) and a shuffle tree sums it; lane j keeps output j of the group.
template <int NV>
__device__ __forceinline__ float dot_warp(const float* __restrict__ w, const float (&xr)[NV],
                                          int K, int lane) {
  float acc = 0.f;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int i = v * 32 + lane;
    if (i < K) acc = fmaf(xr[v], w[i], acc);
  }
  return warp_sum(acc);
}

// h[r][f] = act(src_r . W1_e[f]); SwiGLU: silu(clamp(gate)) * clamp(up).  K = d.
template <int NV>
__global__ void __launch_bounds__(256) ffn_up_f32_kernel(
    const float* __restrict__ xp, const float* __restrict__ x, const int32_t* __restrict__ offsets,
    int64_t N, int64_t Nk, int d, int E, int F, int n_shared, int act, float clamp,
    const float* __restrict__ W_gu, float* __restrict__ h) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int f0 = blockIdx.y * 32;
  const float* src = nullptr;
  const int e = resolve_row(offsets, E, Nk, N, n_shared, r, xp, x, d, &src);
  if (e < 0) return;
  float xr[NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int i = v * 32 + lane;
    xr[v] = i < d ? src[i] : 0.f;
  }
  const int64_t rows = (act == 0) ? 2 * (int64_t)F : F;
  const float* wbase = W_gu + (int64_t)e * rows * d;
  float mine = 0.f;
  for (int j = 0; j < 32 && f0 + j < F; ++j) {
    const int f = f0 + j;
    float g = dot_warp<NV>(wbase + (int64_t)f * d, xr, d, lane);
    float out;
    if (act == 0) {
      float u = dot_warp<NV>(wbase + (int64_t)(F + f) * d, xr, d, lane);
      if (clamp > 0.f) {
        g = fminf(fmaxf(g, -clamp), clamp);
        u = fminf(fmaxf(u, -clamp), clamp);
      }
      out = g / (1.0f + expf(-g)) * u;
    } else {
      out = fmaxf(g, 0.f);
    }
    if (lane == j) mine = out;
  }
  if (f0 + lane < F) h[r * F + f0 + lane] = mine;
}

// ye[r][c] = h[r] . W2_e[c].  K = F.
template <int NV>
__global__ void __launch_bounds__(256) ffn_down_f32_kernel(
    const float* __restrict__ h, const float* __restrict__ xp, const float* __restrict__ x,
    const int32_t* __restrict__ offsets, int64_t N, int64_t Nk, int d, int E, int F,
    int n_shared, const float* __restrict__ W_down, float* __restrict__ ye) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int c0 = blockIdx.y * 32;
  const float* src = nullptr;
  const int e = resolve_row(offsets, E, Nk, N, n_shared, r, xp, x, d, &src);
  if (e < 0) return;
  float hr[NV];
  const float* hrow = h + r * F;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int i = v * 32 + lane;
    hr[v] = i < F ? hrow[i] : 0.f;
  }
  const float* wbase = W_down + (int64_t)e * d * F;
  float mine = 0.f;
  for (int j = 0; j < 32 && c0 + j < d; ++j) {
    const float acc = dot_warp<NV>(wbase + (int64_t)(c0 + j) * F, hr, F, lane);
    if (lane == j) mine = acc;
  }
  if (c0 + lane < d) ye[r * d + c0 + lane] = mine;
}

template <int NV>
void launch_up(dim3 g, cudaStream_t st, const float* xp, const float* x, const int32_t* offsets,
               int64_t N, int64_t Nk, int d, int E, int F, int n_shared, int act, float clamp,
               const float* W_gu, float* h) {
  launch_pdl(ffn_up_f32_kernel<NV>, g, 256, 0, st, xp, x, offsets, N, Nk, d, E, F, n_shared, act, clamp,
                                           W_gu, h);
}
template <int NV>
void launch_down(dim3 g, cudaStream_t st, const float* h, const float* xp, const float* x,
                 const int32_t* offsets, int64_t N, int64_t Nk, int d, int E, int F,
                 int n_shared, const float* W_down, float* ye) {
  launch_pdl(ffn_down_f32_kernel<NV>, g, 256, 0, st, h, xp, x, offsets, N, Nk, d, E, F, n_shared,
                                             W_down, ye);
}

// Smallest register width (floats per lane) that holds K inputs.
int lanes_width(int K) {
  int nv = 1;
  while (nv * 32 < K) nv *= 2;
  return nv;
}

}  // namespace

cudaError_t launch_router_f32(const float* x, const float* W_g, const float* logit_offset,
                              int64_t N, int d, int E, float* logits, cudaStream_t stream,
                              int* launches) {
  if (N == 0) return cudaSuccess;
  ++*launches;
  const int64_t total = N * E;
  launch_pdl(router_f32_kernel, (unsigned)((total + 255) / 256), 256, 0, stream, x, W_g, logit_offset,
                                                                         N, d, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_ffn_f32(const float* xp, const float* x, const int32_t* offsets,
                           int64_t N, int64_t Nk, int d, int E, int F, int n_shared, int act,
                           float clamp, const float* W_gu, const float* W_down, float* h,
                           float* ye, cudaStream_t stream, int* launches) {
  if (N == 0) return cudaSuccess;
  const int64_t rows = Nk + (n_shared ? N : 0);
  dim3 g1((unsigned)((rows + 7) / 8), (F + 31) / 32);
  switch (lanes_width(d)) {
#define MOE_UP(NV) case NV: launch_up<NV>(g1, stream, xp, x, offsets, N, Nk, d, E, F, n_shared, act, clamp, W_gu, h); break;
    MOE_UP(1) MOE_UP(2) MOE_UP(4) MOE_UP(8) MOE_UP(16) MOE_UP(32) MOE_UP(64) MOE_UP(128)
#undef MOE_UP
    default: return cudaErrorInvalidValue;
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dim3 g2((unsigned)((rows + 7) / 8), (d + 31) / 32);
  switch (lanes_width(F)) {
#define MOE_DOWN(NV) case NV: launch_down<NV>(g2, stream, h, xp, x, offsets, N, Nk, d, E, F, n_shared, W_down, ye); break;
    MOE_DOWN(1) MOE_DOWN(2) MOE_DOWN(4) MOE_DOWN(8) MOE_DOWN(16) MOE_DOWN(32) MOE_DOWN(64) MOE_DOWN(128)
#undef MOE_DOWN
    default: return cudaErrorInvalidValue;
  }
  *launches += 2;
  return cudaGetLastError();
}

}  // namespace moe
