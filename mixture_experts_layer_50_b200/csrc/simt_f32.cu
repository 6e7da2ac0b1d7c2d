// float32 path of the layer: the router projection and the two-layer experts in plain
// fp32 FMAs.  It serves the fp32 toy layer of the dataistudio "Mixture of Experts" page
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

// h[r][f] = act(src_r . W1_e[f]); SwiGLU: silu(clamp(gate)) * clamp(up).
__global__ void __launch_bounds__(256) ffn_up_f32_kernel(
    const float* __restrict__ xp, const float* __restrict__ x, const int32_t* __restrict__ offsets,
    int64_t N, int64_t Nk, int d, int E, int F, int n_shared, int act, float clamp,
    const float* __restrict__ W_gu, float* __restrict__ h) {
  const int f = blockIdx.y * 32 + threadIdx.x;
  const int64_t r = (int64_t)blockIdx.x * 8 + threadIdx.y;
  if (f >= F) return;
  const float* src = nullptr;
  const int e = resolve_row(offsets, E, Nk, N, n_shared, r, xp, x, d, &src);
  if (e < 0) return;
  const int64_t rows = (act == 0) ? 2 * (int64_t)F : F;
  const float* wg = W_gu + ((int64_t)e * rows + f) * d;
  float g = 0.f;
  for (int i = 0; i < d; ++i) g = fmaf(src[i], wg[i], g);
  float out;
  if (act == 0) {
    const float* wu = wg + (int64_t)F * d;
    float u = 0.f;
    for (int i = 0; i < d; ++i) u = fmaf(src[i], wu[i], u);
    if (clamp > 0.f) {
      g = fminf(fmaxf(g, -clamp), clamp);
      u = fminf(fmaxf(u, -clamp), clamp);
    }
    out = g / (1.0f + expf(-g)) * u;
  } else {
    out = fmaxf(g, 0.f);
  }
  h[r * F + f] = out;
}

// ye[r][c] = h[r] . W2_e[c].
__global__ void __launch_bounds__(256) ffn_down_f32_kernel(
    const float* __restrict__ h, const float* __restrict__ xp, const float* __restrict__ x,
    const int32_t* __restrict__ offsets, int64_t N, int64_t Nk, int d, int E, int F,
    int n_shared, const float* __restrict__ W_down, float* __restrict__ ye) {
  const int c = blockIdx.y * 32 + threadIdx.x;
  const int64_t r = (int64_t)blockIdx.x * 8 + threadIdx.y;
  if (c >= d) return;
  const float* src = nullptr;
  const int e = resolve_row(offsets, E, Nk, N, n_shared, r, xp, x, d, &src);
  if (e < 0) return;
  const float* hr = h + r * F;
  const float* w = W_down + ((int64_t)e * d + c) * F;
  float acc = 0.f;
  for (int f = 0; f < F; ++f) acc = fmaf(hr[f], w[f], acc);
  ye[r * d + c] = acc;
}

}  // namespace

cudaError_t launch_router_f32(const float* x, const float* W_g, const float* logit_offset,
                              int64_t N, int d, int E, float* logits, cudaStream_t stream,
                              int* launches) {
  if (N == 0) return cudaSuccess;
  ++*launches;
  const int64_t total = N * E;
  router_f32_kernel<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(x, W_g, logit_offset,
                                                                         N, d, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_ffn_f32(const float* xp, const float* x, const int32_t* offsets,
                           int64_t N, int64_t Nk, int d, int E, int F, int n_shared, int act,
                           float clamp, const float* W_gu, const float* W_down, float* h,
                           float* ye, cudaStream_t stream, int* launches) {
  if (N == 0) return cudaSuccess;
  const int64_t rows = Nk + (n_shared ? N : 0);
  dim3 block(32, 8);
  dim3 g1((unsigned)((rows + 7) / 8), (F + 31) / 32);
  ffn_up_f32_kernel<<<g1, block, 0, stream>>>(xp, x, offsets, N, Nk, d, E, F, n_shared, act,
                                              clamp, W_gu, h);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dim3 g2((unsigned)((rows + 7) / 8), (d + 31) / 32);
  ffn_down_f32_kernel<<<g2, block, 0, stream>>>(h, xp, x, offsets, N, Nk, d, E, F, n_shared,
                                                W_down, ye);
  *launches += 2;
  return cudaGetLastError();
}

}  // namespace moe
