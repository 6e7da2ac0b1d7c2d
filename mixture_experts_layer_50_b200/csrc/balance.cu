// Load-balancing statistics of a routed batch, and the aux-loss-free bias update.
//
// "Основы MoE", "Вспомогательный лосс Switch Transformer": f_i is the share of the top-k
// assignments that went to expert i, P_i the router probability of expert i averaged over the
// tokens, and the balance statistic is E * sum_i f_i P_i (1 when balanced, about E when every
// token goes to one expert).  "Le groupe d'experts (MoE)" (load-balance section) and the
// DeepSeek-V4.1-Flash page ("L'équilibrage de charge", "l'équilibrage par modalité"): after a
// step each expert's selection bias moves by -gamma if its load is above the mean and +gamma
// if below, with one bias set and one load count per modality.
//
// Deterministic: pass 1 gives every tile of kTile tokens its per-expert probability sums
// (tokens added in order) and its per-(set, expert) assignment counts; pass 2 adds the tiles
// in order, one thread per expert, and applies the bias step.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kTile = 64;
constexpr int kMaxSets = 8;

__global__ void __launch_bounds__(256) balance_tile_kernel(
    const float* __restrict__ logits, const int32_t* __restrict__ ids,
    const uint8_t* __restrict__ modality, int64_t N, int E, int k, int score_fn, int n_sets,
    float* __restrict__ part_p, int32_t* __restrict__ part_load) {
  pdl_wait();
  extern __shared__ float sm[];
  float* s_m = sm;                                   // [kTile] per-token max (softmax)
  float* s_inv = sm + kTile;                         // [kTile] 1 / normaliser
  int32_t* s_load = reinterpret_cast<int32_t*>(sm + 2 * kTile);  // [n_sets][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)blockIdx.x * kTile;
  const int ntok = (int)min((int64_t)kTile, N - t0);
  for (int i = threadIdx.x; i < n_sets * E; i += blockDim.x) s_load[i] = 0;
  // per-token normaliser: softmax max and sum, or the sum of sigmoid affinities
  for (int t = warp; t < ntok; t += blockDim.x / 32) {
    const float* z = logits + (t0 + t) * E;
    float m = -INFINITY;
    if (score_fn == 0)
      for (int e = lane; e < E; e += 32) m = fmaxf(m, z[e]);
    m = warp_max(m);
    float s = 0.f;
    for (int e = lane; e < E; e += 32)
      s += score_fn == 0 ? expf(z[e] - m) : 1.0f / (1.0f + expf(-z[e]));
    s = warp_sum(s);
    if (lane == 0) {
      s_m[t] = m;
      s_inv[t] = 1.0f / s;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ntok * k; i += blockDim.x) {
    const int e = ids[t0 * k + i];
    int set = modality != nullptr ? (int)modality[t0 + i / k] : 0;
    if (set >= n_sets) set = 0;  // the routing uses set 0 for an unknown flag too
    if (e >= 0 && e < E) atomicAdd(&s_load[set * E + e], 1);
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float acc = 0.f;
    for (int t = 0; t < ntok; ++t) {
      const float zz = logits[(t0 + t) * E + e];
      const float p = score_fn == 0 ? expf(zz - s_m[t]) : 1.0f / (1.0f + expf(-zz));
      acc += p * s_inv[t];
    }
    part_p[(int64_t)blockIdx.x * E + e] = acc;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_sets * E; i += blockDim.x)
    part_load[(int64_t)blockIdx.x * n_sets * E + i] = s_load[i];
}

__global__ void __launch_bounds__(1024) balance_final_kernel(
    const float* __restrict__ part_p, const int32_t* __restrict__ part_load, int n_tiles,
    int64_t N, int E, int k, int n_sets, float* __restrict__ f, float* __restrict__ P,
    float* __restrict__ aux, int32_t* __restrict__ set_load, float* __restrict__ bias,
    float gamma) {
  pdl_wait();
  __shared__ float s_fp[1024];
  __shared__ int64_t s_red[1024];
  __shared__ int64_t s_tot[kMaxSets];
  const int e = threadIdx.x;
  float fp = 0.f;
  int64_t my_load[kMaxSets];
  for (int m = 0; m < kMaxSets; ++m) my_load[m] = 0;
  if (e < E) {
    float p = 0.f;
    for (int i = 0; i < n_tiles; ++i) p += part_p[(int64_t)i * E + e];
    p = N > 0 ? p / (float)N : 0.f;
    int64_t all = 0;
    for (int m = 0; m < n_sets; ++m) {
      int64_t c = 0;
      for (int i = 0; i < n_tiles; ++i) c += part_load[((int64_t)i * n_sets + m) * E + e];
      my_load[m] = c;
      all += c;
      if (set_load != nullptr) set_load[m * E + e] = (int32_t)c;
    }
    const float fe = N > 0 ? (float)((double)all / (double)(N * k)) : 0.f;
    if (f != nullptr) f[e] = fe;
    if (P != nullptr) P[e] = p;
    fp = fe * p;
  }
  s_fp[e] = fp;
  // per-set totals (integers: any order is exact)
  for (int m = 0; m < n_sets; ++m) {
    __syncthreads();
    s_red[e] = my_load[m];
    for (int w = 512; w > 0; w >>= 1) {
      __syncthreads();
      if (e < w) s_red[e] += s_red[e + w];
    }
    __syncthreads();
    if (e == 0) s_tot[m] = s_red[0];
  }
  // fixed-shape tree over the 1024 slots for the statistic
  for (int w = 512; w > 0; w >>= 1) {
    __syncthreads();
    if (e < w) s_fp[e] += s_fp[e + w];
  }
  __syncthreads();
  if (e == 0 && aux != nullptr) aux[0] = (float)E * s_fp[0];
  if (bias != nullptr && e < E) {
    for (int m = 0; m < n_sets; ++m) {
      const int64_t diff = s_tot[m] - my_load[m] * E;   // > 0: below the mean load
      const float step = diff > 0 ? gamma : (diff < 0 ? -gamma : 0.f);
      bias[m * E + e] = __fadd_rn(bias[m * E + e], step);
    }
  }
}

}  // namespace

size_t balance_scratch_bytes(int64_t N, int E, int n_sets) {
  const int64_t tiles = (N + kTile - 1) / kTile;
  return (size_t)tiles * E * sizeof(float) + (size_t)tiles * n_sets * E * sizeof(int32_t);
}

cudaError_t launch_balance(const float* logits, const int32_t* ids, const uint8_t* modality,
                           int64_t N, int E, int k, int score_fn, int n_sets, void* scratch,
                           float* f, float* P, float* aux, int32_t* set_load, float* bias,
                           float gamma, cudaStream_t stream, int* launches) {
  const int tiles = (int)((N + kTile - 1) / kTile);
  float* part_p = reinterpret_cast<float*>(scratch);
  int32_t* part_load = reinterpret_cast<int32_t*>(part_p + (size_t)tiles * E);
  if (tiles > 0) {
    const size_t smem = sizeof(float) * 2 * kTile + sizeof(int32_t) * (size_t)n_sets * E;
    launch_pdl(balance_tile_kernel, tiles, 256, smem, stream, logits, ids, modality, N, E, k, score_fn,
                                                      n_sets, part_p, part_load);
    ++*launches;
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  launch_pdl(balance_final_kernel, 1, 1024, 0, stream, part_p, part_load, tiles, N, E, k, n_sets, f, P,
                                               aux, set_load, bias, gamma);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace moe
