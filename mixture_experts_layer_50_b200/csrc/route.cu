// Router scores, top-k selection and gates: one warp per token.
//
// "Основы MoE" (ai.flicky.cc), section "Как устроен MoE-слой", steps 2-3: p = softmax(z),
// keep the k largest, g_i = p_i / sum_{j in T} p_j; with k = 1 (Switch) the weight is p_i.
// DeepSeek-V3 scores with a sigmoid.  "Le groupe d'experts (MoE)", "Étape 1: le routeur"
// and the DeepSeek-V4.1-Flash "Mixture-of-Experts" page ("L'équilibrage de charge",
// "l'équilibrage par modalité"): a per-expert bias, one set per modality, is added for
// the selection only; the gates use the unbiased scores.
//
// Selection keys are float32: z + b (softmax) or sigma(z) + b (sigmoid).  The k rounds
// of a warp arg-max pick the largest key, ties to the lower expert index, so ids come out
// by descending key.  sigma(z) is evaluated with the exp below, built from Cody & Waite's
// range reduction and a Taylor polynomial out of correctly rounded float32 operations
// (explicit _rn intrinsics, never contracted into FMAs), so that sigmoid keys -- and the
// experts they select -- are reproducible bit for bit on any IEEE float32 machine.
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// e^x for |x| <= 80.  x = n ln2 + r with n = rint(x / ln2); ln2 is split into a 16-bit
// high part (so n * ln2_hi is exact for |n| < 256) and its float remainder; e^r comes
// from the degree-7 Taylor polynomial in Horner form; 2^n is applied exactly.
__device__ __forceinline__ float exp_reduced_taylor(float x) {
  const float inv_ln2 = 1.4426950408889634f;
  const float ln2_hi = 45426.0f / 65536.0f;
  const float ln2_lo = (float)(0.6931471805599453 - 0.693145751953125);
  const float n = rintf(__fmul_rn(x, inv_ln2));
  float r = __fsub_rn(x, __fmul_rn(n, ln2_hi));
  r = __fsub_rn(r, __fmul_rn(n, ln2_lo));
  float p = 1.0f / 5040.0f;
  p = __fadd_rn(__fmul_rn(p, r), 1.0f / 720.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f / 120.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f / 24.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f / 6.0f);
  p = __fadd_rn(__fmul_rn(p, r), 0.5f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  p = __fadd_rn(__fmul_rn(p, r), 1.0f);
  const int ni = (int)n;  // |ni| <= 116 for |x| <= 80: 2^ni is a normal float
  return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

__device__ __forceinline__ float sigmoid_reproducible(float z) {
  const float zc = fminf(fmaxf(z, -80.0f), 80.0f);
  // the correctly rounded reciprocal: the same bits as the correctly rounded 1 / y
  return __frcp_rn(__fadd_rn(1.0f, exp_reduced_taylor(-zc)));
}

// (key, expert) order used by the selection: larger key first, then lower index.
__device__ __forceinline__ bool beats(float ka, int ea, float kb, int eb) {
  return ka > kb || (ka == kb && ea < eb);
}

// The selection of one token by one warp: scores, keys, `rounds` rounds of arg-max and the
// gates.  Lane r returns the r-th selection (e = -1 past `rounds`), its score and, for r < k,
// its gate.  Every lane of the warp must call it.
struct TokenSel {
  int e;
  float sc;
  float g;
};

template <int J>  // keys per lane: E <= 32 * J
__device__ __forceinline__ TokenSel select_token(
    const float* __restrict__ logits, int n_parts, int64_t part_stride,
    const float* __restrict__ offset, float* __restrict__ logits_out, int64_t t, int E, int k,
    int score_fn, int renorm, const float* __restrict__ bias, int n_bias_sets,
    const uint8_t* __restrict__ modality, int* status, int rounds) {
  const int lane = threadIdx.x & 31;
  const float* z = logits + t * E;
  const float* b = nullptr;
  if (bias != nullptr) {
    int set = 0;
    if (modality != nullptr) {
      set = modality[t];
      if (set >= n_bias_sets) {
        if (lane == 0) report_status(status, kStatusInvalidInput);
        set = 0;
      }
    }
    b = bias + (int64_t)set * E;
  }

  float key[J], sc[J], zv[J];
  float zmax = -INFINITY;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    key[j] = -INFINITY;
    sc[j] = 0.0f;
    zv[j] = 0.0f;
    if (e < E) {
      float zz = z[e];
      if (n_parts > 1 || offset != nullptr) {
        // split-K partial logits, added in slice order, then the per-expert offset
        for (int s = 1; s < n_parts; ++s) zz += z[s * part_stride + e];
        if (offset != nullptr) zz += offset[e];
        if (logits_out != nullptr) logits_out[t * E + e] = zz;
      }
      zv[j] = zz;
      zmax = fmaxf(zmax, zz);
      const float s = (score_fn == 1) ? sigmoid_reproducible(zz) : zz;
      sc[j] = s;
      key[j] = (b != nullptr) ? __fadd_rn(s, b[e]) : s;
    }
  }

  // `rounds` rounds of warp arg-max (k, or more when the next-best candidates are asked for;
  // at most E).  Lane r keeps the r-th selection.
  uint32_t taken = 0;
  int my_e = -1;
  float my_sc = 0.0f;
  for (int r = 0; r < rounds; ++r) {
    float bk = -INFINITY, bs = 0.0f;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u) && (be == 0x7fffffff || key[j] > bk)) {
        bk = key[j];
        be = e;
        bs = sc[j];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      if (oe != 0x7fffffff && (be == 0x7fffffff || beats(ok, oe, bk, be))) {
        bk = ok;
        be = oe;
        bs = os;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == r) {
      my_e = be;
      my_sc = bs;
    }
  }

  const bool mine = lane < k;
  float g;
  if (score_fn == 0) {
    if (renorm) {
      // softmax over the selected logits
      const float m = warp_max(mine ? my_sc : -INFINITY);
      const float ex = mine ? expf(my_sc - m) : 0.0f;
      g = ex / warp_sum(ex);
    } else {
      // raw probability of the full softmax
      const float M = warp_max(zmax);
      float part = 0.0f;
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int e = lane + 32 * j;
        if (e < E) part += expf(zv[j] - M);
      }
      g = expf(my_sc - M) / warp_sum(part);
    }
  } else {
    if (renorm) {
      g = my_sc / warp_sum(mine ? my_sc : 0.0f);
    } else {
      g = my_sc;
    }
  }
  return TokenSel{my_e, my_sc, g};
}

template <int J>
__global__ void __launch_bounds__(256) route_topk_kernel(
    const float* __restrict__ logits, int n_parts, int64_t part_stride,
    const float* __restrict__ offset, float* __restrict__ logits_out, int64_t N, int E, int k,
    int score_fn, int renorm, const float* __restrict__ bias, int n_bias_sets,
    const uint8_t* __restrict__ modality, int32_t* __restrict__ ids, float* __restrict__ gates,
    int* status, int k_extra, int32_t* __restrict__ cand, float* __restrict__ cand_val) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= N) return;
  const int rounds = cand != nullptr ? min(E, k + k_extra) : k;
  const TokenSel s = select_token<J>(logits, n_parts, part_stride, offset, logits_out, t, E, k,
                                     score_fn, renorm, bias, n_bias_sets, modality, status,
                                     rounds);
  if (lane < k) {
    ids[t * k + lane] = s.e;
    gates[t * k + lane] = s.g;
  }
  if (cand != nullptr) {
    // candidates k .. k + k_extra - 1 (-1 past E), and per selection the value the gates are
    // computed from: the unbiased score (renorm) or the raw gate (no renorm)
    if (lane >= k && lane < k + k_extra) cand[t * k_extra + (lane - k)] = lane < rounds ? s.e : -1;
    if (lane < k + k_extra)
      cand_val[t * (k + k_extra) + lane] = lane < rounds ? (renorm ? s.sc : s.g) : 0.0f;
  }
}

// Top-k and the dispatch's rank pass in one launch: block b selects the experts of the
// kRankTile tokens of tile b (one warp per token, the selection above), then its first warp
// ranks the tile's assignments in token order and writes the tile's per-expert histogram --
// the rank pass's outputs for that tile.
template <int J>
__global__ void __launch_bounds__(32 * kRankTile) route_topk_rank_kernel(
    const float* __restrict__ logits, int n_parts, int64_t part_stride,
    const float* __restrict__ offset, float* __restrict__ logits_out, int64_t N, int E, int k,
    int score_fn, int renorm, const float* __restrict__ bias, int n_bias_sets,
    const uint8_t* __restrict__ modality, int32_t* __restrict__ ids, float* __restrict__ gates,
    int* status, int32_t* __restrict__ local_rank, int32_t* __restrict__ tile_hist) {
  pdl_wait();
  extern __shared__ int32_t sm[];
  int32_t* cnt = sm;       // [E]
  int32_t* sid = sm + E;   // [kRankTile * k]
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kRankTile;
  const int ntok = (int)min((int64_t)kRankTile, N - t0);
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  if (w < ntok) {
    const int64_t t = t0 + w;
    const TokenSel s = select_token<J>(logits, n_parts, part_stride, offset, logits_out, t, E,
                                       k, score_fn, renorm, bias, n_bias_sets, modality, status,
                                       k);
    if (lane < k) {
      ids[t * k + lane] = s.e;
      gates[t * k + lane] = s.g;
      sid[w * k + lane] = s.e;
    }
  }
  __syncthreads();
  if (w == 0) {
    const bool bad = warp_rank_walk(sid, ntok, k, cnt, lane, [&](int t, int j, int r) {
      local_rank[(t0 + t) * k + j] = r;
    });
    if (bad && lane == 0) report_status(status, kStatusInvalidInput);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) tile_hist[(int64_t)blockIdx.x * E + e] = cnt[e];
}

template <int J>
cudaError_t launch_j(const float* logits, int n_parts, int64_t part_stride, const float* offset,
                     float* logits_out, int64_t N, int E, int k, int score_fn, int renorm,
                     const float* bias, int n_bias_sets, const uint8_t* modality,
                     int32_t* ids, float* gates, int* status, int k_extra, int32_t* cand,
                     float* cand_val, cudaStream_t stream) {
  const int threads = 256;
  const int64_t blocks = (N * 32 + threads - 1) / threads;
  launch_pdl(route_topk_kernel<J>, (unsigned)blocks, threads, 0, stream, 
      logits, n_parts, part_stride, offset, logits_out, N, E, k, score_fn, renorm, bias,
      n_bias_sets, modality, ids, gates, status, k_extra, cand, cand_val);
  return cudaGetLastError();
}

template <int J>
cudaError_t launch_rank_j(const float* logits, int n_parts, int64_t part_stride,
                          const float* offset, float* logits_out, int64_t N, int E, int k,
                          int score_fn, int renorm, const float* bias, int n_bias_sets,
                          const uint8_t* modality, int32_t* ids, float* gates, int* status,
                          int32_t* local_rank, int32_t* tile_hist, cudaStream_t stream) {
  const int64_t tiles = (N + kRankTile - 1) / kRankTile;
  const size_t smem = sizeof(int32_t) * ((size_t)E + (size_t)kRankTile * k);
  launch_pdl(route_topk_rank_kernel<J>, (unsigned)tiles, 32 * kRankTile, smem, stream, logits,
             n_parts, part_stride, offset, logits_out, N, E, k, score_fn, renorm, bias,
             n_bias_sets, modality, ids, gates, status, local_rank, tile_hist);
  return cudaGetLastError();
}

// MurmurHash3's 32-bit finaliser (A. Appleby, public domain): a bijection that mixes every
// input bit into every output bit.
__device__ __forceinline__ uint32_t fmix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85ebca6bu;
  h ^= h >> 13;
  h *= 0xc2b2ae35u;
  h ^= h >> 16;
  return h;
}

// Hash router ("Le groupe d'experts (MoE)", exercise "Medium": deterministic, not learned).
// Expert e's key for token id t is fmix32(t * 0x9E3779B1 + e); the k largest keys win (they
// are distinct within a token), listed by descending key; every gate is 1/k.
template <int J>
__global__ void __launch_bounds__(256) hash_topk_kernel(const int32_t* __restrict__ token_ids,
                                                        int64_t N, int E, int k,
                                                        int32_t* __restrict__ ids,
                                                        float* __restrict__ gates) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= N) return;
  const uint32_t base = (uint32_t)token_ids[t] * 0x9E3779B1u;
  uint32_t key[J];
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int e = lane + 32 * j;
    key[j] = e < E ? fmix32(base + (uint32_t)e) : 0u;
  }
  uint32_t taken = 0;
  int my_e = -1;
  for (int r = 0; r < k; ++r) {
    uint32_t bk = 0;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u) && (be == 0x7fffffff || key[j] > bk)) {
        bk = key[j];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (oe != 0x7fffffff && (be == 0x7fffffff || ok > bk || (ok == bk && oe < be))) {
        bk = ok;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == r) my_e = be;
  }
  if (lane < k) {
    ids[t * k + lane] = my_e;
    gates[t * k + lane] = 1.0f / (float)k;
  }
}

}  // namespace

// Opt-in (MOE_B200_FUSED_TOPK_RANK=1): the fusion saves a launch but its 1024-thread blocks
// ran the top-k slower than the 256-thread top-k kernel, and the capacity and Switch layers
// measured 0.7-1.2 % slower per step with it (0.3104 vs 0.3081 ms, 0.2708 vs 0.2675 ms).
bool fused_topk_rank_enabled() {
  const char* v = std::getenv("MOE_B200_FUSED_TOPK_RANK");
  return v != nullptr && v[0] == '1';
}

cudaError_t launch_route_topk_rank(const float* logits, int n_parts, int64_t part_stride,
                                   const float* offset, float* logits_out, int64_t N, int E,
                                   int k, int score_fn, int renorm, const float* bias,
                                   int n_bias_sets, const uint8_t* modality, int32_t* ids,
                                   float* gates, int* status, int32_t* local_rank,
                                   int32_t* tile_hist, cudaStream_t stream, int* launches) {
  if (N == 0) return cudaSuccess;
  ++*launches;
  const int J = (E + 31) / 32;
#define MOE_ROUTE_RANK_CASE(JJ) \
  if (J <= JJ)                  \
    return launch_rank_j<JJ>(logits, n_parts, part_stride, offset, logits_out, N, E, k, score_fn, renorm, bias, n_bias_sets, modality, ids, gates, status, local_rank, tile_hist, stream);
  MOE_ROUTE_RANK_CASE(1)
  MOE_ROUTE_RANK_CASE(2)
  MOE_ROUTE_RANK_CASE(4)
  MOE_ROUTE_RANK_CASE(8)
  MOE_ROUTE_RANK_CASE(12)  // E <= kFusedTopkRankMaxE = 384
#undef MOE_ROUTE_RANK_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_route_hash(const int32_t* token_ids, int64_t N, int E, int k, int32_t* ids,
                              float* gates, cudaStream_t stream, int* launches) {
  if (N == 0) return cudaSuccess;
  ++*launches;
  const int J = (E + 31) / 32;
  const unsigned blocks = (unsigned)((N * 32 + 255) / 256);
#define MOE_HASH_CASE(JJ) \
  if (J <= JJ) {          \
    launch_pdl(hash_topk_kernel<JJ>, blocks, 256, 0, stream, token_ids, N, E, k, ids, gates); \
    return cudaGetLastError(); \
  }
  MOE_HASH_CASE(1)
  MOE_HASH_CASE(2)
  MOE_HASH_CASE(4)
  MOE_HASH_CASE(8)
  MOE_HASH_CASE(12)
  MOE_HASH_CASE(16)
  MOE_HASH_CASE(32)
#undef MOE_HASH_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_route_topk(const float* logits, int n_parts, int64_t part_stride,
                              const float* offset, float* logits_out, int64_t N, int E, int k,
                              int score_fn, int renorm, const float* bias, int n_bias_sets,
                              const uint8_t* modality, int32_t* ids, float* gates,
                              int* status, cudaStream_t stream, int* launches, int k_extra,
                              int32_t* cand, float* cand_val) {
  if (N == 0) return cudaSuccess;
  if (cand != nullptr && k + k_extra > 32) return cudaErrorInvalidValue;
  ++*launches;
  const int J = (E + 31) / 32;
#define MOE_ROUTE_CASE(JJ) \
  if (J <= JJ)             \
    return launch_j<JJ>(logits, n_parts, part_stride, offset, logits_out, N, E, k, score_fn, renorm, bias, n_bias_sets, modality, ids, gates, status, k_extra, cand, cand_val, stream);
  MOE_ROUTE_CASE(1)
  MOE_ROUTE_CASE(2)
  MOE_ROUTE_CASE(4)
  MOE_ROUTE_CASE(8)
  MOE_ROUTE_CASE(12)
  MOE_ROUTE_CASE(16)
  MOE_ROUTE_CASE(32)
#undef MOE_ROUTE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe
