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

template <int J>  // keys per lane: E <= 32 * J
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

  // k rounds of warp arg-max (k + k_extra when the next-best candidates are asked for, at
  // most E).  Lane r keeps the r-th selection.
  const int rounds = cand != nullptr ? min(E, k + k_extra) : k;
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
  if (mine) {
    ids[t * k + lane] = my_e;
    gates[t * k + lane] = g;
  }
  if (cand != nullptr) {
    // candidates k .. k + k_extra - 1 (-1 past E), and per selection the value the gates are
    // computed from: the unbiased score (renorm) or the raw gate (no renorm)
    if (lane >= k && lane < k + k_extra) cand[t * k_extra + (lane - k)] = lane < rounds ? my_e : -1;
    if (lane < k + k_extra)
      cand_val[t * (k + k_extra) + lane] = lane < rounds ? (renorm ? my_sc : g) : 0.0f;
  }
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
