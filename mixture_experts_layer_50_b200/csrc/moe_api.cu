// C ABI of the MoE layer (declared in include/moe.h): argument checks, the workspace
// layout, and the order of launches on the caller's stream.  No entry point allocates
// device memory; none synchronises except moe_check_status and moe_forward_host.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <climits>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>
#include <utility>
#include <vector>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"

// NVTX range over the host-side span of an API call or of a stage of the fused forward:
// visible on a profiler's timeline and usable to filter kernels (ncu --nvtx --nvtx-include
// "moe_forward/"); a no-op when no tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

namespace {

thread_local std::string g_last_error;
thread_local int32_t g_last_launches = 0;

// Launch timing (moe_profile_begin / moe_profile_end).
struct Profile {
  int32_t max_calls = 0;
  int32_t call = -1;          // index of the call being recorded
  bool recording = false;     // inside a moe_forward call that is being recorded
  std::vector<std::vector<cudaEvent_t>> ev;
  bool active() const { return recording && call >= 0 && call < max_calls; }
};
thread_local Profile g_prof;

void prof_mark(cudaStream_t st) {
  if (!g_prof.active()) return;
  cudaEvent_t e;
  if (cudaEventCreate(&e) != cudaSuccess) return;
  cudaEventRecord(e, st);
  g_prof.ev[g_prof.call].push_back(e);
}
void prof_call_begin(cudaStream_t st) {
  if (g_prof.max_calls <= 0) return;
  ++g_prof.call;
  g_prof.recording = true;
  if (g_prof.active()) {
    g_prof.ev.emplace_back();
    prof_mark(st);
  }
}

moe_status fail(moe_status s, const char* msg) {
  g_last_error = msg;
  return s;
}

moe_status cuda_fail(cudaError_t e, const char* where) {
  char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", where, cudaGetErrorString(e));
  g_last_error = buf;
  return MOE_ERR_CUDA;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Ws {
  size_t status, logits, ids, gates, local_rank, tile_hist, tile_base, demand, counts, offsets,
      slot_row, row_token, drop_mask, xp, h, ye, x_stage, y_stage, x_stage2, y_stage2, balance,
      offsets_pad, logit_parts, rr_cand, rr_val, rr_drop1, rr_offer, rr_not_offer, rr_counts1,
      rr_scratch, total;
};

size_t el_size(const moe_config& c) { return c.dtype == MOE_DT_BF16 ? 2 : 4; }

// Router split-K: at most this many K slices.
constexpr int kMaxLogitSplits = 16;
int router_splits(const moe_config& c);

// Rows of the padded dispatch buffer [E][C] (0 without a capacity).
int64_t padded_rows(const moe_config& c) { return c.capacity > 0 ? (int64_t)c.E * c.capacity : 0; }

Ws layout(const moe_config& c) {
  Ws w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t N = (size_t)c.N, k = (size_t)c.k, E = (size_t)c.E, d = (size_t)c.d,
               F = (size_t)c.F, S = (size_t)c.n_shared, el = el_size(c);
  const size_t Nk = N * k;
  const size_t R = std::max(Nk, (size_t)padded_rows(c));  // routed region: compact or padded
  const size_t tiles = (N + moe::kRankTile - 1) / moe::kRankTile;
  w.status = take(256);
  w.logits = take(N * E * 4);
  w.ids = take(Nk * 4);
  w.gates = take(Nk * 4);
  w.local_rank = take(Nk * 4);
  w.tile_hist = take(tiles * E * 4);
  w.tile_base = take(tiles * E * 4);
  w.demand = take(E * 4);
  w.counts = take(E * 4);
  w.offsets = take((E + 1) * 4);
  w.slot_row = take(Nk * 4);
  w.row_token = take(R * 4);
  w.drop_mask = take(Nk);
  w.xp = take(R * d * el);
  w.h = take((R + S * N) * F * el);
  w.ye = take((R + S * N) * d * el);
  w.x_stage = take(N * d * el);
  w.y_stage = take(N * d * el);
  w.x_stage2 = take(N * d * el);  // second staging pair: pipelined host batches
  w.y_stage2 = take(N * d * el);
  w.balance = take(moe::balance_scratch_bytes((int64_t)N, (int)E, std::max(1, c.n_bias_sets)));
  w.offsets_pad = take((E + 1) * 4);
  const int splits = router_splits(c);
  w.logit_parts = take(splits > 1 ? (size_t)splits * N * E * 4 : 0);
  // overflow policy "report": next-best candidates, their gate values, the first pass
  w.rr_cand = take(Nk * 4);
  w.rr_val = take(2 * Nk * 4);
  w.rr_drop1 = take(Nk);
  w.rr_offer = take(Nk * 4);
  w.rr_not_offer = take(Nk);
  w.rr_counts1 = take(E * 4);
  w.rr_scratch = take(3 * (E + 1) * 4);
  w.total = off;
  return w;
}

// The workspace of an expert-parallel rank: the layout of the same layer over world * N
// tokens, so that the owner's grouped GEMMs can take every row the ranks may send it (each
// token sends at most one row per expert, so at most world * N * k rows arrive).
moe_config ep_ws_config(const moe_config& c, int32_t world) {
  moe_config w = c;
  w.N = c.N * world;
  w.capacity = 0;
  return w;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// Ticket counter of the dispatch scan: an int in the zeroed 256-byte status region (the
// status word is at byte 0); every scan leaves it at zero.
int32_t* arrive_counter(void* ws, const Ws& L) { return at<int32_t>(ws, L.status + 128); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status check_cfg(const moe_config* c) {
  if (c == nullptr) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (c->N < 0) return fail(MOE_ERR_INVALID_ARG, "N < 0");
  if (c->d <= 0 || c->F <= 0) return fail(MOE_ERR_INVALID_ARG, "d and F must be positive");
  if (c->E < 1) return fail(MOE_ERR_INVALID_ARG, "E < 1");
  if (c->k < 1 || c->k > c->E) return fail(MOE_ERR_INVALID_ARG, "k must be in [1, E]");
  if (c->E > 1024) return fail(MOE_ERR_UNSUPPORTED, "E > 1024");
  if (c->k > 32) return fail(MOE_ERR_UNSUPPORTED, "k > 32");
  if (c->n_shared < 0) return fail(MOE_ERR_INVALID_ARG, "n_shared < 0");
  if (c->n_shared > 1) return fail(MOE_ERR_UNSUPPORTED, "n_shared > 1");
  if (c->score_fn != MOE_SCORE_SOFTMAX && c->score_fn != MOE_SCORE_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "unknown score_fn");
  if (c->renorm != 0 && c->renorm != 1) return fail(MOE_ERR_INVALID_ARG, "renorm must be 0 or 1");
  if (c->act != MOE_ACT_SWIGLU && c->act != MOE_ACT_RELU)
    return fail(MOE_ERR_INVALID_ARG, "unknown act");
  if (c->dtype != MOE_DT_BF16 && c->dtype != MOE_DT_F32)
    return fail(MOE_ERR_INVALID_ARG, "unknown dtype");
  if (c->n_bias_sets < 0) return fail(MOE_ERR_INVALID_ARG, "n_bias_sets < 0");
  if (!(c->clamp == c->clamp)) return fail(MOE_ERR_INVALID_ARG, "clamp is NaN");
  if (c->dtype == MOE_DT_BF16 && (c->d % 8 != 0 || c->F % 8 != 0))
    return fail(MOE_ERR_UNSUPPORTED, "bf16 layers need d and F multiples of 8");
  if (c->dtype == MOE_DT_F32 && (c->d % 4 != 0 || c->d > 4096 || c->F > 4096))
    return fail(MOE_ERR_UNSUPPORTED, "fp32 layers need d a multiple of 4, d and F at most 4096");
  const int64_t rows = c->N * (int64_t)c->k + c->N * (int64_t)c->n_shared;
  if (rows > (int64_t)INT32_MAX / 2) return fail(MOE_ERR_UNSUPPORTED, "N*k too large for int32 rows");
  return MOE_OK;
}

moe_status check_ws(const moe_config* c, void* ws) {
  if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(ws, 256)) return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  (void)c;
  return MOE_OK;
}

moe_status need(const void* p, const char* name) {
  if (p == nullptr) {
    std::string m = std::string(name) + " is NULL";
    return fail(MOE_ERR_INVALID_ARG, m.c_str());
  }
  if (!aligned(p, 16)) {
    std::string m = std::string(name) + " must be 16-byte aligned";
    return fail(MOE_ERR_UNSUPPORTED, m.c_str());
  }
  return MOE_OK;
}

moe_status check_bias(const moe_config* c, const float* bias, const uint8_t* modality) {
  if (c->n_bias_sets == 0 && bias != nullptr)
    return fail(MOE_ERR_INVALID_ARG, "bias given but n_bias_sets == 0");
  if (c->n_bias_sets > 0 && bias == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "n_bias_sets > 0 but bias is NULL");
  if (c->n_bias_sets > 1 && modality == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "several bias sets need the modality flags");
  return MOE_OK;
}

#define MOE_TRY(expr)               \
  do {                              \
    const moe_status _s = (expr);   \
    if (_s != MOE_OK) return _s;    \
  } while (0)
#define MOE_CUDA(expr, where)                        \
  do {                                               \
    const cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

// ---- the stages, shared by the split entry points and moe_forward --------------------

// Where the top-k kernel reads the router logits: `n_parts` split-K slices `part_stride`
// floats apart that it adds in order (plus `offset`), writing the sums to `final_out`; or, with
// one part and no offset, the finished logits themselves.
struct LogitSrc {
  const float* src;
  int n_parts;
  int64_t part_stride;
  const float* offset;
  float* final_out;
};

LogitSrc finished_logits(const float* z) { return LogitSrc{z, 1, 0, nullptr, nullptr}; }

// Number of K slices for the router GEMM: a launch with few output tiles (few 128-token
// tiles, or one tile column) would run on a fraction of the SMs, so its K loop is split over
// more CTAs (about 128 work items, at most kMaxLogitSplits slices); the partial logits sit
// in the workspace and the top-k kernel adds them in slice order.

int router_splits(const moe_config& c) {
  if (c.dtype != MOE_DT_BF16 || c.N == 0) return 1;
  const int bn = moe::router_tile_n(c.E);
  const int64_t tiles = ((c.N + 127) / 128) * ((c.E + bn - 1) / bn);
  const int nk = (c.d + 63) / 64;
  int64_t want = 128 / tiles;
  if (want < 2) return 1;
  int splits = (int)std::min<int64_t>({want, (int64_t)kMaxLogitSplits, (int64_t)nk});
  const int per = (nk + splits - 1) / splits;
  return (nk + per - 1) / per;  // no empty slice
}

moe_status stage_logits(const moe_config& c, const Ws& L, void* ws, const void* x,
                        const void* W_g, const float* logit_offset, float* logits, int* status,
                        cudaStream_t st, int* launches, LogitSrc* out) {
  *out = finished_logits(logits);
  if (c.N == 0) return MOE_OK;
  if (c.dtype == MOE_DT_F32) {
    MOE_CUDA(moe::launch_router_f32((const float*)x, (const float*)W_g, logit_offset, c.N, c.d,
                                    c.E, logits, st, launches),
             "router (fp32)");
    prof_mark(st);
    return MOE_OK;
  }
  moe::GroupedGemm g{};
  g.a = nullptr;
  g.a_shared = x;
  g.rows_a_shared = c.N;
  g.shared_a_row0 = 0;
  g.b = W_g;
  g.groups_b = 1;
  g.rows_b = c.E;
  g.K = c.d;
  g.offsets = nullptr;
  g.n_routed = 0;
  g.has_shared = 1;
  g.shared_rows = c.N;
  g.shared_out_row0 = 0;
  g.n_out = c.E;
  g.epilogue = moe::kEpiStoreF32;
  g.col_bias = logit_offset;
  g.out = logits;
  g.ld_out = c.E;
  g.rows_out = c.N;
  g.status = status;
  const int splits = router_splits(c);
  if (splits > 1) {
    float* parts = at<float>(ws, L.logit_parts);
    g.k_splits = splits;
    g.split_rows = c.N;
    g.col_bias = nullptr;
    g.out = parts;
    g.rows_out = c.N * splits;
    *out = LogitSrc{parts, splits, c.N * (int64_t)c.E, logit_offset, logits};
  }
  const char* why = "router GEMM launch";
  MOE_CUDA(moe::launch_grouped_gemm(g, st, launches, &why), why);
  prof_mark(st);
  return MOE_OK;
}

moe_status stage_route(const moe_config& c, const LogitSrc& z, const float* bias,
                       const uint8_t* modality, int32_t* ids, float* gates, int* status,
                       cudaStream_t st, int* launches) {
  MOE_CUDA(moe::launch_route_topk(z.src, z.n_parts, z.part_stride, z.offset, z.final_out, c.N,
                                  c.E, c.k, c.score_fn, c.renorm, bias, c.n_bias_sets, modality,
                                  ids, gates, status, st, launches),
           "top-k routing");
  prof_mark(st);
  return MOE_OK;
}

// A batch that takes the three dispatch passes (not a small one) runs top-k and the rank
// pass as one launch (route_topk_rank); stage_dispatch then skips its rank pass.
// (E <= kFusedTopkRankMaxE: with 1024 threads a block, more keys per lane would spill.)
bool fuse_topk_rank(const moe_config& c) {
  return c.N > 0 && c.E <= moe::kFusedTopkRankMaxE && moe::fused_topk_rank_enabled() &&
         !moe::use_small_dispatch(c.N, c.k, c.E);
}

moe_status stage_route_rank(const moe_config& c, const Ws& L, void* ws, const LogitSrc& z,
                            const float* bias, const uint8_t* modality, int32_t* ids,
                            float* gates, int* status, cudaStream_t st, int* launches) {
  MOE_CUDA(moe::launch_route_topk_rank(z.src, z.n_parts, z.part_stride, z.offset, z.final_out,
                                       c.N, c.E, c.k, c.score_fn, c.renorm, bias, c.n_bias_sets,
                                       modality, ids, gates, status,
                                       at<int32_t>(ws, L.local_rank),
                                       at<int32_t>(ws, L.tile_hist), st, launches),
           "top-k routing with the rank pass");
  prof_mark(st);
  return MOE_OK;
}

// Ranks, capacity, offsets, slot rows; gathers x into xp when xp != nullptr.  ranked: the rank
// pass already ran (stage_route_rank) and only the scan and scatter passes remain.
moe_status stage_dispatch(const moe_config& c, const Ws& L, void* ws, const int32_t* ids,
                          const uint8_t* drop_in, int64_t C, int32_t* demand, int32_t* counts,
                          int32_t* offsets, int32_t* slot_row, int32_t* row_token,
                          uint8_t* drop_out, const void* x, void* xp, cudaStream_t st,
                          int* launches, const int32_t* cap_e = nullptr,
                          bool ranked = false, const moe::RemoteRows* rem = nullptr) {
  int* status = at<int>(ws, L.status);
  if (!ranked && moe::use_small_dispatch(c.N, c.k, c.E)) {
    // a small batch: the three passes in one launch, with the same outputs
    MOE_CUDA(moe::launch_dispatch_small(ids, drop_in, c.N, c.k, c.E, C, cap_e, demand, counts,
                                        offsets, slot_row, row_token, drop_out, x, xp,
                                        (int)(c.d * el_size(c)), status, st, launches, rem),
             "dispatch (small batch)");
    prof_mark(st);
    return MOE_OK;
  }
  if (!ranked) {
    MOE_CUDA(moe::launch_rank_local(ids, drop_in, c.N, c.k, c.E, at<int32_t>(ws, L.local_rank),
                                    at<int32_t>(ws, L.tile_hist), status, st, launches),
             "rank pass");
    prof_mark(st);
  }
  MOE_CUDA(moe::launch_dispatch_scan(at<int32_t>(ws, L.tile_hist), c.N, c.E, C,
                                     at<int32_t>(ws, L.tile_base), demand, counts, offsets,
                                     arrive_counter(ws, L), st, launches, cap_e),
           "scan pass");
  prof_mark(st);
  MOE_CUDA(moe::launch_dispatch_scatter(ids, at<int32_t>(ws, L.local_rank),
                                        at<int32_t>(ws, L.tile_base), offsets, c.N, c.k, c.E, C,
                                        slot_row, row_token, drop_out, x, xp,
                                        (int)(c.d * el_size(c)), st, launches, cap_e, rem),
           "scatter pass");
  prof_mark(st);
  return MOE_OK;
}

// Routing under the overflow policy "report" ("Mixture-of-Experts : routage et capacité",
// table "Politiques de débordement", row "Report sur E2/E3"): the top-k kernel also lists each
// token's next k candidates; a plain capacity pass finds the dropped slots; each dropped slot
// is offered the token's next unused candidate; the offers are ranked per expert in token
// order like the first pass and taken while the expert has room; the gates are recomputed
// over the final slot list.  Writes ids and gates (final), demand (first pass), drop_out
// (slots still dropped) and rerouted (optional).  Uses the workspace's rank arrays and slot_row.
moe_status stage_route_reroute(const moe_config& c, const Ws& L, void* ws, const LogitSrc& z,
                               const float* bias, const uint8_t* modality, int32_t* ids,
                               float* gates, int32_t* demand, uint8_t* drop_out,
                               uint8_t* rerouted, cudaStream_t st, int* launches) {
  int* status = at<int>(ws, L.status);
  int32_t* cand = at<int32_t>(ws, L.rr_cand);
  float* val = at<float>(ws, L.rr_val);
  uint8_t* drop1 = at<uint8_t>(ws, L.rr_drop1);
  int32_t* offer = at<int32_t>(ws, L.rr_offer);
  uint8_t* not_offer = at<uint8_t>(ws, L.rr_not_offer);
  int32_t* counts1 = at<int32_t>(ws, L.rr_counts1);
  int32_t* scratch = at<int32_t>(ws, L.rr_scratch);  // [3][E + 1]
  const int64_t E1 = c.E + 1;
  MOE_CUDA(moe::launch_route_topk(z.src, z.n_parts, z.part_stride, z.offset, z.final_out, c.N,
                                  c.E, c.k, c.score_fn, c.renorm, bias, c.n_bias_sets, modality,
                                  ids, gates, status, st, launches, c.k, cand, val),
           "top-k routing with candidates");
  prof_mark(st);
  // first pass: the plain capacity decision
  MOE_TRY(stage_dispatch(c, L, ws, ids, nullptr, c.capacity, demand, counts1, scratch,
                         at<int32_t>(ws, L.slot_row), nullptr, drop1, nullptr, nullptr, st,
                         launches));
  // offers to the next-best candidates, ranked per expert in token order
  MOE_CUDA(moe::launch_reroute_offer(ids, drop1, cand, c.N, c.k, offer, not_offer, st, launches),
           "reroute offers");
  prof_mark(st);
  MOE_CUDA(moe::launch_rank_local(offer, not_offer, c.N, c.k, c.E, at<int32_t>(ws, L.local_rank),
                                  at<int32_t>(ws, L.tile_hist), status, st, launches),
           "rank pass (offers)");
  prof_mark(st);
  MOE_CUDA(moe::launch_dispatch_scan(at<int32_t>(ws, L.tile_hist), c.N, c.E, 0,
                                     at<int32_t>(ws, L.tile_base), scratch + E1,
                                     scratch + 2 * E1, scratch, arrive_counter(ws, L), st,
                                     launches),
           "scan pass (offers)");
  prof_mark(st);
  MOE_CUDA(moe::launch_reroute_accept(ids, drop1, offer, not_offer, at<int32_t>(ws, L.local_rank),
                                      at<int32_t>(ws, L.tile_base), counts1, val, c.N, c.E, c.k,
                                      c.capacity, c.score_fn, c.renorm, gates, drop_out,
                                      rerouted, st, launches),
           "reroute decision");
  prof_mark(st);
  return MOE_OK;
}

// The two grouped GEMMs of the expert FFN (bf16).  Nk: rows of the routed region; the shared
// expert's N rows follow it.  The kernel choice depends on the configuration alone (not on
// the pointers), so moe_ffn_kernels can name it without any device memory, and the compact
// and the padded layouts of the same call take the same kernels.
moe::GroupedGemm gate_up_gemm(const moe_config& c, int64_t Nk, const void* xp, const void* x,
                              const void* W_gu, const int32_t* offsets, void* h, int* status) {
  moe::GroupedGemm g{};
  g.a = xp;
  g.rows_a = Nk;
  g.a_shared = c.n_shared ? x : xp;
  g.rows_a_shared = c.n_shared ? c.N : Nk;
  g.shared_a_row0 = 0;
  g.b = W_gu;
  g.groups_b = c.E + c.n_shared;
  g.rows_b = c.act == MOE_ACT_SWIGLU ? 2 * c.F : c.F;
  g.K = c.d;
  g.offsets = offsets;
  g.n_routed = c.E;
  g.has_shared = c.n_shared;
  g.shared_rows = c.N;
  g.shared_out_row0 = Nk;
  g.n_out = c.F;
  g.epilogue = c.act == MOE_ACT_SWIGLU ? moe::kEpiSwiglu : moe::kEpiRelu;
  g.clamp = c.clamp;
  g.out = h;
  g.ld_out = c.F;
  g.rows_out = Nk + c.n_shared * c.N;
  g.max_rows_routed = Nk;
  g.rows_per_group_hint = c.N * (int64_t)c.k / c.E;
  g.status = status;
  return g;
}

moe::GroupedGemm down_gemm(const moe_config& c, int64_t Nk, const void* h, const void* W_down,
                           const int32_t* offsets, void* ye, int* status) {
  moe::GroupedGemm g{};
  g.a = h;
  g.rows_a = Nk + c.n_shared * c.N;
  g.a_shared = h;
  g.rows_a_shared = g.rows_a;
  g.shared_a_row0 = Nk;
  g.b = W_down;
  g.groups_b = c.E + c.n_shared;
  g.rows_b = c.d;
  g.K = c.F;
  g.offsets = offsets;
  g.n_routed = c.E;
  g.has_shared = c.n_shared;
  g.shared_rows = c.N;
  g.shared_out_row0 = Nk;
  g.n_out = c.d;
  g.epilogue = moe::kEpiStoreBf16;
  g.out = ye;
  g.ld_out = c.d;
  g.rows_out = g.rows_a;
  g.max_rows_routed = Nk;
  g.rows_per_group_hint = c.N * (int64_t)c.k / c.E;
  g.status = status;
  return g;
}

// R: rows of the routed region of xp / h / ye (N k for the compact layout, E C for the
// padded one); the shared expert's rows follow it in h, and in ye unless y_shared is given:
// then (bf16) the down GEMM writes the shared expert's output row t straight into y_shared[t]
// (the layer output, which stage_combine then completes in place).
moe_status stage_ffn(const moe_config& c, const Ws& L, void* ws, const void* xp,
                     const int32_t* offsets, const void* x, const void* W_gu,
                     const void* W_down, void* ye, cudaStream_t st, int* launches,
                     int64_t R = -1, void* y_shared = nullptr, int64_t group_rows_max = -1,
                     bool routed_only = false) {
  if (c.N == 0) return MOE_OK;
  const int64_t Nk = R >= 0 ? R : c.N * (int64_t)c.k;
  // the most rows a routed group can have: N in the layer's own compact layout (a token
  // picks an expert at most once); otherwise what the caller states, or the whole region
  const int64_t grp_max = group_rows_max > 0 ? group_rows_max : Nk;
  if (c.dtype == MOE_DT_F32) {
    MOE_CUDA(moe::launch_ffn_f32((const float*)xp, (const float*)x, offsets, c.N, Nk, c.d, c.E,
                                 c.F, c.n_shared, c.act, c.clamp, (const float*)W_gu,
                                 (const float*)W_down, at<float>(ws, L.h), (float*)ye, st,
                                 launches),
             "fp32 expert FFN");
    prof_mark(st);
    return MOE_OK;
  }
  int* status = at<int>(ws, L.status);
  void* h = at<char>(ws, L.h);
  moe::GroupedGemm g1 = gate_up_gemm(c, Nk, xp, x, W_gu, offsets, h, status);
  g1.max_group_rows = grp_max;
  if (routed_only) g1.has_shared = 0;  // the shared expert runs on the side stream
  const char* why = "gate/up GEMM launch";
  MOE_CUDA(moe::launch_grouped_gemm(g1, st, launches, &why), why);
  prof_mark(st);

  moe::GroupedGemm g2 = down_gemm(c, Nk, h, W_down, offsets, ye, status);
  g2.max_group_rows = grp_max;
  if (routed_only) g2.has_shared = 0;
  if (y_shared != nullptr && c.n_shared) {
    g2.out_shared = y_shared;
    g2.shared_out_row0 = 0;
  }
  why = "down GEMM launch";
  MOE_CUDA(moe::launch_grouped_gemm(g2, st, launches, &why), why);
  prof_mark(st);
  return MOE_OK;
}

// shared_in_y: stage_ffn wrote the shared expert's rows into y (bf16 only).
moe_status stage_combine(const moe_config& c, const void* ye, const int32_t* slot_row,
                         const float* gates, void* y, cudaStream_t st, int* launches,
                         int64_t R = -1, bool shared_in_y = false,
                         const moe::RemoteSrc* rem = nullptr) {
  const bool in_y = shared_in_y && c.n_shared && c.dtype == MOE_DT_BF16;
  const int64_t shared_row0 = (c.n_shared && !in_y) ? (R >= 0 ? R : c.N * (int64_t)c.k) : -1;
  MOE_CUDA(moe::launch_combine(ye, slot_row, gates, c.N, c.k, c.d, shared_row0, in_y ? 1 : 0,
                               c.dtype == MOE_DT_F32, y, st, launches, rem),
           "combine");
  prof_mark(st);
  return MOE_OK;
}

// MOE_B200_DEBUG=1: the fused forward calls check their dispatch layout on the host after the
// dispatch passes (moe_check_dispatch_host).  Synchronises the stream: for eager calls only,
// never inside a stream capture.
bool debug_checks() {
  const char* v = std::getenv("MOE_B200_DEBUG");
  return v != nullptr && v[0] == '1';
}

moe_status check_dispatch_device(const moe_config& c, const int32_t* ids, const uint8_t* drop,
                                 const int32_t* counts, const int32_t* demand,
                                 const int32_t* offsets, const int32_t* slot_row,
                                 const int32_t* row_token, int64_t capacity, cudaStream_t st) {
  const size_t nk = (size_t)c.N * c.k, E = (size_t)c.E;
  std::vector<int32_t> h_ids(nk), h_cnt(E), h_dem(E), h_off(E + 1), h_slot(nk);
  std::vector<uint8_t> h_drop(nk);
  MOE_CUDA(cudaStreamSynchronize(st), "debug check: synchronise");
  auto get = [&](void* dst, const void* src, size_t bytes) {
    return bytes == 0 ? cudaSuccess : cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost);
  };
  MOE_CUDA(get(h_ids.data(), ids, nk * 4), "debug check: copy ids");
  MOE_CUDA(get(h_drop.data(), drop, nk), "debug check: copy drop mask");
  MOE_CUDA(get(h_cnt.data(), counts, E * 4), "debug check: copy counts");
  if (demand != nullptr) MOE_CUDA(get(h_dem.data(), demand, E * 4), "debug check: copy demand");
  MOE_CUDA(get(h_off.data(), offsets, (E + 1) * 4), "debug check: copy offsets");
  MOE_CUDA(get(h_slot.data(), slot_row, nk * 4), "debug check: copy slot rows");
  std::vector<int32_t> h_rt;
  if (row_token != nullptr && h_off[E] >= 0 && (size_t)h_off[E] <= nk) {
    h_rt.resize((size_t)h_off[E]);
    MOE_CUDA(get(h_rt.data(), row_token, h_rt.size() * 4), "debug check: copy row map");
  }
  char msg[200];
  const moe_status s = moe_check_dispatch_host(
      c.N, c.k, c.E, capacity, h_ids.data(), h_drop.data(), h_cnt.data(),
      demand != nullptr ? h_dem.data() : nullptr, h_off.data(), h_slot.data(),
      h_rt.empty() ? nullptr : h_rt.data(), msg, sizeof(msg));
  if (s != MOE_OK) {
    std::string m = std::string("dispatch layout check: ") + msg;
    return fail(s, m.c_str());
  }
  return MOE_OK;
}

// ---- the shared expert on a side stream ------------------------------------------------
// The shared expert reads x alone ("Des experts partagés": always on, for every token), so in
// the fused bf16 forward its two GEMMs run on a library stream forked from the caller's stream
// before the router and joined before the combine: the routing chain's small kernels (top-k,
// the dispatch passes) run beside the shared GEMMs' CTAs instead of between full-GPU GEMMs.
// The fork and join are event edges, so a stream capture takes the side stream in.  The
// stream and its two events are created by the first such call on a device and thread.
// Taken where the shared expert is at least a third of the expert work (k <= 2): the capacity
// and Switch layers gained 4.7-6.3 % per step (0.3095 -> 0.2950 ms, 0.2705 -> 0.2535 ms),
// while the k = 6 and k = 8 ridge-point layers, whose dispatch copies compete with the shared
// GEMMs for HBM, came out even or slightly slower.
// MOE_B200_SHARED_STREAM=0 keeps the shared expert inside the routed GEMM launches.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxSideDevices = 64;
thread_local SideStream g_side[kMaxSideDevices];

bool shared_stream_enabled() {
  const char* v = std::getenv("MOE_B200_SHARED_STREAM");
  return !(v != nullptr && v[0] == '0');
}

moe_status side_stream(SideStream** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxSideDevices) return fail(MOE_ERR_UNSUPPORTED, "device ordinal >= 64");
  SideStream& ss = g_side[dev];
  if (ss.s == nullptr) {
    MOE_CUDA(cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking), "create side stream");
    MOE_CUDA(cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming), "create event");
    MOE_CUDA(cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming), "create event");
  }
  *out = &ss;
  return MOE_OK;
}

// The shared expert's gate/up and down GEMMs alone (bf16): one group, its weights the slice
// at index E; hidden rows at h[N k + t], output rows straight into y[t].
moe_status stage_shared_ffn(const moe_config& c, const Ws& L, void* ws, const void* x,
                            const void* W_gu, const void* W_down, void* y, cudaStream_t st,
                            int* launches) {
  int* status = at<int>(ws, L.status);
  void* h = at<char>(ws, L.h);
  const int64_t Nk = c.N * (int64_t)c.k;
  const int64_t gu_rows = c.act == MOE_ACT_SWIGLU ? 2 * (int64_t)c.F : c.F;
  moe::GroupedGemm g1 = gate_up_gemm(c, Nk, nullptr, x, W_gu, nullptr, h, status);
  g1.a = nullptr;
  g1.n_routed = 0;
  g1.b = static_cast<const char*>(W_gu) + (size_t)c.E * gu_rows * c.d * 2;
  g1.groups_b = 1;
  g1.max_rows_routed = 0;
  const char* why = "shared gate/up GEMM launch";
  MOE_CUDA(moe::launch_grouped_gemm(g1, st, launches, &why), why);
  moe::GroupedGemm g2 = down_gemm(c, Nk, h, W_down, nullptr, y, status);
  g2.n_routed = 0;
  g2.b = static_cast<const char*>(W_down) + (size_t)c.E * c.d * c.F * 2;
  g2.groups_b = 1;
  g2.max_rows_routed = 0;
  g2.out_shared = y;
  g2.shared_out_row0 = 0;
  why = "shared down GEMM launch";
  MOE_CUDA(moe::launch_grouped_gemm(g2, st, launches, &why), why);
  return MOE_OK;
}

moe_status forward_impl(const moe_config* cfg, const void* x, const void* W_g,
                        const float* logit_offset, const float* bias, const uint8_t* modality,
                        const void* W_gu, const void* W_down, void* y,
                        const moe_route_out* ro, void* ws, cudaStream_t st, int* launches,
                        bool reroute = false, uint8_t* rerouted = nullptr) {
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  int* status = at<int>(ws, L.status);
  auto pick = [&](auto* user, size_t off) {
    using T = std::remove_pointer_t<decltype(user)>;
    return user != nullptr ? user : at<T>(ws, off);
  };
  float* logits = pick(ro ? ro->logits : (float*)nullptr, L.logits);
  int32_t* ids = pick(ro ? ro->ids : (int32_t*)nullptr, L.ids);
  float* gates = pick(ro ? ro->gates : (float*)nullptr, L.gates);
  int32_t* counts = pick(ro ? ro->counts : (int32_t*)nullptr, L.counts);
  int32_t* demand = pick(ro ? ro->demand : (int32_t*)nullptr, L.demand);
  uint8_t* drop = pick(ro ? ro->drop_mask : (uint8_t*)nullptr, L.drop_mask);
  int32_t* offsets = pick(ro ? ro->offsets : (int32_t*)nullptr, L.offsets);
  void* xp = at<char>(ws, L.xp);
  void* ye = at<char>(ws, L.ye);
  int32_t* row_token = at<int32_t>(ws, L.row_token);
  prof_call_begin(st);
  // the shared expert on the side stream (not while per-launch timing records this call: the
  // recorded events assume one stream)
  SideStream* side = nullptr;
  if (c.dtype == MOE_DT_BF16 && c.n_shared && c.N > 0 && c.k <= 2 && shared_stream_enabled() &&
      !g_prof.active()) {
    MOE_TRY(side_stream(&side));
    MOE_CUDA(cudaEventRecord(side->fork, st), "fork the side stream");
  }
  LogitSrc zsrc;
  {
    NvtxRange r("moe.router");
    MOE_TRY(stage_logits(c, L, ws, x, W_g, logit_offset, logits, status, st, launches, &zsrc));
  }
  if (side != nullptr) {
    // launched after the router, so the router's CTAs are placed first
    NvtxRange r("moe.shared_expert");
    MOE_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0), "fork the side stream");
    MOE_TRY(stage_shared_ffn(c, L, ws, x, W_gu, W_down, y, side->s, launches));
    MOE_CUDA(cudaEventRecord(side->join, side->s), "join the side stream");
  }
  if (reroute && c.capacity > 0) {
    // final slots after the overflow policy; the capacity is already met, so the dispatch
    // below only lays the kept slots out (its demand output is scratch: demand keeps the
    // router's first-pass demand)
    NvtxRange r("moe.route_dispatch");
    MOE_TRY(stage_route_reroute(c, L, ws, zsrc, bias, modality, ids, gates, demand, drop,
                                rerouted, st, launches));
    MOE_TRY(stage_dispatch(c, L, ws, ids, drop, 0, at<int32_t>(ws, L.rr_scratch), counts,
                           offsets, at<int32_t>(ws, L.slot_row), row_token, drop, x, xp, st,
                           launches));
  } else {
    NvtxRange r("moe.route_dispatch");
    const bool fused = fuse_topk_rank(c);
    if (fused)
      MOE_TRY(stage_route_rank(c, L, ws, zsrc, bias, modality, ids, gates, status, st, launches));
    else
      MOE_TRY(stage_route(c, zsrc, bias, modality, ids, gates, status, st, launches));
    MOE_TRY(stage_dispatch(c, L, ws, ids, nullptr, c.capacity, demand, counts, offsets,
                           at<int32_t>(ws, L.slot_row), row_token, drop, x, xp, st,
                           launches, nullptr, fused));
    if (rerouted != nullptr && c.N > 0)
      MOE_CUDA(cudaMemsetAsync(rerouted, 0, (size_t)c.N * c.k, st), "clear rerouted flags");
  }
  if (debug_checks())
    MOE_TRY(check_dispatch_device(c, ids, drop, counts, (reroute && c.capacity > 0) ? nullptr : demand,
                                  offsets, at<int32_t>(ws, L.slot_row),
                                  at<int32_t>(ws, L.row_token), c.capacity, st));
  // fused layer: the shared expert's rows go straight into y (bf16), completed by the combine
  {
    NvtxRange r("moe.expert_ffn");
    MOE_TRY(stage_ffn(c, L, ws, xp, offsets, x, W_gu, W_down, ye, st, launches, -1, y, c.N,
                      side != nullptr));
  }
  if (side != nullptr) MOE_CUDA(cudaStreamWaitEvent(st, side->join, 0), "join the side stream");
  {
    NvtxRange r("moe.combine");
    MOE_TRY(stage_combine(c, ye, at<int32_t>(ws, L.slot_row), gates, y, st, launches, -1, true));
  }
  g_prof.recording = false;
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return layout(*cfg).total;
}

moe_status moe_workspace_init(void* ws, moe_stream_t stream) {
  if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  MOE_CUDA(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream), "workspace init");
  return MOE_OK;
}

int64_t moe_capacity(int64_t T, int32_t k, int32_t E, int64_t cf_num, int64_t cf_den) {
  if (cf_num <= 0) return 0;
  if (T < 0 || k < 1 || E < 1 || cf_den <= 0) return -1;
  const __int128 p = (__int128)T * k * cf_num;
  const __int128 q = (__int128)E * cf_den;
  return (int64_t)((p + q - 1) / q);
}

moe_status moe_route(const moe_config* cfg, const float* logits, const void* x,
                     const void* W_g, const float* logit_offset, const float* bias,
                     const uint8_t* modality, int32_t* ids, float* gates, int32_t* counts,
                     int32_t* demand, uint8_t* drop_mask, float* logits_out, void* ws,
                     moe_stream_t stream) {
  NvtxRange nvtx_range("moe_route");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  MOE_TRY(check_bias(cfg, bias, modality));
  if (logits == nullptr) {
    MOE_TRY(need(x, "x"));
    MOE_TRY(need(W_g, "W_g"));
  }
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  cudaStream_t st = (cudaStream_t)stream;
  int launches = 0;
  int* status = at<int>(ws, L.status);
  LogitSrc z = finished_logits(logits);
  if (logits == nullptr) {
    float* dst = logits_out != nullptr ? logits_out : at<float>(ws, L.logits);
    MOE_TRY(stage_logits(c, L, ws, x, W_g, logit_offset, dst, status, st, &launches, &z));
  }
  int32_t* ids_p = ids != nullptr ? ids : at<int32_t>(ws, L.ids);
  float* gates_p = gates != nullptr ? gates : at<float>(ws, L.gates);
  const bool fused = fuse_topk_rank(c);
  if (fused)
    MOE_TRY(stage_route_rank(c, L, ws, z, bias, modality, ids_p, gates_p, status, st, &launches));
  else
    MOE_TRY(stage_route(c, z, bias, modality, ids_p, gates_p, status, st, &launches));
  MOE_TRY(stage_dispatch(c, L, ws, ids_p, nullptr, c.capacity,
                         demand != nullptr ? demand : at<int32_t>(ws, L.demand),
                         counts != nullptr ? counts : at<int32_t>(ws, L.counts),
                         at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.slot_row), nullptr,
                         drop_mask != nullptr ? drop_mask : at<uint8_t>(ws, L.drop_mask),
                         nullptr, nullptr, st, &launches, nullptr, fused));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_route_reroute(const moe_config* cfg, const float* logits, const void* x,
                             const void* W_g, const float* logit_offset, const float* bias,
                             const uint8_t* modality, int32_t* ids, float* gates,
                             int32_t* counts, int32_t* demand, uint8_t* drop_mask,
                             uint8_t* rerouted, float* logits_out, void* ws,
                             moe_stream_t stream) {
  NvtxRange nvtx_range("moe_route_reroute");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  MOE_TRY(check_bias(cfg, bias, modality));
  if (cfg->k > 16) return fail(MOE_ERR_UNSUPPORTED, "the report overflow policy needs k <= 16");
  if (logits == nullptr) {
    MOE_TRY(need(x, "x"));
    MOE_TRY(need(W_g, "W_g"));
  }
  const moe_config& c = *cfg;
  if (c.capacity <= 0) {
    // no capacity: nothing overflows, plain routing
    MOE_TRY(moe_route(cfg, logits, x, W_g, logit_offset, bias, modality, ids, gates, counts,
                      demand, drop_mask, logits_out, ws, stream));
    if (rerouted != nullptr && c.N > 0)
      MOE_CUDA(cudaMemsetAsync(rerouted, 0, (size_t)c.N * c.k, (cudaStream_t)stream),
               "clear rerouted flags");
    return MOE_OK;
  }
  const Ws L = layout(c);
  cudaStream_t st = (cudaStream_t)stream;
  int launches = 0;
  int* status = at<int>(ws, L.status);
  LogitSrc z = finished_logits(logits);
  if (logits == nullptr) {
    float* dst = logits_out != nullptr ? logits_out : at<float>(ws, L.logits);
    MOE_TRY(stage_logits(c, L, ws, x, W_g, logit_offset, dst, status, st, &launches, &z));
  }
  int32_t* ids_p = ids != nullptr ? ids : at<int32_t>(ws, L.ids);
  float* gates_p = gates != nullptr ? gates : at<float>(ws, L.gates);
  uint8_t* drop_p = drop_mask != nullptr ? drop_mask : at<uint8_t>(ws, L.drop_mask);
  MOE_TRY(stage_route_reroute(c, L, ws, z, bias, modality, ids_p, gates_p,
                              demand != nullptr ? demand : at<int32_t>(ws, L.demand), drop_p,
                              rerouted, st, &launches));
  // kept assignments per expert after the policy
  MOE_TRY(stage_dispatch(c, L, ws, ids_p, drop_p, 0, at<int32_t>(ws, L.rr_scratch),
                         counts != nullptr ? counts : at<int32_t>(ws, L.counts),
                         at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.slot_row), nullptr, drop_p,
                         nullptr, nullptr, st, &launches));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_permute(const moe_config* cfg, const int32_t* ids, const uint8_t* drop_mask,
                       const void* x, int32_t* offsets, int32_t* row_token,
                       int32_t* slot_row, void* xp, void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_permute");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (ids == nullptr || offsets == nullptr || slot_row == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "ids, offsets and slot_row are required");
  MOE_TRY(need(x, "x"));
  MOE_TRY(need(xp, "xp"));
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  int launches = 0;
  MOE_TRY(stage_dispatch(c, L, ws, ids, drop_mask, 0, at<int32_t>(ws, L.demand),
                         at<int32_t>(ws, L.counts), offsets, slot_row, row_token, nullptr, x,
                         xp, (cudaStream_t)stream, &launches));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_expert_ffn(const moe_config* cfg, const void* xp, const int32_t* offsets,
                          const void* x, const void* W_gu, const void* W_down, void* ye,
                          void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_expert_ffn");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  MOE_TRY(need(xp, "xp"));
  if (offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "offsets is NULL");
  if (cfg->n_shared) MOE_TRY(need(x, "x"));
  MOE_TRY(need(W_gu, "W_gu"));
  MOE_TRY(need(W_down, "W_down"));
  MOE_TRY(need(ye, "ye"));
  int launches = 0;
  MOE_TRY(stage_ffn(*cfg, layout(*cfg), ws, xp, offsets, x, W_gu, W_down, ye,
                    (cudaStream_t)stream, &launches));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_ffn_kernels(const moe_config* cfg, char* gate_up, char* down, size_t len) {
  MOE_TRY(check_cfg(cfg));
  if (len == 0 && (gate_up != nullptr || down != nullptr))
    return fail(MOE_ERR_INVALID_ARG, "len is 0");
  const moe_config& c = *cfg;
  const char* gu = "ffn_up_f32_kernel (SIMT fp32)";
  const char* dn = "ffn_down_f32_kernel (SIMT fp32)";
  if (c.dtype == MOE_DT_BF16) {
    const int64_t Nk = c.N * (int64_t)c.k;
    // the choice of the fused forward calls, whose groups have at most N rows
    moe::GroupedGemm g1 = gate_up_gemm(c, Nk, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
    moe::GroupedGemm g2 = down_gemm(c, Nk, nullptr, nullptr, nullptr, nullptr, nullptr);
    g1.max_group_rows = g2.max_group_rows = c.N;
    gu = moe::grouped_gemm_kernel_name(g1);
    dn = moe::grouped_gemm_kernel_name(g2);
  }
  if (c.N == 0) gu = dn = "none";
  for (auto [buf, name] : {std::pair<char*, const char*>{gate_up, gu}, {down, dn}}) {
    if (buf == nullptr) continue;
    const size_t n = std::min(len - 1, std::strlen(name));
    std::memcpy(buf, name, n);
    buf[n] = '\0';
  }
  return MOE_OK;
}

moe_status moe_combine(const moe_config* cfg, const void* ye, const int32_t* slot_row,
                       const float* gates, void* y, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_combine");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(need(ye, "ye"));
  MOE_TRY(need(y, "y"));
  if (slot_row == nullptr || gates == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "slot_row and gates are required");
  int launches = 0;
  MOE_TRY(stage_combine(*cfg, ye, slot_row, gates, y, (cudaStream_t)stream, &launches));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_forward_reroute(const moe_config* cfg, const void* x, const void* W_g,
                               const float* logit_offset, const float* bias,
                               const uint8_t* modality, const void* W_gu, const void* W_down,
                               void* y, const moe_route_out* route_out, uint8_t* rerouted,
                               void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_forward_reroute");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  MOE_TRY(check_bias(cfg, bias, modality));
  if (cfg->k > 16) return fail(MOE_ERR_UNSUPPORTED, "the report overflow policy needs k <= 16");
  MOE_TRY(need(x, "x"));
  MOE_TRY(need(W_g, "W_g"));
  MOE_TRY(need(W_gu, "W_gu"));
  MOE_TRY(need(W_down, "W_down"));
  MOE_TRY(need(y, "y"));
  int launches = 0;
  const moe_status fs = forward_impl(cfg, x, W_g, logit_offset, bias, modality, W_gu, W_down,
                                     y, route_out, ws, (cudaStream_t)stream, &launches, true,
                                     rerouted);
  g_prof.recording = false;
  MOE_TRY(fs);
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_forward(const moe_config* cfg, const void* x, const void* W_g,
                       const float* logit_offset, const float* bias,
                       const uint8_t* modality, const void* W_gu, const void* W_down,
                       void* y, const moe_route_out* route_out, void* ws,
                       moe_stream_t stream) {
  NvtxRange nvtx_range("moe_forward");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  MOE_TRY(check_bias(cfg, bias, modality));
  MOE_TRY(need(x, "x"));
  MOE_TRY(need(W_g, "W_g"));
  MOE_TRY(need(W_gu, "W_gu"));
  MOE_TRY(need(W_down, "W_down"));
  MOE_TRY(need(y, "y"));
  int launches = 0;
  const moe_status fs = forward_impl(cfg, x, W_g, logit_offset, bias, modality, W_gu, W_down,
                                     y, route_out, ws, (cudaStream_t)stream, &launches);
  g_prof.recording = false;
  MOE_TRY(fs);
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_forward_routed(const moe_config* cfg, const void* x, const int32_t* ids,
                              const float* gates, const void* W_gu, const void* W_down,
                              void* y, const moe_route_out* route_out, void* ws,
                              moe_stream_t stream) {
  NvtxRange nvtx_range("moe_forward_routed");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (ids == nullptr || gates == nullptr) return fail(MOE_ERR_INVALID_ARG, "ids and gates are required");
  MOE_TRY(need(x, "x"));
  MOE_TRY(need(W_gu, "W_gu"));
  MOE_TRY(need(W_down, "W_down"));
  MOE_TRY(need(y, "y"));
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  cudaStream_t st = (cudaStream_t)stream;
  const moe_route_out* ro = route_out;
  int32_t* counts = (ro && ro->counts) ? ro->counts : at<int32_t>(ws, L.counts);
  int32_t* demand = (ro && ro->demand) ? ro->demand : at<int32_t>(ws, L.demand);
  uint8_t* drop = (ro && ro->drop_mask) ? ro->drop_mask : at<uint8_t>(ws, L.drop_mask);
  int32_t* offsets = (ro && ro->offsets) ? ro->offsets : at<int32_t>(ws, L.offsets);
  void* xp = at<char>(ws, L.xp);
  void* ye = at<char>(ws, L.ye);
  int launches = 0;
  MOE_TRY(stage_dispatch(c, L, ws, ids, nullptr, c.capacity, demand, counts, offsets,
                         at<int32_t>(ws, L.slot_row), at<int32_t>(ws, L.row_token), drop, x, xp,
                         st, &launches));
  MOE_TRY(stage_ffn(c, L, ws, xp, offsets, x, W_gu, W_down, ye, st, &launches, -1, y, c.N));
  MOE_TRY(stage_combine(c, ye, at<int32_t>(ws, L.slot_row), gates, y, st, &launches, -1, true));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_route_hash(const moe_config* cfg, const int32_t* token_ids, int32_t* ids,
                          float* gates, int32_t* counts, int32_t* demand, uint8_t* drop_mask,
                          void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_route_hash");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (token_ids == nullptr || ids == nullptr || gates == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "token_ids, ids and gates are required");
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  cudaStream_t st = (cudaStream_t)stream;
  int launches = 0;
  MOE_CUDA(moe::launch_route_hash(token_ids, c.N, c.E, c.k, ids, gates, st, &launches),
           "hash routing");
  MOE_TRY(stage_dispatch(c, L, ws, ids, nullptr, c.capacity,
                         demand != nullptr ? demand : at<int32_t>(ws, L.demand),
                         counts != nullptr ? counts : at<int32_t>(ws, L.counts),
                         at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.slot_row), nullptr,
                         drop_mask != nullptr ? drop_mask : at<uint8_t>(ws, L.drop_mask),
                         nullptr, nullptr, st, &launches));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_balance(const moe_config* cfg, const float* logits, const int32_t* ids,
                       const uint8_t* modality, float* f, float* P, float* aux,
                       int32_t* set_load, float* bias, float gamma, void* ws,
                       moe_stream_t stream) {
  NvtxRange nvtx_range("moe_balance");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (logits == nullptr || ids == nullptr) return fail(MOE_ERR_INVALID_ARG, "logits and ids are required");
  const int n_sets = std::max(1, cfg->n_bias_sets);
  if (n_sets > 8) return fail(MOE_ERR_UNSUPPORTED, "moe_balance handles at most 8 bias sets");
  if (n_sets > 1 && modality == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "several bias sets need the modality flags");
  if (!(gamma == gamma)) return fail(MOE_ERR_INVALID_ARG, "gamma is NaN");
  const Ws L = layout(*cfg);
  int launches = 0;
  MOE_CUDA(moe::launch_balance(logits, ids, modality, cfg->N, cfg->E, cfg->k, cfg->score_fn,
                               n_sets, at<char>(ws, L.balance), f, P, aux, set_load, bias, gamma,
                               (cudaStream_t)stream, &launches),
           "balance statistics");
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_permute_padded(const moe_config* cfg, const int32_t* ids,
                              const uint8_t* drop_mask, const void* x, int32_t* offsets_pad,
                              int32_t* counts, int32_t* row_token_pad, int32_t* slot_row,
                              void* xp_pad, void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_permute_padded");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (cfg->capacity <= 0) return fail(MOE_ERR_INVALID_ARG, "the padded layout needs capacity > 0");
  if (padded_rows(*cfg) > (int64_t)INT32_MAX / 2) return fail(MOE_ERR_UNSUPPORTED, "E*C too large");
  if (ids == nullptr || offsets_pad == nullptr || counts == nullptr || slot_row == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "ids, offsets_pad, counts and slot_row are required");
  MOE_TRY(need(x, "x"));
  MOE_TRY(need(xp_pad, "xp_pad"));
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  cudaStream_t st = (cudaStream_t)stream;
  int launches = 0;
  int* status = at<int>(ws, L.status);
  MOE_CUDA(moe::launch_rank_local(ids, drop_mask, c.N, c.k, c.E, at<int32_t>(ws, L.local_rank),
                                  at<int32_t>(ws, L.tile_hist), status, st, &launches),
           "rank pass");
  MOE_CUDA(moe::launch_dispatch_scan(at<int32_t>(ws, L.tile_hist), c.N, c.E, c.capacity,
                                     at<int32_t>(ws, L.tile_base), at<int32_t>(ws, L.demand),
                                     counts, at<int32_t>(ws, L.offsets),
                                     arrive_counter(ws, L), st, &launches),
           "scan pass");
  MOE_CUDA(moe::launch_pad_offsets(c.E, c.capacity, offsets_pad, st, &launches), "pad offsets");
  MOE_CUDA(moe::launch_dispatch_scatter(ids, at<int32_t>(ws, L.local_rank),
                                        at<int32_t>(ws, L.tile_base), offsets_pad, c.N, c.k, c.E,
                                        c.capacity, slot_row, row_token_pad, nullptr, x, xp_pad,
                                        (int)(c.d * el_size(c)), st, &launches),
           "scatter pass");
  MOE_CUDA(moe::launch_zero_padding(counts, c.E, c.capacity, xp_pad, (int)(c.d * el_size(c)),
                                    row_token_pad, st, &launches),
           "zero padding");
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_forward_padded(const moe_config* cfg, const void* x, const void* W_g,
                              const float* logit_offset, const float* bias,
                              const uint8_t* modality, const void* W_gu, const void* W_down,
                              void* y, const moe_route_out* ro, void* ws,
                              moe_stream_t stream) {
  NvtxRange nvtx_range("moe_forward_padded");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  MOE_TRY(check_bias(cfg, bias, modality));
  if (cfg->capacity <= 0) return fail(MOE_ERR_INVALID_ARG, "the padded layout needs capacity > 0");
  if (padded_rows(*cfg) + cfg->N > (int64_t)INT32_MAX / 2) return fail(MOE_ERR_UNSUPPORTED, "E*C too large");
  MOE_TRY(need(x, "x"));
  MOE_TRY(need(W_g, "W_g"));
  MOE_TRY(need(W_gu, "W_gu"));
  MOE_TRY(need(W_down, "W_down"));
  MOE_TRY(need(y, "y"));
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  cudaStream_t st = (cudaStream_t)stream;
  int* status = at<int>(ws, L.status);
  const int64_t R = padded_rows(c);
  float* logits = (ro && ro->logits) ? ro->logits : at<float>(ws, L.logits);
  int32_t* ids = (ro && ro->ids) ? ro->ids : at<int32_t>(ws, L.ids);
  float* gates = (ro && ro->gates) ? ro->gates : at<float>(ws, L.gates);
  int32_t* counts = (ro && ro->counts) ? ro->counts : at<int32_t>(ws, L.counts);
  int32_t* demand = (ro && ro->demand) ? ro->demand : at<int32_t>(ws, L.demand);
  uint8_t* drop = (ro && ro->drop_mask) ? ro->drop_mask : at<uint8_t>(ws, L.drop_mask);
  int32_t* offsets_pad = (ro && ro->offsets) ? ro->offsets : at<int32_t>(ws, L.offsets_pad);
  int32_t* slot_row = at<int32_t>(ws, L.slot_row);
  int32_t* row_token = at<int32_t>(ws, L.row_token);
  void* xp = at<char>(ws, L.xp);
  void* ye = at<char>(ws, L.ye);
  int launches = 0;
  LogitSrc zsrc;
  MOE_TRY(stage_logits(c, L, ws, x, W_g, logit_offset, logits, status, st, &launches, &zsrc));
  MOE_TRY(stage_route(c, zsrc, bias, modality, ids, gates, status, st, &launches));
  MOE_CUDA(moe::launch_rank_local(ids, nullptr, c.N, c.k, c.E, at<int32_t>(ws, L.local_rank),
                                  at<int32_t>(ws, L.tile_hist), status, st, &launches),
           "rank pass");
  MOE_CUDA(moe::launch_dispatch_scan(at<int32_t>(ws, L.tile_hist), c.N, c.E, c.capacity,
                                     at<int32_t>(ws, L.tile_base), demand, counts,
                                     at<int32_t>(ws, L.offsets), arrive_counter(ws, L), st,
                                     &launches),
           "scan pass");
  MOE_CUDA(moe::launch_pad_offsets(c.E, c.capacity, offsets_pad, st, &launches), "pad offsets");
  MOE_CUDA(moe::launch_dispatch_scatter(ids, at<int32_t>(ws, L.local_rank),
                                        at<int32_t>(ws, L.tile_base), offsets_pad, c.N, c.k, c.E,
                                        c.capacity, slot_row, row_token, drop, x, xp,
                                        (int)(c.d * el_size(c)), st, &launches),
           "scatter pass");
  MOE_CUDA(moe::launch_zero_padding(counts, c.E, c.capacity, xp, (int)(c.d * el_size(c)),
                                    row_token, st, &launches),
           "zero padding");
  MOE_TRY(stage_ffn(c, L, ws, xp, offsets_pad, x, W_gu, W_down, ye, st, &launches, R, y,
                    c.capacity));
  MOE_TRY(stage_combine(c, ye, slot_row, gates, y, st, &launches, R, true));
  g_last_launches = launches;
  return MOE_OK;
}

// ---- expert parallelism ("Le problème — Communication", "L'idée — Communication") ----------
size_t moe_ep_workspace_size(const moe_config* cfg, int32_t world) {
  if (world < 1 || check_cfg(cfg) != MOE_OK || world > cfg->E) return 0;
  const moe_config w = ep_ws_config(*cfg, world);
  if (check_cfg(&w) != MOE_OK) return 0;
  return layout(w).total;
}

moe_status moe_permute_ep(const moe_config* cfg, const int32_t* ids, const int32_t* cap,
                          const void* x, int32_t* offsets, int32_t* row_token, int32_t* slot_row,
                          void* xp, int32_t* counts, uint8_t* drop_mask, void* ws,
                          moe_stream_t stream) {
  NvtxRange nvtx_range("moe_permute_ep");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (ids == nullptr || cap == nullptr || offsets == nullptr || slot_row == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "ids, cap, offsets and slot_row are required");
  MOE_TRY(need(x, "x"));
  MOE_TRY(need(xp, "xp"));
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  int launches = 0;
  MOE_TRY(stage_dispatch(c, L, ws, ids, nullptr, 0, at<int32_t>(ws, L.demand),
                         counts != nullptr ? counts : at<int32_t>(ws, L.counts), offsets,
                         slot_row, row_token,
                         drop_mask != nullptr ? drop_mask : at<uint8_t>(ws, L.drop_mask), x, xp,
                         (cudaStream_t)stream, &launches, cap));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_permute_ep_p2p(const moe_config* cfg, const int32_t* ids, const int32_t* cap,
                              const void* x, int32_t* offsets, int32_t* slot_row,
                              const uint64_t* dst_base, const int32_t* dst_row0,
                              const int64_t* dst_rows, int32_t* counts, uint8_t* drop_mask,
                              void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_permute_ep_p2p");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (ids == nullptr || cap == nullptr || offsets == nullptr || slot_row == nullptr ||
      dst_base == nullptr || dst_row0 == nullptr || dst_rows == nullptr)
    return fail(MOE_ERR_INVALID_ARG,
                "ids, cap, offsets, slot_row, dst_base, dst_row0 and dst_rows are required");
  MOE_TRY(need(x, "x"));
  const moe_config& c = *cfg;
  if (c.dtype != MOE_DT_BF16 || (c.d * el_size(c)) % 16 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_permute_ep_p2p: bf16 rows of a multiple of 16 bytes");
  const Ws L = layout(c);
  const moe::RemoteRows rem{(const unsigned long long*)dst_base, dst_row0, dst_rows,
                            at<int>(ws, L.status)};
  int launches = 0;
  MOE_TRY(stage_dispatch(c, L, ws, ids, nullptr, 0, at<int32_t>(ws, L.demand),
                         counts != nullptr ? counts : at<int32_t>(ws, L.counts), offsets,
                         slot_row, nullptr,
                         drop_mask != nullptr ? drop_mask : at<uint8_t>(ws, L.drop_mask), x,
                         nullptr, (cudaStream_t)stream, &launches, cap, false, &rem));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_ep_expert_ffn(const moe_config* cfg, int32_t world, int32_t rank,
                             int64_t n_tokens, int64_t rows, const void* xr,
                             const int32_t* offsets, const void* x, const void* W_gu,
                             const void* W_down, void* ye, void* y, void* ws,
                             moe_stream_t stream) {
  NvtxRange nvtx_range("moe_ep_expert_ffn");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (world < 1 || rank < 0 || rank >= world)
    return fail(MOE_ERR_INVALID_ARG, "rank must be in [0, world)");
  if (world > cfg->E) return fail(MOE_ERR_UNSUPPORTED, "more ranks than experts");
  if (cfg->dtype != MOE_DT_BF16)
    return fail(MOE_ERR_UNSUPPORTED, "the expert-parallel FFN is bf16 only");
  if (n_tokens < 0 || n_tokens > cfg->N)
    return fail(MOE_ERR_INVALID_ARG, "n_tokens must be in [0, cfg->N]");
  if (rows < 0 || rows > cfg->N * (int64_t)world * cfg->k)
    return fail(MOE_ERR_INVALID_ARG, "rows must be in [0, world * N * k]");
  if (offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "offsets is NULL");
  if (rows > 0) {
    MOE_TRY(need(xr, "xr"));
    MOE_TRY(need(ye, "ye"));
  }
  if (cfg->n_shared && n_tokens > 0) {
    MOE_TRY(need(x, "x"));
    MOE_TRY(need(y, "y"));
  }
  MOE_TRY(need(W_gu, "W_gu"));
  MOE_TRY(need(W_down, "W_down"));
  const int32_t e0 = moe_ep_first_expert(world, rank, cfg->E);
  const int32_t e1 = moe_ep_first_expert(world, rank + 1, cfg->E);
  moe_config c = *cfg;  // the owned experts as the layer's routed experts, this call's tokens
  c.E = e1 - e0;
  c.N = n_tokens;
  c.capacity = 0;
  if (c.N == 0) {
    // no tokens of its own (no shared rows), but the owner may still have received rows;
    // N only sizes the shared group and the rows-per-expert estimate of the kernel choice
    c.n_shared = 0;
    c.N = std::max<int64_t>(1, (rows + c.k - 1) / c.k);
  }
  const Ws L = layout(ep_ws_config(*cfg, world));
  int launches = 0;
  if (rows == 0 && c.n_shared == 0) return MOE_OK;
  // routed groups: the received rows [offsets[i], offsets[i+1]) of owned expert e0 + i; the
  // shared expert runs on this rank's own tokens and writes its rows into y
  MOE_TRY(stage_ffn(c, L, ws, rows > 0 ? xr : x, offsets, x, W_gu, W_down, rows > 0 ? ye : y,
                    (cudaStream_t)stream, &launches, rows, c.n_shared ? y : nullptr));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_ep_combine(const moe_config* cfg, const void* ye, const int32_t* slot_row,
                          const float* gates, void* y, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_ep_combine");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  if (cfg->dtype != MOE_DT_BF16) return fail(MOE_ERR_UNSUPPORTED, "the expert-parallel combine is bf16 only");
  MOE_TRY(need(ye, "ye"));
  MOE_TRY(need(y, "y"));
  if (slot_row == nullptr || gates == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "slot_row and gates are required");
  int launches = 0;
  MOE_TRY(stage_combine(*cfg, ye, slot_row, gates, y, (cudaStream_t)stream, &launches, -1,
                        cfg->n_shared != 0));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_ep_combine_p2p(const moe_config* cfg, const int32_t* ids,
                              const int32_t* slot_row, const float* gates,
                              const int32_t* offsets, const uint64_t* src_base,
                              const int32_t* src_row0, const int64_t* src_rows, void* y,
                              void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_ep_combine_p2p");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (ids == nullptr || slot_row == nullptr || gates == nullptr || offsets == nullptr ||
      src_base == nullptr || src_row0 == nullptr || src_rows == nullptr)
    return fail(MOE_ERR_INVALID_ARG,
                "ids, slot_row, gates, offsets, src_base, src_row0 and src_rows are required");
  MOE_TRY(need(y, "y"));
  const moe_config& c = *cfg;
  if (c.dtype != MOE_DT_BF16 || (c.d * el_size(c)) % 16 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_ep_combine_p2p: bf16 rows of a multiple of 16 bytes");
  const Ws L = layout(c);
  const moe::RemoteSrc rem{(const unsigned long long*)src_base, src_row0, src_rows, offsets, ids,
                           c.E, at<int>(ws, L.status)};
  int launches = 0;
  MOE_TRY(stage_combine(c, nullptr, slot_row, gates, y, (cudaStream_t)stream, &launches, -1,
                        c.n_shared != 0, &rem));
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_ep_copy_runs(const void* src, int64_t src_rows, const uint64_t* dst_base,
                            const int64_t* dst_rows, int32_t n_bufs, const int32_t* runs,
                            const int32_t* run_start, int32_t n_runs, int64_t total_rows,
                            int64_t row_bytes, void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_ep_copy_runs");
  g_last_launches = 0;
  if (src_rows < 0 || n_bufs < 0 || n_runs < 0 || total_rows < 0 || row_bytes <= 0 ||
      row_bytes % 16 != 0 || row_bytes > (int64_t)INT32_MAX)
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_copy_runs: bad sizes (row_bytes a multiple of 16)");
  if (n_runs == 0 || total_rows == 0) return MOE_OK;
  if (src == nullptr || dst_base == nullptr || dst_rows == nullptr || runs == nullptr ||
      run_start == nullptr || n_bufs == 0)
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_copy_runs: null pointer");
  if ((reinterpret_cast<uintptr_t>(src) & 15) != 0)
    return fail(MOE_ERR_INVALID_ARG, "moe_ep_copy_runs: src not 16-byte aligned");
  int launches = 0;
  MOE_CUDA(moe::launch_copy_runs(src, src_rows, (const unsigned long long*)dst_base, dst_rows,
                                 n_bufs, runs, run_start, n_runs, total_rows, (int)row_bytes,
                                 ws != nullptr ? (int*)ws : nullptr, (cudaStream_t)stream,
                                 &launches),
           "copy runs");
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_ipc_handle(const void* ptr, void* handle, int64_t* offset) {
  if (ptr == nullptr || handle == nullptr || offset == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_ipc_handle: null pointer");
  void* base = nullptr;
  MOE_CUDA(moe::allocation_base(ptr, &base), "moe_ipc_handle: allocation of the pointer");
  cudaIpcMemHandle_t h;
  MOE_CUDA(cudaIpcGetMemHandle(&h, base), "cudaIpcGetMemHandle");
  static_assert(sizeof(h) == 64, "CUDA IPC handles are 64 bytes");
  std::memcpy(handle, &h, sizeof(h));
  *offset = (int64_t)((const char*)ptr - (const char*)base);
  return MOE_OK;
}

moe_status moe_ipc_open(const void* handle, void** base) {
  if (handle == nullptr || base == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_ipc_open: null pointer");
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  MOE_CUDA(cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess), "cudaIpcOpenMemHandle");
  return MOE_OK;
}

moe_status moe_ipc_close(void* base) {
  if (base == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_ipc_close: null pointer");
  MOE_CUDA(cudaIpcCloseMemHandle(base), "cudaIpcCloseMemHandle");
  return MOE_OK;
}

moe_status moe_forward_host(const moe_config* cfg, const void* x_host, const void* W_g,
                            const float* logit_offset, const float* bias,
                            const uint8_t* modality, const void* W_gu, const void* W_down,
                            void* y_host, void* ws, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_forward_host");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  MOE_TRY(check_bias(cfg, bias, modality));
  if (x_host == nullptr || y_host == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "x_host and y_host are required");
  MOE_TRY(need(W_g, "W_g"));
  MOE_TRY(need(W_gu, "W_gu"));
  MOE_TRY(need(W_down, "W_down"));
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t bytes = (size_t)c.N * c.d * el_size(c);
  void* xd = at<char>(ws, L.x_stage);
  void* yd = at<char>(ws, L.y_stage);
  int launches = 0;
  if (bytes > 0) MOE_CUDA(cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, st), "copy x to device");
  const moe_status fs = forward_impl(cfg, xd, W_g, logit_offset, bias, modality, W_gu, W_down,
                                     yd, nullptr, ws, st, &launches);
  g_prof.recording = false;
  MOE_TRY(fs);
  if (bytes > 0) MOE_CUDA(cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, st), "copy y to host");
  MOE_CUDA(cudaStreamSynchronize(st), "synchronise");
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_forward_host_batches(const moe_config* cfg, int32_t n_batches,
                                    const void* const* x_host, const void* W_g,
                                    const float* logit_offset, const float* bias,
                                    const uint8_t* const* modality, const void* W_gu,
                                    const void* W_down, void* const* y_host, void* ws,
                                    moe_stream_t stream) {
  NvtxRange nvtx_range("moe_forward_host_batches");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws));
  if (n_batches < 0) return fail(MOE_ERR_INVALID_ARG, "n_batches < 0");
  if (n_batches > 0 && (x_host == nullptr || y_host == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "x_host and y_host arrays are required");
  for (int b = 0; b < n_batches; ++b) {
    if (x_host[b] == nullptr || y_host[b] == nullptr)
      return fail(MOE_ERR_INVALID_ARG, "a host batch pointer is NULL");
    MOE_TRY(check_bias(cfg, bias, modality != nullptr ? modality[b] : nullptr));
  }
  if (n_batches == 0) return MOE_OK;
  MOE_TRY(need(W_g, "W_g"));
  MOE_TRY(need(W_gu, "W_gu"));
  MOE_TRY(need(W_down, "W_down"));
  const moe_config& c = *cfg;
  const Ws L = layout(c);
  const size_t bytes = (size_t)c.N * c.d * el_size(c);
  cudaStream_t main = (cudaStream_t)stream;
  // two copy streams and the events that chain them to the layer (created once per thread)
  thread_local cudaStream_t copy_in = nullptr, copy_out = nullptr;
  thread_local cudaEvent_t ev_in[2], ev_done[2], ev_out[2];
  thread_local int owner_dev = -1;
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (copy_in == nullptr || owner_dev != dev) {
    MOE_CUDA(cudaStreamCreateWithFlags(&copy_in, cudaStreamNonBlocking), "create copy stream");
    MOE_CUDA(cudaStreamCreateWithFlags(&copy_out, cudaStreamNonBlocking), "create copy stream");
    for (int i = 0; i < 2; ++i) {
      MOE_CUDA(cudaEventCreateWithFlags(&ev_in[i], cudaEventDisableTiming), "create event");
      MOE_CUDA(cudaEventCreateWithFlags(&ev_done[i], cudaEventDisableTiming), "create event");
      MOE_CUDA(cudaEventCreateWithFlags(&ev_out[i], cudaEventDisableTiming), "create event");
    }
    owner_dev = dev;
  }
  void* xd[2] = {at<char>(ws, L.x_stage), at<char>(ws, L.x_stage2)};
  void* yd[2] = {at<char>(ws, L.y_stage), at<char>(ws, L.y_stage2)};
  int launches = 0;
  for (int b = 0; b < n_batches; ++b) {
    const int s = b & 1;
    // x slot s is free once batch b-2's layer is done; y slot s once its copy-out is done
    if (b >= 2) MOE_CUDA(cudaStreamWaitEvent(copy_in, ev_done[s], 0), "wait");
    MOE_CUDA(cudaMemcpyAsync(xd[s], x_host[b], bytes, cudaMemcpyHostToDevice, copy_in), "copy x to device");
    MOE_CUDA(cudaEventRecord(ev_in[s], copy_in), "record");
    MOE_CUDA(cudaStreamWaitEvent(main, ev_in[s], 0), "wait");
    if (b >= 2) MOE_CUDA(cudaStreamWaitEvent(main, ev_out[s], 0), "wait");
    const moe_status fs = forward_impl(cfg, xd[s], W_g, logit_offset, bias,
                                       modality != nullptr ? modality[b] : nullptr, W_gu, W_down,
                                       yd[s], nullptr, ws, main, &launches);
    g_prof.recording = false;
    MOE_TRY(fs);
    MOE_CUDA(cudaEventRecord(ev_done[s], main), "record");
    MOE_CUDA(cudaStreamWaitEvent(copy_out, ev_done[s], 0), "wait");
    MOE_CUDA(cudaMemcpyAsync(y_host[b], yd[s], bytes, cudaMemcpyDeviceToHost, copy_out), "copy y to host");
    MOE_CUDA(cudaEventRecord(ev_out[s], copy_out), "record");
  }
  MOE_CUDA(cudaStreamSynchronize(copy_out), "synchronise");
  MOE_CUDA(cudaStreamSynchronize(main), "synchronise");
  g_last_launches = launches;
  return MOE_OK;
}

}  // extern "C"

// ---- moe_route_static: routing with its scratch in a fixed device array ---------------
namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB
// Scratch of moe_route_static.  In host code this name is only a host-side stand-in: the
// kernels get the device address looked up below.
__device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};  // the context the address was looked up in

// The current driver context (cuCtxGetCurrent through the runtime's entry-point lookup, so
// the library does not link libcuda); nullptr if it cannot be read.
void* current_context() {
  using Fn = int (*)(void**);
  static Fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(p);
  });
  void* ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of g_route_scratch on the current device: looked up once per device and
// context (a device reset or another context on the device loads the module anew, at a new
// address, so the lookup is repeated then).
moe_status static_scratch(void** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device ordinal >= 64");
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr || ctx == nullptr || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    MOE_CUDA(cudaGetSymbolAddress(&p, g_route_scratch), "cudaGetSymbolAddress(route scratch)");
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context();
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_route_static(const moe_config* cfg, const float* logits, const float* bias,
                            const uint8_t* modality, int32_t* ids, float* gates,
                            int32_t* counts, int32_t* demand, uint8_t* drop_mask,
                            int32_t* status, moe_stream_t stream) {
  NvtxRange nvtx_range("moe_route_static");
  g_last_launches = 0;
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_bias(cfg, bias, modality));
  if (logits == nullptr || ids == nullptr || gates == nullptr || counts == nullptr ||
      demand == nullptr || drop_mask == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "logits, ids, gates, counts, demand and drop_mask are required");
  const moe_config& c = *cfg;
  const size_t Nk = (size_t)c.N * c.k;
  const size_t tiles = ((size_t)c.N + moe::kRankTile - 1) / moe::kRankTile;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  // o_arrive: the scan's ticket counter, set to zero by every call before its scan (so an
  // earlier overlapping call that raced on it cannot leave it wrong for later ones)
  const size_t o_arrive = take(256);
  const size_t o_rank = take(Nk * 4), o_hist = take(tiles * c.E * 4),
               o_base = take(tiles * c.E * 4), o_offs = take(((size_t)c.E + 1) * 4);
  if (off > kStaticScratchBytes) {
    char buf[160];
    snprintf(buf, sizeof(buf), "moe_route_static needs %zu bytes of scratch; its static array holds %zu",
             off, kStaticScratchBytes);
    return fail(MOE_ERR_UNSUPPORTED, buf);
  }
  void* scratch = nullptr;
  MOE_TRY(static_scratch(&scratch));
  cudaStream_t st = (cudaStream_t)stream;
  int launches = 0;
  MOE_CUDA(cudaMemsetAsync(at<int32_t>(scratch, o_arrive), 0, sizeof(int32_t), st),
           "clear the scan ticket");
  MOE_TRY(stage_route(c, finished_logits(logits), bias, modality, ids, gates, status, st,
                      &launches));
  MOE_CUDA(moe::launch_rank_local(ids, nullptr, c.N, c.k, c.E, at<int32_t>(scratch, o_rank),
                                  at<int32_t>(scratch, o_hist), status, st, &launches),
           "rank pass");
  MOE_CUDA(moe::launch_dispatch_scan(at<int32_t>(scratch, o_hist), c.N, c.E, c.capacity,
                                     at<int32_t>(scratch, o_base), demand, counts,
                                     at<int32_t>(scratch, o_offs),
                                     at<int32_t>(scratch, o_arrive), st, &launches),
           "scan pass");
  MOE_CUDA(moe::launch_dispatch_scatter(ids, at<int32_t>(scratch, o_rank),
                                        at<int32_t>(scratch, o_base),
                                        at<int32_t>(scratch, o_offs), c.N, c.k, c.E,
                                        c.capacity, nullptr, nullptr, drop_mask, nullptr,
                                        nullptr, 0, st, &launches),
           "scatter pass");
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(void* ws, int64_t limit_ns, moe_stream_t stream) {
  g_last_launches = 0;
  if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if (limit_ns < 0 || limit_ns > 1000000000) return fail(MOE_ERR_INVALID_ARG, "limit_ns outside 0 .. 1e9");
  int launches = 0;
  MOE_CUDA(moe::launch_wait_selftest(static_cast<int*>(ws), (uint64_t)limit_ns, nullptr,
                                     (cudaStream_t)stream, &launches),
           "wait self-test");
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_check_status(void* ws, moe_stream_t stream) {
  if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st = (cudaStream_t)stream;
  MOE_CUDA(cudaStreamSynchronize(st), "asynchronous error");
  int host = 0;
  MOE_CUDA(cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, st), "read status");
  MOE_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), st), "clear status");
  MOE_CUDA(cudaStreamSynchronize(st), "read status");
  if (host == MOE_ERR_INVALID_INPUT)
    return fail(MOE_ERR_INVALID_INPUT, "device found an invalid expert id or modality flag");
  if (host == MOE_ERR_TIMEOUT) return fail(MOE_ERR_TIMEOUT, "a bounded device wait ran out");
  if (host != 0) return fail(MOE_ERR_CUDA, "unknown device status");
  return MOE_OK;
}

moe_status moe_check_dispatch(const moe_config* cfg, const int32_t* ids,
                              const uint8_t* drop_mask, const int32_t* counts,
                              const int32_t* demand, const int32_t* offsets,
                              const int32_t* slot_row, const int32_t* row_token,
                              moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  if (ids == nullptr || drop_mask == nullptr || counts == nullptr || offsets == nullptr ||
      slot_row == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "ids, drop_mask, counts, offsets and slot_row are required");
  return check_dispatch_device(*cfg, ids, drop_mask, counts, demand, offsets, slot_row,
                               row_token, cfg->capacity, (cudaStream_t)stream);
}

moe_status moe_profile_begin(int32_t max_calls) {
  if (max_calls < 0) return fail(MOE_ERR_INVALID_ARG, "max_calls < 0");
  for (auto& v : g_prof.ev)
    for (auto e : v) cudaEventDestroy(e);
  g_prof = Profile();
  g_prof.max_calls = max_calls;
  return MOE_OK;
}

int32_t moe_profile_end(float* launch_ms, int32_t max_launches, int32_t* calls) {
  int32_t per_call = 0;
  bool ok = true;
  if (launch_ms != nullptr)
    for (int i = 0; i < max_launches; ++i) launch_ms[i] = 0.f;
  for (auto& v : g_prof.ev) {
    if (v.empty()) continue;
    if (cudaEventSynchronize(v.back()) != cudaSuccess) ok = false;
    per_call = std::max<int32_t>(per_call, (int32_t)v.size() - 1);
    for (size_t i = 0; ok && i + 1 < v.size(); ++i) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, v[i], v[i + 1]) != cudaSuccess) ok = false;
      if (launch_ms != nullptr && (int)i < max_launches) launch_ms[i] += ms;
    }
  }
  if (calls != nullptr) *calls = (int32_t)g_prof.ev.size();
  for (auto& v : g_prof.ev)
    for (auto e : v) cudaEventDestroy(e);
  g_prof = Profile();
  if (!ok) {
    g_last_error = "moe_profile_end: event timing failed";
    return -1;
  }
  return per_call;
}

const char* moe_last_error(void) { return g_last_error.c_str(); }

int32_t moe_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
