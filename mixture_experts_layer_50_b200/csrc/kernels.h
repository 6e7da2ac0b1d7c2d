// Internal launchers of the MoE layer kernels.  Each returns the cudaError_t of its
// launch(es) and adds the number of kernels it enqueued to *launches.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// ---- routing (route.cu) ---------------------------------------------------------------
// Scores, selection keys, top-k (descending, ties to the lower index) and gates.
// logits = sum over n_parts slices (part_stride elements apart) plus offset (when not null);
// with n_parts > 1 or an offset the summed logits are written to logits_out (when not null).
cudaError_t launch_route_topk(const float* logits, int n_parts, int64_t part_stride,
                              const float* offset, float* logits_out, int64_t N, int E, int k,
                              int score_fn, int renorm, const float* bias, int n_bias_sets,
                              const uint8_t* modality, int32_t* ids, float* gates,
                              int* status, cudaStream_t stream, int* launches,
                              int k_extra = 0, int32_t* cand = nullptr,
                              float* cand_val = nullptr);
// Top-k and the dispatch's rank pass in one launch (kRankTile tokens per block): ids, gates,
// and the local ranks and tile histograms launch_rank_local would write (no drop mask).
// Opt-in: MOE_B200_FUSED_TOPK_RANK=1.
constexpr int kFusedTopkRankMaxE = 384;
bool fused_topk_rank_enabled();
cudaError_t launch_route_topk_rank(const float* logits, int n_parts, int64_t part_stride,
                                   const float* offset, float* logits_out, int64_t N, int E,
                                   int k, int score_fn, int renorm, const float* bias,
                                   int n_bias_sets, const uint8_t* modality, int32_t* ids,
                                   float* gates, int* status, int32_t* local_rank,
                                   int32_t* tile_hist, cudaStream_t stream, int* launches);
// Overflow policy "report": offers of the dropped slots to the next-best candidates, and the
// decision on them (csrc/reroute.cu).
cudaError_t launch_reroute_offer(const int32_t* ids, const uint8_t* drop1, const int32_t* cand,
                                 int64_t N, int k, int32_t* offer, uint8_t* not_offer,
                                 cudaStream_t stream, int* launches);
cudaError_t launch_reroute_accept(int32_t* ids, const uint8_t* drop1, const int32_t* offer,
                                  const uint8_t* not_offer, const int32_t* local_rank,
                                  const int32_t* tile_base, const int32_t* counts1,
                                  const float* cand_val, int64_t N, int E, int k, int64_t C,
                                  int score_fn, int renorm, float* gates, uint8_t* drop_out,
                                  uint8_t* rerouted, cudaStream_t stream, int* launches);

// Hash router: ids = the k experts with the largest fmix32(token_id * 0x9E3779B1 + e), gates 1/k.
cudaError_t launch_route_hash(const int32_t* token_ids, int64_t N, int E, int k, int32_t* ids,
                              float* gates, cudaStream_t stream, int* launches);

// ---- dispatch (dispatch.cu) -----------------------------------------------------------
// Pass 1: per token tile, ranks of each assignment among the tile's earlier tokens that
// chose the same expert, and the tile's per-expert histogram.  Assignments whose
// drop_mask entry is set (when drop_mask != nullptr), or whose id is invalid, get rank -1.
cudaError_t launch_rank_local(const int32_t* ids, const uint8_t* drop_mask, int64_t N, int k,
                              int E, int32_t* local_rank, int32_t* tile_hist, int* status,
                              cudaStream_t stream, int* launches);
// Pass 2: scan over tiles and experts: tile_base, demand, counts (capped at C when C > 0,
// or at cap_e[e] per expert when cap_e is not null) and offsets (exclusive scan of counts,
// E + 1 entries).
cudaError_t launch_dispatch_scan(const int32_t* tile_hist, int64_t N, int E, int64_t C,
                                 int32_t* tile_base, int32_t* demand, int32_t* counts,
                                 int32_t* offsets, int32_t* arrive, cudaStream_t stream,
                                 int* launches, const int32_t* cap_e = nullptr);
// Per-expert destinations of the gathered rows (expert parallelism over peer memory): the
// kept rows of expert e go to rows row0[e], row0[e] + 1, ... (in their layout order) of the
// buffer at base[e] -- another device's receive buffer, or a local one.  Device arrays [E].
struct RemoteRows {
  const unsigned long long* base;
  const int32_t* row0;
  const int64_t* rows;   // [E]: rows of the buffer at base[e]; a row past it is skipped
  int* status;           // where a skipped row is reported (invalid input), or null
};

// Pass 3: capacity decision (rank < C, or rank < cap_e[e] when cap_e is not null), slot
// rows (when slot_row is not null), row -> token map, drop mask, and (when xp is not null)
// the gather of x rows into the per-expert layout -- or, with rem, into each expert's
// destination instead (row_bytes % 16 == 0).
cudaError_t launch_dispatch_scatter(const int32_t* ids, const int32_t* local_rank,
                                    const int32_t* tile_base, const int32_t* offsets,
                                    int64_t N, int k, int E, int64_t C, int32_t* slot_row,
                                    int32_t* row_token, uint8_t* drop_mask_out,
                                    const void* x, void* xp, int row_bytes,
                                    cudaStream_t stream, int* launches,
                                    const int32_t* cap_e = nullptr,
                                    const RemoteRows* rem = nullptr);

// The three passes in one launch for a small batch (N <= kSmallDispatchMaxTokens and
// N * k <= kSmallDispatchMaxSlots): the same outputs, plus the device status for bad ids.
constexpr int kSmallDispatchThreads = 1024;   // >= E (at most 1024)
constexpr int kSmallDispatchMaxTokens = 64;
constexpr int kSmallDispatchMaxSlots = 1024;
bool use_small_dispatch(int64_t N, int k, int E);   // MOE_B200_SMALL_DISPATCH=0: never
cudaError_t launch_dispatch_small(const int32_t* ids, const uint8_t* drop_in, int64_t N, int k,
                                  int E, int64_t C, const int32_t* cap_e, int32_t* demand,
                                  int32_t* counts, int32_t* offsets, int32_t* slot_row,
                                  int32_t* row_token, uint8_t* drop_mask_out, const void* x,
                                  void* xp, int row_bytes, int* status, cudaStream_t stream,
                                  int* launches, const RemoteRows* rem = nullptr);

// ---- expert-parallel rows over peer memory (ep_p2p.cu) ---------------------------------
// Copy row runs (runs [n_runs][4] int32: src_row, dst_buf, dst_row, rows; run_start
// [n_runs + 1] the prefix of their rows) from src [src_rows][row_bytes] to the buffers
// dst_base[dst_buf] ([dst_rows[dst_buf]][row_bytes]); out-of-range runs are skipped and
// reported (status, when not null).  row_bytes % 16 == 0, buffers 16-byte aligned.
cudaError_t launch_copy_runs(const void* src, int64_t src_rows, const unsigned long long* dst_base,
                             const int64_t* dst_rows, int n_bufs, const int32_t* runs,
                             const int32_t* run_start, int n_runs, int64_t total_rows,
                             int row_bytes, int* status, cudaStream_t stream, int* launches);
// Base of the device allocation containing ptr.
cudaError_t allocation_base(const void* ptr, void** base);

// ---- balancing statistics (balance.cu) ------------------------------------------------
// f [E] share of assignments, P [E] mean router probability, aux = E sum f P, set_load
// [n_sets][E] assignments per modality set; when bias != nullptr, bias += gamma * sign(mean
// load - load) per set.  n_sets <= 8.  Any output pointer may be null.
size_t balance_scratch_bytes(int64_t N, int E, int n_sets);
cudaError_t launch_balance(const float* logits, const int32_t* ids, const uint8_t* modality,
                           int64_t N, int E, int k, int score_fn, int n_sets, void* scratch,
                           float* f, float* P, float* aux, int32_t* set_load, float* bias,
                           float gamma, cudaStream_t stream, int* launches);

// Padded layout: offsets_pad[e] = e * C for e <= E.
cudaError_t launch_pad_offsets(int E, int64_t C, int32_t* offsets_pad, cudaStream_t stream,
                               int* launches);
// Zero the empty slots (rows e*C + c with c >= counts[e]) of a padded buffer and mark them
// -1 in row_token_pad (when not null).
cudaError_t launch_zero_padding(const int32_t* counts, int E, int64_t C, void* xp_pad,
                                int row_bytes, int32_t* row_token_pad, cudaStream_t stream,
                                int* launches);

// ---- combine (combine.cu) -------------------------------------------------------------
// y[t] = sum_j gates[t,j] ye[slot_row[t,j]] (+ ye[shared_row0 + t] when shared_row0 >= 0).
// shared_row0 >= 0: the shared row of token t is ye[shared_row0 + t]; shared_in_y (bf16):
// y[t] holds it already (written by the down GEMM) and is updated in place.
// rem (bf16 only): slot (t, j) kept for expert e = ids[t, j] at send-layout row r reads row
// row0[e] + (r - offsets[e]) of the buffer at base[e] (rows[e] rows; offsets [E + 1]) instead
// of ye[r]; a slot outside those bounds contributes nothing and is reported in status.
struct RemoteSrc {
  const unsigned long long* base;
  const int32_t* row0;
  const int64_t* rows;
  const int32_t* offsets;
  const int32_t* ids;
  int E;
  int* status;
};
cudaError_t launch_combine(const void* ye, const int32_t* slot_row, const float* gates,
                           int64_t N, int k, int d, int64_t shared_row0, int shared_in_y,
                           int is_f32, void* y, cudaStream_t stream, int* launches,
                           const RemoteSrc* rem = nullptr);

// ---- fp32 path (simt_f32.cu) ----------------------------------------------------------
cudaError_t launch_router_f32(const float* x, const float* W_g, const float* logit_offset,
                              int64_t N, int d, int E, float* logits, cudaStream_t stream,
                              int* launches);
// h[r] = act(A_r . W1_e) for every row r of the groups (routed rows from xp, shared rows
// from x, starting at row Nk), then ye[r] = h[r] . W2_e.
cudaError_t launch_ffn_f32(const float* xp, const float* x, const int32_t* offsets,
                           int64_t N, int64_t Nk, int d, int E, int F, int n_shared, int act,
                           float clamp, const float* W_gu, const float* W_down, float* h,
                           float* ye, cudaStream_t stream, int* launches);

// ---- tensor-core grouped GEMM (gemm_tc.cu) --------------------------------------------
enum GemmEpilogue : int { kEpiStoreBf16 = 0, kEpiSwiglu = 1, kEpiRelu = 2, kEpiStoreF32 = 3 };

struct GroupedGemm {
  // A: rows of activations, bf16 [rows_a][K]; routed group e reads rows
  // [offsets[e], offsets[e+1]).  a_shared: bf16 [rows_a_shared][K], read by the shared
  // group (rows [shared_a_row0, shared_a_row0 + shared_rows)).
  const void* a;
  int64_t rows_a;
  const void* a_shared;
  int64_t rows_a_shared;
  int64_t shared_a_row0;
  // B: weights bf16 [groups][rows_b][K]; routed group e uses slice e, the shared group
  // slice n_routed.
  const void* b;
  int groups_b;
  int rows_b;
  int K;
  const int32_t* offsets;  // [n_routed + 1] device, or null when n_routed == 0
  int n_routed;
  int has_shared;
  int64_t shared_rows;
  int64_t shared_out_row0;
  int n_out;               // output columns (SwiGLU: F, with up rows starting at row F)
  int epilogue;            // GemmEpilogue
  float clamp;
  const float* col_bias;   // [n_out] fp32 added before the store (fp32 store only)
  void* out;
  void* out_shared = nullptr;  // non-null: the shared group's row r is written to row r of
                               // out_shared (same ld_out), not to row shared_out_row0 + r of out
  int64_t ld_out;          // elements
  int64_t rows_out;
  int64_t max_rows_routed; // upper bound of offsets[n_routed] (grid sizing)
  int64_t rows_per_group_hint = -1;  // >= 0: the caller's estimate of a routed group's
                                     // rows (kernel choice); else max_rows_routed / n_routed
  int* status;
  int k_splits = 1;        // > 1 (fp32 store only): K split in slices, slice s written at
  int64_t split_rows = 0;  // out rows [s * split_rows, ...): partial sums, col_bias ignored
  int64_t max_group_rows = -1;  // > 0: no routed group has more rows (lets a batch whose
                                // groups all fit 64 rows use 64-row A stages)
};

cudaError_t launch_grouped_gemm(const GroupedGemm& g, cudaStream_t stream, int* launches,
                                const char** why);
namespace tc {
// SM count of the current device, cached per device (gemm_tc.cu).
int num_sms();
}  // namespace tc

// Name of the kernel launch_grouped_gemm launches for g (host only).
const char* grouped_gemm_kernel_name(const GroupedGemm& g);
// N width of the tiles of an fp32-store GEMM with n_out columns (the router).
int router_tile_n(int n_out);
// Failure-detection self-test: a bounded wait on a barrier nothing completes (gemm_tc.cu).
cudaError_t launch_wait_selftest(int* status, uint64_t limit_ns, int* out, cudaStream_t stream,
                                 int* launches);

}  // namespace moe
