/*
 * moe.h -- C ABI of the B200 (sm_100a) forward pass of a Mixture-of-Experts FFN layer.
 *
 * The layer (notation of "Основы MoE", section "Как устроен MoE-слой", steps 1-4, and of
 * the "Mixture-of-Experts : routage et capacité" slides):
 *
 *   z   = x . W_g                                  router projection, fp32 logits  [N][E]
 *   key = z + b            (softmax scoring)       selection keys; b is a per-expert,
 *       = sigma(z) + b     (sigmoid scoring)       selection-only bias, one set per modality
 *   T   = the k largest keys, descending, ties to the lower expert index
 *   g_i = softmax over the selected unbiased z     (softmax, renorm = 1)
 *       = p_i of the full softmax                  (softmax, renorm = 0: Switch k = 1)
 *       = s_i / sum_{j in T} s_j                   (sigmoid, renorm = 1)
 *   capacity C: the assignments to one expert are served in token order, the first C
 *       are kept, the others dropped (a dropped slot contributes 0; the kept gates are
 *       not renormalised)
 *   y_t = sum_{kept i in T} g_i FFN_i(x_t) + FFN_shared(x_t)
 *   FFN = (SiLU(x W_gate) * (x W_up)) W_down   with an optional clamp of both
 *         pre-activations to [-clamp, clamp] ("SwiGLU, écrêtée à 10"), or
 *         max(x W1, 0) W2 (the two-layer ReLU expert of the dataistudio listing).
 *
 * Conventions shared by every entry point:
 *  - All array pointers are caller-owned DEVICE memory unless a parameter says "host".
 *    The library never allocates device memory; scratch comes from the caller's workspace
 *    (moe_workspace_size bytes, 256-byte aligned, prepared once by moe_workspace_init).
 *  - Row-major everywhere.  Weights are stored out-major / K-contiguous (nn.Linear style):
 *      W_g    [E][d]                      (the math d x E matrix, transposed)
 *      W_gu   [E+S][2F][d]  SwiGLU        rows [0,F) = W_gate, rows [F,2F) = W_up
 *             [E+S][F][d]   ReLU          W1
 *      W_down [E+S][d][F]
 *    S = n_shared (0 or 1); the shared expert is stored last, at index E.
 *  - Element types: dtype MOE_DT_BF16 means x, weights, xp, ye and y are bf16 (fp32
 *    accumulation); MOE_DT_F32 means they are all fp32.  Logits, gates and biases are
 *    always fp32; ids, counts, offsets, rows are int32; masks and modality flags uint8.
 *  - Row layout of the per-expert buffers: routed rows of expert e occupy
 *    [offsets[e], offsets[e+1]) (offsets[E] = M, the kept assignments, M <= N*k); the
 *    shared expert's row for token t is N*k + t.  So xp has N*k rows, ye has N*k + S*N.
 *  - Every call is asynchronous and stream-ordered on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  No call synchronises the host, except
 *    moe_check_status and moe_forward_host.
 *  - Errors: host-side checks return a status before anything is enqueued.  Device-side
 *    findings (bad ids or modality flags, a bounded wait that ran out) are recorded in
 *    the workspace status word and reported by moe_check_status.  No device code traps.
 *  - Thread safety: calls on different workspaces may run concurrently; calls sharing a
 *    workspace must be ordered on one stream.  moe_last_error() is per thread.
 */
#ifndef MOE_B200_MOE_H_
#define MOE_B200_MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* a host-checked argument is wrong; nothing was enqueued */
  MOE_ERR_UNSUPPORTED = 2,   /* valid request outside what the library implements
                                (alignment, d or F not a multiple of 8, k > 32, ...) */
  MOE_ERR_CUDA = 3,          /* a CUDA call or launch failed; see moe_last_error() */
  MOE_ERR_INVALID_INPUT = 4, /* device-detected: expert id out of range or repeated in a
                                token, modality flag >= n_bias_sets */
  MOE_ERR_TIMEOUT = 5        /* device-detected: a bounded wait inside a kernel ran out */
} moe_status;

typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_fn;
typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_RELU = 1 } moe_act;
typedef enum { MOE_DT_BF16 = 0, MOE_DT_F32 = 1 } moe_dtype;

/* Shapes and options of one layer call. */
typedef struct {
  int64_t N;           /* tokens in this call (0 is allowed: every call is a no-op) */
  int32_t d;           /* model dimension */
  int32_t E;           /* routed experts, 1..1024 */
  int32_t k;           /* experts per token, 1..min(E, 32) */
  int32_t F;           /* hidden dimension of every expert (routed and shared) */
  int32_t n_shared;    /* always-on shared experts: 0 or 1 */
  int32_t n_bias_sets; /* 0: no selection bias; >= 1: bias is [n_bias_sets][E], token t
                          uses set modality[t] (set 0 when modality is NULL) */
  int32_t score_fn;    /* moe_score_fn */
  int32_t renorm;      /* 1: gates renormalised over the selected experts; 0: raw score */
  int32_t act;         /* moe_act */
  int32_t dtype;       /* moe_dtype */
  float clamp;         /* > 0: clamp gate and up pre-activations to [-clamp, clamp] */
  int64_t capacity;    /* C; <= 0 means unlimited */
} moe_config;

/* Optional routing outputs of moe_forward; every member may be NULL. */
typedef struct {
  float* logits;       /* [N][E]  fp32 router logits (z, plus logit_offset) */
  int32_t* ids;        /* [N][k]  selected experts, descending key */
  float* gates;        /* [N][k]  gate weights (dropped slots keep their gate value) */
  int32_t* counts;     /* [E]     kept assignments per expert */
  int32_t* demand;     /* [E]     assignments per expert before capacity */
  uint8_t* drop_mask;  /* [N][k]  1 = assignment dropped by capacity */
  int32_t* offsets;    /* [E+1]   exclusive scan of counts */
} moe_route_out;

/* Bytes of device workspace a call with this configuration needs (0 on a bad config).
 * The size depends on N, d, E, k, F, n_shared, n_bias_sets and dtype only. */
MOE_API size_t moe_workspace_size(const moe_config* cfg);

/* Zero the workspace header (the device status word and the dispatch scan's ticket
 * counter).  Call once after allocating; later calls leave the header's counter at zero. */
MOE_API moe_status moe_workspace_init(void* ws, moe_stream_t stream);

/* Capacity C = ceil(T * k / E * f) with f = cf_num / cf_den, in exact integer
 * arithmetic ("Mixture-of-Experts : routage et capacité", section "L'idée — Capacité").
 * cf_num <= 0 means no limit and returns 0.  Returns -1 on a bad argument.  Host only. */
MOE_API int64_t moe_capacity(int64_t T, int32_t k, int32_t E, int64_t cf_num, int64_t cf_den);

/* Router and capacity ("Основы MoE", steps 1-3; slides, "L'idée — Capacité").
 *   logits     [N][E] fp32 input, or NULL: then logits = x . W_g^T (+ logit_offset) are
 *              computed on the tensor cores (bf16) or in fp32 (MOE_DT_F32)
 *   x          [N][d], W_g [E][d]: read only when logits == NULL
 *   logit_offset [E] fp32 or NULL: added to computed logits (enters selection AND gates)
 *   bias       [n_bias_sets][E] fp32 or NULL (NULL iff n_bias_sets == 0)
 *   modality   [N] uint8 or NULL (required when n_bias_sets > 1)
 *   ids [N][k], gates [N][k], counts [E], demand [E], drop_mask [N][k]: outputs
 *   logits_out [N][E] or NULL: where computed logits are written (else workspace)
 * Ids, counts, demand and drop_mask are a deterministic function of the fp32 logits. */
MOE_API moe_status moe_route(const moe_config* cfg, const float* logits, const void* x,
                     const void* W_g, const float* logit_offset, const float* bias,
                     const uint8_t* modality, int32_t* ids, float* gates, int32_t* counts,
                     int32_t* demand, uint8_t* drop_mask, float* logits_out, void* ws,
                     moe_stream_t stream);

/* Permutation into per-expert contiguous groups (the per-expert gather of the
 * "Эксперимент на PyTorch" MoE.forward, laid out as the slides' dispatch table).
 *   ids [N][k] (values checked on the device), drop_mask [N][k] or NULL (none dropped)
 *   x [N][d] input rows
 *   offsets [E+1], row_token [N*k] (entries >= M are left untouched),
 *   slot_row [N][k] (-1 = dropped), xp [N*k][d]: outputs.
 * Within an expert, rows follow token order. */
MOE_API moe_status moe_permute(const moe_config* cfg, const int32_t* ids, const uint8_t* drop_mask,
                       const void* x, int32_t* offsets, int32_t* row_token,
                       int32_t* slot_row, void* xp, void* ws, moe_stream_t stream);

/* Expert FFNs over the groups: ye[r] = FFN_e(xp[r]) for r in [offsets[e], offsets[e+1]),
 * and ye[N*k + t] = FFN_shared(x[t]) when n_shared == 1.
 *   xp [N*k][d], offsets [E+1] (device), x [N][d] (read iff n_shared == 1)
 *   W_gu, W_down as above; ye [N*k + S*N][d] output.  Rows of ye outside the groups are
 *   left untouched.  bf16: tcgen05 grouped GEMMs, SwiGLU/ReLU fused in the epilogue,
 *   hidden activations rounded to bf16 in the workspace. */
MOE_API moe_status moe_expert_ffn(const moe_config* cfg, const void* xp, const int32_t* offsets,
                          const void* x, const void* W_gu, const void* W_down, void* ye,
                          void* ws, moe_stream_t stream);

/* Names of the kernels moe_expert_ffn (and every forward call) launches for the gate/up and
 * the down projections of cfg.  The choice is made on the host from the configuration alone
 * (N, k, E, d, F, act, dtype, n_shared, and the device's SM count and L2 size), so this call
 * answers without device memory: a bf16 layer takes the 1-SM grouped GEMM (128x256 or 128x128
 * tiles) or the 2-SM grouped GEMM (256x256 tiles on two SMs) per projection; an fp32 layer
 * the SIMT kernels.  Each non-NULL buffer receives at most len bytes, NUL included (the
 * name is truncated to fit).  MOE_ERR_INVALID_ARG for a bad cfg or len == 0 with a buffer;
 * MOE_ERR_UNSUPPORTED for a configuration the forward calls reject. */
MOE_API moe_status moe_ffn_kernels(const moe_config* cfg, char* gate_up, char* down, size_t len);

/* Gate-weighted combine back to token order ("Основы MoE", step 4):
 *   y[t] = sum_{j: slot_row[t][j] >= 0} gates[t][j] ye[slot_row[t][j]]  (+ ye[N*k + t])
 * summed in fp32 and rounded once.  y [N][d] output. */
MOE_API moe_status moe_combine(const moe_config* cfg, const void* ye, const int32_t* slot_row,
                       const float* gates, void* y, moe_stream_t stream);

/* The whole layer: route, capacity, permute, expert FFNs (routed + shared), combine.
 * Inputs as above; y [N][d] output; route_out may be NULL or have NULL members.  With a
 * shared expert (bf16) the down GEMM writes the shared expert's rows into y and the combine
 * adds the kept slots to them in place (y is written by two kernels of the call). */
MOE_API moe_status moe_forward(const moe_config* cfg, const void* x, const void* W_g,
                       const float* logit_offset, const float* bias,
                       const uint8_t* modality, const void* W_gu, const void* W_down,
                       void* y, const moe_route_out* route_out, void* ws,
                       moe_stream_t stream);

/* The layer with forced (replayed) routing: caller-supplied ids [N][k] and gates [N][k]
 * replace the router, the scores and the top-k; capacity, permutation, expert FFNs, the
 * shared expert and the combine run as in moe_forward ("Le groupe d'experts (MoE)",
 * exercise "Hard": record the experts that fired, force the same routing later).  ids are
 * checked on the device: an id outside [0, E) or repeated within a token is dropped and
 * reported as MOE_ERR_INVALID_INPUT by moe_check_status.  route_out may carry counts,
 * demand, drop_mask and offsets outputs (its logits, ids and gates members are ignored). */
MOE_API moe_status moe_forward_routed(const moe_config* cfg, const void* x, const int32_t* ids,
                                      const float* gates, const void* W_gu, const void* W_down,
                                      void* y, const moe_route_out* route_out, void* ws,
                                      moe_stream_t stream);

/* Overflow policy "report" ("Mixture-of-Experts : routage et capacité" slides, table
 * "Politiques de débordement quand E1 reçoit 6 tokens pour C = 5", row "Report sur E2/E3": the
 * rejected token is handled by its third-best score).  Routing and capacity as in moe_route,
 * then a token's i-th dropped slot (slot order, i = 0, 1, ...) is offered the token's
 * (k+i)-th best expert by selection key; the offers to one expert are served in token order,
 * then slot order, while its kept count plus the offers it took stays below C; a slot whose
 * offer finds no room stays dropped and keeps its expert id.  Gates are recomputed over each
 * token's final slot list as in moe_route (a moved slot takes its new expert's unbiased
 * score; a slot still dropped stays in the list and contributes 0).  With capacity <= 0
 * nothing overflows and the result is moe_route's.
 * Outputs: ids [N][k] (final experts), gates [N][k], counts [E] (kept assignments after the
 * policy), demand [E] (the router's assignments per expert before capacity), drop_mask
 * [N][k] (slots still dropped), rerouted [N][k] uint8 or NULL (1 = slot moved).  Requires
 * k <= 16 (MOE_ERR_UNSUPPORTED otherwise).  Other arguments as in moe_route. */
MOE_API moe_status moe_route_reroute(const moe_config* cfg, const float* logits, const void* x,
                                     const void* W_g, const float* logit_offset,
                                     const float* bias, const uint8_t* modality, int32_t* ids,
                                     float* gates, int32_t* counts, int32_t* demand,
                                     uint8_t* drop_mask, uint8_t* rerouted, float* logits_out,
                                     void* ws, moe_stream_t stream);

/* moe_forward with the "report" overflow policy of moe_route_reroute: the kept and moved
 * slots are permuted, run through their experts and combined as in moe_forward.  route_out
 * members as in moe_forward (counts after the policy, demand before capacity, drop_mask =
 * slots still dropped); rerouted [N][k] uint8 or NULL.  Requires k <= 16. */
MOE_API moe_status moe_forward_reroute(const moe_config* cfg, const void* x, const void* W_g,
                                       const float* logit_offset, const float* bias,
                                       const uint8_t* modality, const void* W_gu,
                                       const void* W_down, void* y,
                                       const moe_route_out* route_out, uint8_t* rerouted,
                                       void* ws, moe_stream_t stream);

/* Hash router ("Le groupe d'experts (MoE)", exercise "Medium": deterministic, not learned):
 * for token id t (token_ids [N], int32), expert e's key is fmix32(t * 0x9E3779B1 + e) with
 * 32-bit wrap-around, fmix32 being MurmurHash3's finaliser; the k largest keys are selected
 * (descending) and every gate is 1/k.  Then capacity and counts as in moe_route.
 * Outputs: ids [N][k], gates [N][k], counts [E], demand [E], drop_mask [N][k] (the last three
 * may be NULL).  cfg->score_fn, renorm and n_bias_sets are not used. */
MOE_API moe_status moe_route_hash(const moe_config* cfg, const int32_t* token_ids, int32_t* ids,
                                  float* gates, int32_t* counts, int32_t* demand,
                                  uint8_t* drop_mask, void* ws, moe_stream_t stream);

/* Load-balancing statistics of a routed batch and the aux-loss-free bias update.
 * ("Основы MoE", "Вспомогательный лосс Switch Transformer"; "Le groupe d'experts (MoE)",
 * load-balance section; DeepSeek-V4.1-Flash page, "L'équilibrage de charge" and
 * "l'équilibrage par modalité".)
 *   logits [N][E] fp32 and ids [N][k] of the batch (e.g. moe_forward's route_out)
 *   modality [N] uint8: the bias set of each token (required when n_bias_sets > 1)
 *   f [E]      share of the assignments per expert (sums to 1)
 *   P [E]      mean router probability per expert: softmax(z), or for sigmoid scoring the
 *              affinities sigma(z) normalised to sum 1 per token
 *   aux [1]    E * sum_i f_i P_i (1 when balanced, about E when collapsed; the Switch loss
 *              is alpha times this)
 *   set_load [max(1, n_bias_sets)][E] assignments per (bias set, expert)
 *   bias [n_sets][E] in/out or NULL: each entry moves by +gamma when its expert's load is
 *              below its set's mean load, -gamma when above, 0 when equal (the pages use
 *              gamma = 0.001)
 * Any of f, P, aux, set_load, bias may be NULL.  Deterministic (fixed summation order).
 * At most 8 bias sets. */
MOE_API moe_status moe_balance(const moe_config* cfg, const float* logits, const int32_t* ids,
                               const uint8_t* modality, float* f, float* P, float* aux,
                               int32_t* set_load, float* bias, float gamma, void* ws,
                               moe_stream_t stream);

/* The padded dispatch buffer [E][C][d] of "Mixture-of-Experts : routage et capacité"
 * ("Support visuel — Capacité": capacity as a tensor dimension): slot c of expert e holds the
 * c-th kept token of e in token order; empty slots are zero rows (row_token_pad = -1).  This is
 * the layout an expert-parallel all-to-all ships.  Needs cfg->capacity = C > 0.
 *   ids [N][k], drop_mask [N][k] or NULL (assignments already dropped are skipped), x [N][d]
 *   offsets_pad [E+1] = e*C, counts [E] (kept per expert, <= C), row_token_pad [E*C] or NULL,
 *   slot_row [N][k] = e*C + rank or -1, xp_pad [E*C][d]: outputs. */
MOE_API moe_status moe_permute_padded(const moe_config* cfg, const int32_t* ids,
                                      const uint8_t* drop_mask, const void* x,
                                      int32_t* offsets_pad, int32_t* counts,
                                      int32_t* row_token_pad, int32_t* slot_row, void* xp_pad,
                                      void* ws, moe_stream_t stream);

/* moe_forward through the padded layout: the expert FFNs run over the E*C padded rows
 * (empty slots are computed on zero rows and never combined), the shared expert's rows follow
 * at E*C + t.  Same result as moe_forward.  route_out->offsets, when given, receives the padded
 * offsets e*C.  Needs cfg->capacity > 0; the workspace of moe_workspace_size covers it. */
MOE_API moe_status moe_forward_padded(const moe_config* cfg, const void* x, const void* W_g,
                                      const float* logit_offset, const float* bias,
                                      const uint8_t* modality, const void* W_gu,
                                      const void* W_down, void* y,
                                      const moe_route_out* route_out, void* ws,
                                      moe_stream_t stream);

/* ---- expert parallelism ---------------------------------------------------------------
 * "Mixture-of-Experts : routage et capacité" slides, "Le problème — Communication", "L'idée —
 * Communication" and "Support visuel — Communication": the routed experts are spread over
 * `world` ranks (one process per GPU); each rank routes its own tokens, ships every kept
 * assignment's row to the rank that owns the expert (dispatch), the owner runs its experts,
 * and the outputs come back to the token's rank (combine).  Rank o owns the contiguous
 * experts [moe_ep_first_expert(world, o, E), moe_ep_first_expert(world, o + 1, E)); every
 * rank holds the router weights and the shared expert.  The result on every rank equals the
 * single-device layer (moe_forward) over the concatenation of all ranks' tokens, rank 0's
 * first: capacity serves each expert's assignments in that order.  The calls below are the
 * per-rank steps; the exchanges between them (an all-gather of per-expert demands and the
 * row messages the plan lists) belong to the caller's communication library (NCCL). */

/* One run of rows exchanged with one peer for one expert. */
typedef struct {
  int32_t peer;    /* the other rank */
  int32_t expert;  /* global expert id; usable as the message tag */
  int64_t row;     /* first row in this rank's buffer */
  int64_t rows;    /* number of rows, > 0 */
} moe_ep_chunk;

/* First expert owned by `rank` (rank in [0, world]; rank == world gives E), or -1 on a bad
 * argument.  Experts are split into contiguous runs of floor or ceil(E / world).  Host only. */
MOE_API int32_t moe_ep_first_expert(int32_t world, int32_t rank, int32_t E);

/* The exchange plan of one rank, from every rank's per-expert demand (host only, no GPU).
 *   demand_all [world][E] host: assignments per expert of each rank's tokens before capacity
 *              (moe_route's demand output, all-gathered)
 *   capacity   C for the whole concatenated batch (<= 0: no limit)
 * Outputs (host, caller-allocated; any may be NULL):
 *   cap [E]              how many of this rank's assignments to e it keeps, the first in its
 *                        token order: C minus the demand of the earlier ranks, clamped to
 *                        [0, C] (INT32_MAX without a limit); the input of moe_permute_ep
 *   kept_all [world][E]  kept assignments of every rank per expert
 *   owned_offsets [E_own + 1]  group offsets of the receive buffer of this rank's experts
 *   sends [<= E]         this rank's send buffer (moe_permute_ep's xp) as runs: expert e's kept
 *                        rows go to its owner; listed by increasing expert
 *   recvs [<= world * E_own]  where the rows of each (expert, source rank) land in the receive
 *                        buffer: expert-major, then source rank (the concatenated batch's token
 *                        order); listed by increasing expert, then rank
 *   n_sends, n_recvs     numbers of runs; rows_kept = this rank's kept rows (send buffer
 *                        rows), rows_owned = receive buffer rows
 * Runs with the same peer appear in the same expert order on both sides, so a grouped
 * send/receive posted in list order matches.  The return trip of the combine uses the same
 * lists with the roles swapped.  MOE_ERR_INVALID_ARG for a bad rank or negative demand;
 * MOE_ERR_UNSUPPORTED when world > E or a buffer would exceed 2^30 rows. */
MOE_API moe_status moe_ep_plan(int32_t world, int32_t rank, int32_t E, int64_t capacity,
                               const int32_t* demand_all, int32_t* cap, int32_t* kept_all,
                               int32_t* owned_offsets, moe_ep_chunk* sends, int32_t* n_sends,
                               moe_ep_chunk* recvs, int32_t* n_recvs, int64_t* rows_kept,
                               int64_t* rows_owned);

/* Workspace bytes of an expert-parallel rank: cfg is the whole layer (all E experts) with
 * cfg->N = the most tokens any rank routes; covers moe_route, moe_permute_ep and
 * moe_ep_expert_ffn.  0 on a bad config or world > E. */
MOE_API size_t moe_ep_workspace_size(const moe_config* cfg, int32_t world);

/* moe_permute with a per-expert capacity: the assignment (t, j) to expert e is kept iff its
 * rank among this rank's assignments to e (token order) is below cap[e] (device int32 [E],
 * from moe_ep_plan).  Outputs as in moe_permute, plus counts [E] (kept per expert) and
 * drop_mask [N][k] (either may be NULL).  cfg->capacity is not used. */
MOE_API moe_status moe_permute_ep(const moe_config* cfg, const int32_t* ids, const int32_t* cap,
                                  const void* x, int32_t* offsets, int32_t* row_token,
                                  int32_t* slot_row, void* xp, int32_t* counts,
                                  uint8_t* drop_mask, void* ws, moe_stream_t stream);

/* moe_permute_ep with the kept rows written straight into their destinations instead of a
 * send buffer: the dispatch passes and the transfer in one pass over the rows (peer-memory
 * expert parallelism).  Expert e's kept rows, in their layout order, go to rows dst_row0[e],
 * dst_row0[e] + 1, ... of the buffer at dst_base[e] (device uint64 [E]: the receive buffer of
 * e's owner -- another process's allocation mapped with moe_ipc_open, or a local buffer),
 * which holds dst_rows[e] rows (device int64 [E]; a row past it is skipped and reported as
 * MOE_ERR_INVALID_INPUT by moe_check_status).  Other outputs as in moe_permute_ep (no
 * row_token).  bf16 only; d * 2 a multiple of 16.  The caller orders it against the
 * destinations' work as for moe_ep_copy_runs. */
MOE_API moe_status moe_permute_ep_p2p(const moe_config* cfg, const int32_t* ids,
                                      const int32_t* cap, const void* x, int32_t* offsets,
                                      int32_t* slot_row, const uint64_t* dst_base,
                                      const int32_t* dst_row0, const int64_t* dst_rows,
                                      int32_t* counts, uint8_t* drop_mask, void* ws,
                                      moe_stream_t stream);

/* The owner's expert FFNs (bf16): the received rows xr [rows][d], grouped by owned_offsets
 * (device int32 [E_own + 1], from moe_ep_plan), through the rank's experts, into ye
 * [rows][d]; with n_shared == 1 also the shared expert on this rank's own n_tokens tokens
 * x [n_tokens][d], written into y [n_tokens][d] (moe_ep_combine then adds the routed slots
 * to it).  cfg is the whole layer exactly as given to moe_ep_workspace_size (cfg->N = the
 * most tokens any rank routes, which sizes the workspace); n_tokens <= cfg->N.  W_gu
 * [E_own + S][.][d] and W_down [E_own + S][d][F] hold this rank's experts (shared last).
 * rows is the host value rows_owned of the plan, at most world * cfg->N * k. */
MOE_API moe_status moe_ep_expert_ffn(const moe_config* cfg, int32_t world, int32_t rank,
                                     int64_t n_tokens, int64_t rows, const void* xr,
                                     const int32_t* owned_offsets, const void* x,
                                     const void* W_gu, const void* W_down, void* ye, void* y,
                                     void* ws, moe_stream_t stream);

/* The combine on the token's rank (bf16): ye [rows_kept][d] holds the expert outputs in the
 * send buffer's row order (the return trip of the plan's runs); with n_shared == 1, y [N][d]
 * already holds the shared expert's rows (moe_ep_expert_ffn) and the kept slots are added to
 * them in place, in slot order, one rounding; with n_shared == 0, y = the gate-weighted sum. */
MOE_API moe_status moe_ep_combine(const moe_config* cfg, const void* ye, const int32_t* slot_row,
                                  const float* gates, void* y, moe_stream_t stream);

/* moe_ep_combine with the return trip folded in ("Support visuel — Communication": the
 * expert's output travels back to the token's device): each kept slot's expert output is read
 * where its owner wrote it, instead of from a local ye.  Slot (t, j), kept for expert
 * e = ids[t][j] at row r = slot_row[t][j] of this rank's send layout (offsets [E + 1] from
 * moe_permute_ep / moe_permute_ep_p2p), reads row src_row0[e] + (r - offsets[e]) of the buffer
 * at src_base[e] (device uint64 [E]: the output buffer of e's owner, another process's
 * allocation mapped with moe_ipc_open, or a local buffer), which holds src_rows[e] rows (device
 * int64 [E]).  A slot whose expert or row falls outside these bounds contributes nothing and
 * is reported as MOE_ERR_INVALID_INPUT by moe_check_status.  The sums, their order and the
 * rounding are those of moe_ep_combine, so the bits are too.  bf16 only; d * 2 a multiple of
 * 16.  The caller orders it after the owners' expert FFNs (a stream-ordered barrier) and
 * keeps the owners from overwriting their outputs until every rank's combine is done. */
MOE_API moe_status moe_ep_combine_p2p(const moe_config* cfg, const int32_t* ids,
                                      const int32_t* slot_row, const float* gates,
                                      const int32_t* offsets, const uint64_t* src_base,
                                      const int32_t* src_row0, const int64_t* src_rows, void* y,
                                      void* ws, moe_stream_t stream);

/* The exchange of the plan's row runs over peer memory ("Support visuel — Communication"):
 * one launch writes rows of src [src_rows][row_bytes] (this device) straight into other
 * buffers -- another process's allocation mapped with moe_ipc_open (on a multi-GPU node,
 * reached over NVLink), or a local buffer.
 *   dst_base [n_bufs]  device array of destination buffer addresses (uint64)
 *   dst_rows [n_bufs]  device array of their sizes in rows (int64): bounds of every write
 *   runs [n_runs][4]   device int32: (src_row, dst_buf, dst_row, rows) per run, rows > 0
 *   run_start [n_runs + 1]  device int32 prefix of the runs' rows; total_rows = its last entry
 *   row_bytes          a multiple of 16; every buffer 16-byte aligned
 *   ws                 NULL, or a workspace whose status word records out-of-range runs
 *                      (those are skipped; MOE_ERR_INVALID_INPUT from moe_check_status)
 * The caller orders it against the destinations' own work: a stream-ordered barrier before
 * (the destination is done with the buffer's previous contents) and after (its next kernels
 * see the rows).  MOE_ERR_INVALID_ARG on a bad size or a null pointer. */
MOE_API moe_status moe_ep_copy_runs(const void* src, int64_t src_rows,
                                    const uint64_t* dst_base, const int64_t* dst_rows,
                                    int32_t n_bufs, const int32_t* runs,
                                    const int32_t* run_start, int32_t n_runs, int64_t total_rows,
                                    int64_t row_bytes, void* ws, moe_stream_t stream);

/* CUDA IPC for moe_ep_copy_runs' destinations.  moe_ipc_handle: the 64-byte handle of the
 * allocation containing the device pointer ptr, and ptr's byte offset inside it (a caching
 * allocator hands out pointers inside larger allocations).  moe_ipc_open: map another
 * process's handle into this one (peer access enabled as needed); *base is the allocation's
 * base, to which the owner's offset is added.  moe_ipc_close: unmap it.  A handle cannot be
 * opened in the process that made it.  MOE_ERR_CUDA on a driver refusal. */
MOE_API moe_status moe_ipc_handle(const void* ptr, void* handle, int64_t* offset);
MOE_API moe_status moe_ipc_open(const void* handle, void** base);
MOE_API moe_status moe_ipc_close(void* base);

/* moe_forward with x_host and y_host in HOST memory (pinned for full copy speed): copies
 * x to the workspace, runs the layer, copies y back and synchronises the stream.
 * Weights, bias, modality and logit_offset are device pointers as in moe_forward. */
MOE_API moe_status moe_forward_host(const moe_config* cfg, const void* x_host, const void* W_g,
                            const float* logit_offset, const float* bias,
                            const uint8_t* modality, const void* W_gu, const void* W_down,
                            void* y_host, void* ws, moe_stream_t stream);

/* moe_route on given logits without a workspace: the same routing and capacity results
 * (ids, gates, counts, demand, drop_mask) for callers that cannot allocate device memory,
 * e.g. a plug-in running inside a host process whose memory manager has already reserved
 * the whole device (a cudaMalloc there fails or breaks the host's budget), or a latency-
 * critical loop that must not risk the implicit device synchronisation of cudaMalloc.
 * The pages have no counterpart of this call; it is a deployment convenience.
 * Scratch: a fixed 4 MiB device array inside the library (every GPU that loads the library
 * holds it until the process exits).  The call needs 256 + 4*N*k + 2*(4*ceil(N/32)*E) +
 * 4*(E + 1) bytes of it, each of the four parts rounded up to 256; larger requests return
 * MOE_ERR_UNSUPPORTED before anything is enqueued.  Examples: N = 16384, k = 8, E = 256 needs
 * 1.5 MiB and fits; N = 65536, k = 8, E = 8 needs 2.1 MiB and fits; N = 16384, k = 8,
 * E = 1024 needs 4.5 MiB (the per-tile histograms dominate) and is refused.
 * The first call on a device (and again after a device reset, which gives the device a new
 * context) looks up the array's device address (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture.
 * All calls share the array and it keeps the last call's contents: calls that may overlap
 * on the GPU (other streams, other host threads) race -- order them on one stream.
 *   status: optional device int32; device findings (a modality flag >= n_bias_sets) are
 *           recorded there as in the workspace status word (the caller zeroes it).
 * Other arguments as in moe_route; cfg->N, E, k, n_bias_sets, score_fn, renorm and
 * capacity are used.  Allocates nothing (no cudaMalloc/cudaFree, no library allocator). */
MOE_API moe_status moe_route_static(const moe_config* cfg, const float* logits,
                                    const float* bias, const uint8_t* modality, int32_t* ids,
                                    float* gates, int32_t* counts, int32_t* demand,
                                    uint8_t* drop_mask, int32_t* status, moe_stream_t stream);

/* A sequence of batches with x and y in HOST memory, pipelined: batch b+1 is copied in on one
 * copy stream and batch b-1 copied out on another while batch b runs on `stream`, through two
 * staging pairs in the workspace.  x_host[b] [N][d] and y_host[b] [N][d] are host pointers
 * (pinned memory lets the copies overlap the layer); modality may be NULL or hold one device
 * pointer per batch.  Each batch is one layer call of cfg->N tokens (capacity applies per
 * batch).  Returns after the last batch's result is in host memory.  The two copy streams and
 * their events are created on first use and kept by the calling thread. */
MOE_API moe_status moe_forward_host_batches(const moe_config* cfg, int32_t n_batches,
                                            const void* const* x_host, const void* W_g,
                                            const float* logit_offset, const float* bias,
                                            const uint8_t* const* modality, const void* W_gu,
                                            const void* W_down, void* const* y_host, void* ws,
                                            moe_stream_t stream);

/* Failure-detection self-test (the pages have no counterpart): one device thread waits, with
 * the same bounded wait the GEMM pipelines use, on a barrier that nothing ever completes.  The
 * wait runs out after limit_ns (0 .. 1e9; a backstop poll count ends it too if the GPU timer
 * stalls) and records MOE_ERR_TIMEOUT in the workspace status word, which moe_check_status
 * then reports -- the path a stalled pipeline takes.  The kernel ends normally: the context
 * stays usable.  Asynchronous on `stream`; MOE_ERR_INVALID_ARG for a NULL ws or a limit
 * outside the range. */
MOE_API moe_status moe_selftest_wait_timeout(void* ws, int64_t limit_ns, moe_stream_t stream);

/* Debugging aid (the pages have no counterpart): checks a dispatch layout's invariants on
 * the host -- ids in range and distinct within a token; offsets[0] = 0 and offsets[e+1] -
 * offsets[e] = counts[e] <= capacity (if > 0) and <= demand[e] (if demand is given); a slot
 * is dropped iff its slot_row is -1; every kept slot's row lies in its expert's group, rows
 * are used once and row_token maps them back (if given); kept + dropped = N k; each expert's
 * rows follow token order and it keeps no token after one it dropped (the capacity rule of
 * "Mixture-of-Experts : routage et capacité", "L'idée — Capacité").  All arrays in HOST memory
 * (row_token [offsets[E]] may be NULL, demand may be NULL).  Returns MOE_OK, or
 * MOE_ERR_INVALID_INPUT with the first broken invariant written to msg (msg_len bytes).
 * With the environment variable MOE_B200_DEBUG=1 the fused forward calls run this check on
 * their own layout after the dispatch passes (synchronising the stream: eager calls only). */
MOE_API moe_status moe_check_dispatch_host(int64_t N, int32_t k, int32_t E, int64_t capacity,
                                           const int32_t* ids, const uint8_t* drop_mask,
                                           const int32_t* counts, const int32_t* demand,
                                           const int32_t* offsets, const int32_t* slot_row,
                                           const int32_t* row_token, char* msg,
                                           size_t msg_len);

/* The same check on DEVICE arrays (copied to the host; synchronises `stream`): cfg->N, k, E
 * and capacity give the shapes and the rule.  The broken invariant is in moe_last_error(). */
MOE_API moe_status moe_check_dispatch(const moe_config* cfg, const int32_t* ids,
                                      const uint8_t* drop_mask, const int32_t* counts,
                                      const int32_t* demand, const int32_t* offsets,
                                      const int32_t* slot_row, const int32_t* row_token,
                                      moe_stream_t stream);

/* Synchronise `stream`, read and clear the workspace status word.  Returns MOE_OK or the
 * first device-detected error (MOE_ERR_INVALID_INPUT, MOE_ERR_TIMEOUT) since the last
 * check; MOE_ERR_CUDA if the stream reports an asynchronous CUDA error. */
MOE_API moe_status moe_check_status(void* ws, moe_stream_t stream);

/* Text of the last error raised on the calling thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* Per-launch timing of moe_forward on the calling thread.  After moe_profile_begin(n), the
 * next n calls of moe_forward / moe_forward_host record a CUDA event on their stream before
 * their first kernel and after each kernel (the events carry timing; nothing else changes).
 * moe_profile_end synchronises on the recorded events, writes into launch_ms[i] the total
 * milliseconds of the i-th launch summed over the recorded calls (i < max_launches), stores
 * the number of recorded calls in *calls, releases the events and returns the number of
 * launches per call (or -1 on a CUDA error).  Launch order of a bf16 forward: router GEMM,
 * top-k, rank pass, scan pass, scatter/gather pass, gate/up GEMM, down GEMM, combine. */
MOE_API moe_status moe_profile_begin(int32_t max_calls);
MOE_API int32_t moe_profile_end(float* launch_ms, int32_t max_launches, int32_t* calls);

/* Number of kernel launches the last successful entry point on this thread enqueued. */
MOE_API int32_t moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_MOE_H_ */
