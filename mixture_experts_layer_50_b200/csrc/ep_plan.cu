// Expert-parallel plan (host only): which rows one rank keeps, sends and receives when the
// routed experts are spread over `world` ranks and every rank routes its own tokens.
//
// "Mixture-of-Experts : routage et capacité" slides, "Le problème — Communication" and "L'idée
// — Communication": the experts live on different devices, so each token's row travels to
// the device of every expert it picked (dispatch all-to-all) and each expert output travels
// back to the token's device (combine all-to-all).
//
// The plan reproduces the single-device layer on the concatenation of all ranks' tokens
// (rank 0's tokens first, then rank 1's, ...).  Capacity ("L'idée — Capacité") serves an
// expert's assignments in that token order, so rank r may keep at most
//   cap_r[e] = C - sum_{r' < r} demand[r'][e]   (clamped to [0, C])
// of its own assignments to e, the first ones in its token order.  The per-expert demands of
// every rank (one all-gather of E counts per rank) fix every rank's kept counts, hence every
// message size, before any row moves.
//
// Layouts:
//  - a rank's send buffer is its compact per-expert layout (moe_permute_ep): expert e's
//    kept rows at [koff[e], koff[e] + kept[rank][e]), experts in increasing order, so the
//    rows bound for one owner (a contiguous range of experts) are contiguous;
//  - an owner's receive buffer is expert-major over the experts it owns, and inside an
//    expert source-rank-major: the rows of expert e from rank r follow those from ranks
//    r' < r, which is the token order of the concatenated batch -- the single-device layout
//    of those experts' groups.
#include <stdint.h>

#include <algorithm>
#include <climits>
#include <vector>

#include "../../include/moe.h"

namespace {

int64_t first_expert(int32_t world, int32_t rank, int32_t E) {
  return (int64_t)rank * E / world;
}

}  // namespace

extern "C" {

int32_t moe_ep_first_expert(int32_t world, int32_t rank, int32_t E) {
  if (world < 1 || rank < 0 || rank > world || E < 1) return -1;
  return (int32_t)first_expert(world, rank, E);
}

moe_status moe_ep_plan(int32_t world, int32_t rank, int32_t E, int64_t capacity,
                       const int32_t* demand_all, int32_t* cap, int32_t* kept_all,
                       int32_t* owned_offsets, moe_ep_chunk* sends, int32_t* n_sends,
                       moe_ep_chunk* recvs, int32_t* n_recvs, int64_t* rows_kept,
                       int64_t* rows_owned) {
  if (world < 1 || rank < 0 || rank >= world || E < 1 || demand_all == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (world > E) return MOE_ERR_UNSUPPORTED;  // every rank owns at least one expert
  for (int64_t i = 0; i < (int64_t)world * E; ++i)
    if (demand_all[i] < 0) return MOE_ERR_INVALID_ARG;

  // kept[r][e]: rank r keeps its first kept[r][e] assignments to e (token order)
  std::vector<int64_t> kept((size_t)world * E);
  std::vector<int64_t> base(E, 0);  // demand of the earlier ranks, per expert
  for (int32_t r = 0; r < world; ++r) {
    for (int32_t e = 0; e < E; ++e) {
      const int64_t dem = demand_all[(int64_t)r * E + e];
      int64_t c = INT32_MAX;
      if (capacity > 0) c = std::max<int64_t>(0, std::min<int64_t>(capacity - base[e], INT32_MAX));
      if (r == rank && cap != nullptr) cap[e] = (int32_t)c;
      kept[(size_t)r * E + e] = std::min(dem, c);
      base[e] += dem;
    }
  }
  if (kept_all != nullptr)
    for (size_t i = 0; i < kept.size(); ++i) kept_all[i] = (int32_t)kept[i];

  // sends: this rank's kept rows, expert by expert, to each expert's owner
  int32_t owner = 0;
  int64_t koff = 0;
  int32_t ns = 0;
  for (int32_t e = 0; e < E; ++e) {
    while (first_expert(world, owner + 1, E) <= e) ++owner;
    const int64_t rows = kept[(size_t)rank * E + e];
    if (rows > 0 && sends != nullptr) sends[ns] = moe_ep_chunk{owner, e, koff, rows};
    if (rows > 0) ++ns;
    koff += rows;
  }
  // receives: the owned experts' rows from every rank, expert-major, then rank order
  const int64_t e0 = first_expert(world, rank, E), e1 = first_expert(world, rank + 1, E);
  int64_t off = 0;
  int32_t nr = 0;
  for (int64_t e = e0; e < e1; ++e) {
    if (owned_offsets != nullptr) owned_offsets[e - e0] = (int32_t)off;
    for (int32_t r = 0; r < world; ++r) {
      const int64_t rows = kept[(size_t)r * E + e];
      if (rows > 0 && recvs != nullptr) recvs[nr] = moe_ep_chunk{r, (int32_t)e, off, rows};
      if (rows > 0) ++nr;
      off += rows;
    }
  }
  if (owned_offsets != nullptr) owned_offsets[e1 - e0] = (int32_t)off;
  if (koff > INT32_MAX / 2 || off > INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
  if (n_sends != nullptr) *n_sends = ns;
  if (n_recvs != nullptr) *n_recvs = nr;
  if (rows_kept != nullptr) *rows_kept = koff;
  if (rows_owned != nullptr) *rows_owned = off;
  return MOE_OK;
}

}  // extern "C"
