// Overflow policy "report": a slot dropped by the capacity goes to the token's next-best expert
// if that expert still has room.
//
// "Mixture-of-Experts : routage et capacité" slides, table "Politiques de débordement quand E1
// reçoit 6 tokens pour C = 5", row "Report sur E2/E3": the rejected token is handled by its
// third-best score.  Read here as: after the capacity pass, a token's i-th dropped slot (slot
// order) is offered its (k+i)-th best expert by selection key; the offers to one expert are
// served in token order, then slot order, while the expert's kept count plus the offers it
// took stays below C; an offer without room leaves the slot dropped.  The gates are then the
// usual ones over the token's final slot list (a moved slot takes its new expert's score; a
// slot still dropped stays in the list and contributes 0).
//
// The offers are ranked with the same deterministic rank / scan passes as the first pass
// (csrc/dispatch.cu), so every decision is a fixed function of the router's keys.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// One thread per token: slot j's offer is the token's next unused candidate if j was dropped.
__global__ void reroute_offer_kernel(const int32_t* __restrict__ ids,
                                     const uint8_t* __restrict__ drop1,
                                     const int32_t* __restrict__ cand, int64_t N, int k,
                                     int32_t* __restrict__ offer, uint8_t* __restrict__ not_offer) {
  pdl_wait();
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= N) return;
  int i = 0;
  for (int j = 0; j < k; ++j) {
    const int64_t s = t * k + j;
    int32_t e = ids[s];   // a valid id where there is no offer: the rank pass skips it
    uint8_t none = 1;
    if (drop1[s]) {
      const int32_t c = cand[t * k + i];
      if (c >= 0) {
        e = c;
        none = 0;
      }
      ++i;
    }
    offer[s] = e;
    not_offer[s] = none;
  }
}

// One warp per token, lane j = slot j: take the offer if it ranks below the room left, then the
// gates over the final slot list with the same arithmetic as the top-k kernel.
__global__ void __launch_bounds__(256) reroute_accept_kernel(
    int32_t* __restrict__ ids, const uint8_t* __restrict__ drop1,
    const int32_t* __restrict__ offer, const uint8_t* __restrict__ not_offer,
    const int32_t* __restrict__ local_rank, const int32_t* __restrict__ tile_base,
    const int32_t* __restrict__ counts1, const float* __restrict__ cand_val, int64_t N, int E,
    int k, int64_t C, int score_fn, int renorm, float* __restrict__ gates,
    uint8_t* __restrict__ drop_out, uint8_t* __restrict__ rerouted) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= N) return;
  const bool mine = lane < k;
  const int64_t s = t * k + lane;
  int e = -1;
  bool d1 = false, moved = false;
  float v = 0.0f;
  if (mine) {
    e = ids[s];
    d1 = drop1[s] != 0;
    v = cand_val[t * 2 * k + lane];
  }
  const unsigned dropped = __ballot_sync(0xffffffffu, mine && d1);
  if (mine && d1 && !not_offer[s]) {
    const int ep = offer[s];
    const int64_t r = (int64_t)tile_base[(t / kRankTile) * E + ep] + local_rank[s];
    if ((int64_t)counts1[ep] + r < C) {
      moved = true;
      e = ep;
      const int i = __popc(dropped & ((1u << lane) - 1u));
      v = cand_val[t * 2 * k + k + i];
    }
  }
  float g;
  if (score_fn == 0) {
    if (renorm) {
      const float m = warp_max(mine ? v : -INFINITY);
      const float ex = mine ? expf(v - m) : 0.0f;
      g = ex / warp_sum(ex);
    } else {
      g = v;
    }
  } else {
    g = renorm ? v / warp_sum(mine ? v : 0.0f) : v;
  }
  if (mine) {
    ids[s] = e;
    gates[s] = g;
    drop_out[s] = (d1 && !moved) ? 1 : 0;
    if (rerouted != nullptr) rerouted[s] = moved ? 1 : 0;
  }
}

}  // namespace

cudaError_t launch_reroute_offer(const int32_t* ids, const uint8_t* drop1, const int32_t* cand,
                                 int64_t N, int k, int32_t* offer, uint8_t* not_offer,
                                 cudaStream_t stream, int* launches) {
  if (N == 0) return cudaSuccess;
  ++*launches;
  launch_pdl(reroute_offer_kernel, (unsigned)((N + 255) / 256), 256, 0, stream, ids, drop1, cand, N, k,
                                                                       offer, not_offer);
  return cudaGetLastError();
}

cudaError_t launch_reroute_accept(int32_t* ids, const uint8_t* drop1, const int32_t* offer,
                                  const uint8_t* not_offer, const int32_t* local_rank,
                                  const int32_t* tile_base, const int32_t* counts1,
                                  const float* cand_val, int64_t N, int E, int k, int64_t C,
                                  int score_fn, int renorm, float* gates, uint8_t* drop_out,
                                  uint8_t* rerouted, cudaStream_t stream, int* launches) {
  if (N == 0) return cudaSuccess;
  ++*launches;
  launch_pdl(reroute_accept_kernel, (unsigned)((N * 32 + 255) / 256), 256, 0, stream, 
      ids, drop1, offer, not_offer, local_rank, tile_base, counts1, cand_val, N, E, k, C,
      score_fn, renorm, gates, drop_out, rerouted);
  return cudaGetLastError();
}

}  // namespace moe
