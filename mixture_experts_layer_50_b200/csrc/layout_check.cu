// Host-side check of a dispatch layout's invariants: the library's debugging aid where no
// device sanitizer is at hand.  The invariants are those of the capacity rule and the
// per-expert layout ("Mixture-of-Experts : routage et capacité", "L'idée — Capacité" and
// "Support visuel — Capacité": an expert keeps its first C assignments in arrival order,
// and its kept tokens are laid out in that order).
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "../../include/moe.h"

namespace {

template <typename... T>
moe_status broken(char* msg, size_t len, const char* fmt, T... v) {
  if (msg != nullptr && len > 0) snprintf(msg, len, fmt, (long long)v...);
  return MOE_ERR_INVALID_INPUT;
}

}  // namespace

extern "C" {

moe_status moe_check_dispatch_host(int64_t N, int32_t k, int32_t E, int64_t capacity,
                                   const int32_t* ids, const uint8_t* drop_mask,
                                   const int32_t* counts, const int32_t* demand,
                                   const int32_t* offsets, const int32_t* slot_row,
                                   const int32_t* row_token, char* msg, size_t msg_len) {
  if (msg != nullptr && msg_len > 0) msg[0] = '\0';
  if (N < 0 || k < 1 || E < 1 || ids == nullptr || drop_mask == nullptr || counts == nullptr ||
      offsets == nullptr || slot_row == nullptr)
    return MOE_ERR_INVALID_ARG;
  // offsets: start at 0, non-decreasing, steps equal to the counts; counts within capacity
  // and demand
  if (offsets[0] != 0) return broken(msg, msg_len, "offsets[0] = %lld, not 0", offsets[0]);
  for (int32_t e = 0; e < E; ++e) {
    if (offsets[e + 1] - offsets[e] != counts[e])
      return broken(msg, msg_len, "expert %lld: offsets step %lld != counts %lld", e,
                    offsets[e + 1] - offsets[e], counts[e]);
    if (counts[e] < 0) return broken(msg, msg_len, "expert %lld: counts %lld < 0", e, counts[e]);
    if (capacity > 0 && counts[e] > capacity)
      return broken(msg, msg_len, "expert %lld keeps %lld > capacity %lld", e, counts[e], capacity);
    if (demand != nullptr && counts[e] > demand[e])
      return broken(msg, msg_len, "expert %lld keeps %lld > its demand %lld", e, counts[e], demand[e]);
  }
  const int64_t M = offsets[E];
  if (M > N * k) return broken(msg, msg_len, "offsets[E] = %lld > N k = %lld", M, N * k);
  // every slot: a valid, distinct expert; dropped iff no row; a kept row inside its expert's
  // group; each row used once; the row maps back to its token
  std::vector<int64_t> owner((size_t)M, -1);
  int64_t kept = 0, drops = 0;
  for (int64_t t = 0; t < N; ++t) {
    for (int32_t j = 0; j < k; ++j) {
      const int64_t i = t * k + j;
      const int32_t e = ids[i];
      if (e < 0 || e >= E) return broken(msg, msg_len, "token %lld slot %lld: expert id %lld out of range", t, j, e);
      for (int32_t jj = 0; jj < j; ++jj)
        if (ids[t * k + jj] == e)
          return broken(msg, msg_len, "token %lld lists expert %lld twice (slot %lld)", t, e, j);
      const int32_t r = slot_row[i];
      if (drop_mask[i] > 1) return broken(msg, msg_len, "token %lld slot %lld: drop flag %lld", t, j, drop_mask[i]);
      if (drop_mask[i]) {
        ++drops;
        if (r != -1) return broken(msg, msg_len, "token %lld slot %lld is dropped but has row %lld", t, j, r);
        continue;
      }
      ++kept;
      if (r < offsets[e] || r >= offsets[e + 1])
        return broken(msg, msg_len, "token %lld slot %lld: row %lld outside its expert's group", t, j, r);
      if (owner[(size_t)r] != -1)
        return broken(msg, msg_len, "row %lld used by tokens %lld and %lld", r, owner[(size_t)r], t);
      owner[(size_t)r] = t;
      if (row_token != nullptr && row_token[r] != t)
        return broken(msg, msg_len, "row %lld maps to token %lld, not %lld", r, row_token[r], t);
    }
  }
  if (kept != M) return broken(msg, msg_len, "%lld kept slots for %lld rows", kept, M);
  if (kept + drops != N * k)
    return broken(msg, msg_len, "kept %lld + dropped %lld != N k = %lld", kept, drops, N * k);
  // per expert: rows in token order, and the kept assignments are the first ones in token
  // order (no kept assignment after a dropped one)
  std::vector<int64_t> first_drop(E, INT64_MAX);
  for (int64_t t = 0; t < N; ++t) {
    for (int32_t j = 0; j < k; ++j) {
      const int64_t i = t * k + j;
      const int32_t e = ids[i];
      if (drop_mask[i]) {
        if (first_drop[e] == INT64_MAX) first_drop[e] = t;
      } else {
        if (t > first_drop[e])
          return broken(msg, msg_len, "expert %lld keeps token %lld after dropping token %lld", e,
                        t, first_drop[e]);
      }
    }
  }
  for (int32_t e = 0; e < E; ++e)
    for (int64_t r = offsets[e] + 1; r < offsets[e + 1]; ++r)
      if (owner[(size_t)r] <= owner[(size_t)r - 1])
        return broken(msg, msg_len, "expert %lld: rows %lld and its predecessor not in token order (token %lld)",
                      e, r, owner[(size_t)r]);
  return MOE_OK;
}

}  // extern "C"
