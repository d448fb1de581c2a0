// partition.cu -- splitting one packed batch's users into contiguous ranges,
// one per GPU, balanced by each user's cost (host code only).
//
// Users are independent (cti2026 README: a packed batch is users laid end to
// end with user_offsets boundaries, and attention never crosses a boundary),
// so a contiguous range of users is a batch of its own.  The cost of a user
// of L tokens is the work the layer does for it: 6,299,648 FLOPs per token
// for the GEMMs (QKV 2*512*1536, output 2*512*512, gate 2*512*8, two expert
// routes of 2*2*512*1024) plus 2048 * L(L+1)/2 for its causal attention (QK^T
// and PV over 8 heads of 64).  The split minimises the largest part's cost
// over all contiguous splits (the "linear partition" problem): the smallest
// bound B for which a greedy left-to-right fill needs at most num_parts
// parts, found by bisection on B; the parts are then that greedy fill.
#include <cstdint>

#include "../../include/ptl.h"

namespace {

constexpr int64_t kGemmFlopsPerToken = 2 * 512 * 1536 + 2 * 512 * 512 + 2 * 512 * 8 + 2 * 2 * (2 * 512 * 1024);

inline int64_t user_cost(int64_t L) { return kGemmFlopsPerToken * L + 1024 * L * (L + 1); }

// Parts a greedy fill with bound B needs (each part takes users while its
// cost stays <= B); num_parts + 1 once it exceeds num_parts, or when a single
// user costs more than B.
int32_t parts_needed(const int32_t* cu, int32_t U, int64_t B, int32_t limit) {
  int32_t parts = 1;
  int64_t acc = 0;
  for (int32_t u = 0; u < U; ++u) {
    const int64_t c = user_cost(int64_t(cu[u + 1]) - cu[u]);
    if (c > B) return limit + 1;
    if (acc + c > B) {
      if (++parts > limit) return parts;
      acc = 0;
    }
    acc += c;
  }
  return parts;
}

}  // namespace

extern "C" ptl_status ptl_partition_users(const int32_t* cu_seqlens, int32_t num_users, int32_t num_parts,
                                          int32_t* user_begin) {
  if (!cu_seqlens || !user_begin) return PTL_ERR_NULL;
  if (num_users < 1 || num_parts < 1) return PTL_ERR_SHAPE;
  if (cu_seqlens[0] != 0) return PTL_ERR_BAD_OFFSETS;
  int64_t total = 0, biggest = 0;
  for (int32_t u = 0; u < num_users; ++u) {
    if (cu_seqlens[u + 1] < cu_seqlens[u]) return PTL_ERR_BAD_OFFSETS;
    const int64_t c = user_cost(int64_t(cu_seqlens[u + 1]) - cu_seqlens[u]);
    total += c;
    if (c > biggest) biggest = c;
  }
  // smallest feasible bound in [biggest, total] (total is always feasible)
  int64_t lo = biggest, hi = total;
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if (parts_needed(cu_seqlens, num_users, mid, num_parts) <= num_parts)
      hi = mid;
    else
      lo = mid + 1;
  }
  // the greedy fill at that bound
  int32_t part = 0;
  int64_t acc = 0;
  user_begin[0] = 0;
  for (int32_t u = 0; u < num_users; ++u) {
    const int64_t c = user_cost(int64_t(cu_seqlens[u + 1]) - cu_seqlens[u]);
    if (acc + c > lo && part + 1 < num_parts) {
      user_begin[++part] = u;
      acc = 0;
    }
    acc += c;
  }
  for (int32_t r = part + 1; r <= num_parts; ++r) user_begin[r] = num_users;
  return PTL_OK;
}
