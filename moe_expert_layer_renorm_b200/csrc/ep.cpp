// Expert-parallel exchange plan (host only).  The fork's production
// configuration splits each MoE layer's experts over two GPUs
// ("sm89-moe-offload" fork README, "Production configuration",
// --moe-ep-size 2); the ownership and row order below are this library's
// reading, stated in ftmoe.h.
//
// From every rank's expert_offsets (an all-gather of G rows of E + 1), rank
// `rank` derives:
//   send_rows[d]  = offsets_rank[e1(d)] - offsets_rank[e0(d)]   (its rows for d)
//   recv_rows[s]  = offsets_s[e1(rank)] - offsets_s[e0(rank)]   (s's rows for it)
// Rows arrive from s at base_s = sum_{s' < s} recv_rows[s'], in s's
// permuted order: expert e's rows from s sit at
//   arrive(s, e, i) = base_s + offsets_s[e] - offsets_s[e0(rank)] + i.
// The FFN visits them expert by expert, sources in rank order inside an
// expert: local row  loc(e, s, i) = local_offsets[e - e0] + sum_{s' < s} n(s', e) + i,
// with n(s, e) = offsets_s[e + 1] - offsets_s[e].  perm_src_local[loc] = arrive
// and ret_idx[arrive] = loc.
#include <cstdint>
#include <vector>

#include "ftmoe.h"

namespace ftmoe {
void set_last_error(const char* msg);
}

extern "C" int ft_ep_plan(const int32_t* all_offsets, int G, int E, int rank, int32_t* send_rows,
                          int32_t* recv_rows, int32_t* local_offsets, int32_t* perm_src_local, int32_t* ret_idx,
                          int cap, int32_t* n_recv) {
  using ftmoe::set_last_error;
  if (G < 1 || E < 1 || E % G || rank < 0 || rank >= G) {
    set_last_error("ft_ep_plan: need G >= 1, E a multiple of G and 0 <= rank < G");
    return FT_ERR_INVALID_ARG;
  }
  if (!all_offsets || !send_rows || !recv_rows || !local_offsets || !n_recv ||
      (perm_src_local == nullptr) != (ret_idx == nullptr) || cap < 0) {
    set_last_error("ft_ep_plan: null pointer (perm_src_local and ret_idx are NULL together or not at all)");
    return FT_ERR_INVALID_ARG;
  }
  const int El = E / G;
  auto off = [&](int s, int e) -> int64_t { return all_offsets[int64_t(s) * (E + 1) + e]; };
  for (int s = 0; s < G; ++s) {
    if (off(s, 0) != 0) {
      set_last_error("ft_ep_plan: an offsets row does not start at 0");
      return FT_ERR_INVALID_ARG;
    }
    for (int e = 0; e < E; ++e)
      if (off(s, e + 1) < off(s, e)) {
        set_last_error("ft_ep_plan: an offsets row decreases");
        return FT_ERR_INVALID_ARG;
      }
  }
  const int e0 = rank * El, e1 = e0 + El;
  for (int d = 0; d < G; ++d) send_rows[d] = int32_t(off(rank, (d + 1) * El) - off(rank, d * El));
  int64_t total = 0;
  std::vector<int64_t> base(G);
  for (int s = 0; s < G; ++s) {
    base[s] = total;
    recv_rows[s] = int32_t(off(s, e1) - off(s, e0));
    total += recv_rows[s];
  }
  if (total > INT32_MAX) {
    set_last_error("ft_ep_plan: more than 2^31 - 1 rows received");
    return FT_ERR_INVALID_ARG;
  }
  *n_recv = int32_t(total);
  int64_t acc = 0;
  for (int e = e0; e < e1; ++e) {
    local_offsets[e - e0] = int32_t(acc);
    for (int s = 0; s < G; ++s) acc += off(s, e + 1) - off(s, e);
  }
  local_offsets[El] = int32_t(acc);
  if (!perm_src_local) return FT_OK;
  if (total > cap) {
    set_last_error("ft_ep_plan: more rows received than cap");
    return FT_ERR_INVALID_ARG;
  }
  int64_t loc = 0;
  for (int e = e0; e < e1; ++e)
    for (int s = 0; s < G; ++s) {
      const int64_t n = off(s, e + 1) - off(s, e);
      const int64_t a0 = base[s] + off(s, e) - off(s, e0);
      for (int64_t i = 0; i < n; ++i, ++loc) {
        perm_src_local[loc] = int32_t(a0 + i);
        ret_idx[a0 + i] = int32_t(loc);
      }
    }
  return FT_OK;
}
