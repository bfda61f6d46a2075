// select_dev.cuh -- warp-level exact top-k of (score, row) pairs held in
// registers, used by the survivor top-k kernel and the single-step kernel.
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central" item 2: each
// half keeps its top-k codebook rows, ordered by (score desc, row asc).  The
// scores are compared through their order-preserving 32-bit images (f2ord), so
// the k-th largest is found by a bitwise search over those images.
#pragma once

#include "sdm_internal.cuh"

namespace sdm {

// The k-th largest (1-based, counting repeats) of the c valid 32-bit keys held
// PL per lane across the warp (key i of lane l is entry i*32 + l; entries
// >= c are not valid; 1 <= k <= c).  Most significant bit first, starting
// below the leading bits that every valid key shares.
template <int PL>
__device__ __forceinline__ uint32_t warp_kth_key(const uint32_t (&key)[PL], int c, int k) {
  const int lane = threadIdx.x & 31;
  uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    if (i * 32 + lane < c) {
      lo = min(lo, key[i]);
      hi = max(hi, key[i]);
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  const uint32_t diff = lo ^ hi;
  if (diff == 0u) return hi;  // every key equal
  const int top = 31 - __clz(diff);
  // every key lies in [thr, thr + 2^(top+1)), so at least c >= k are >= thr
  uint32_t thr = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t cand = thr | (1u << bit);
    int n = 0;
#pragma unroll
    for (int i = 0; i < PL; ++i) n += (i * 32 + lane < c && key[i] >= cand) ? 1 : 0;
    if (__reduce_add_sync(0xffffffffu, n) >= k) thr = cand;
  }
  return thr;
}

// The k best of the c valid (key, row) entries, in no particular order, as
// 64-bit keys (key << 32 | ~row: larger is better, lower row wins a tie) in
// out[0..k).  thr is warp_kth_key(key, c, k).  Rows are distinct.  Entries
// above thr are all taken; of the entries equal to thr, the lowest rows.
template <int PL>
__device__ __forceinline__ void warp_gather_topk(const uint32_t (&key)[PL],
                                                 const uint32_t (&row)[PL], int c, int k,
                                                 uint32_t thr, uint64_t* out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int n_gt = 0, n_eq = 0;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const bool v = i * 32 + lane < c;
    n_gt += (v && key[i] > thr) ? 1 : 0;
    n_eq += (v && key[i] == thr) ? 1 : 0;
  }
  n_gt = __reduce_add_sync(0xffffffffu, n_gt);
  n_eq = __reduce_add_sync(0xffffffffu, n_eq);
  const int m = k - n_gt;  // ties to take, 1 <= m <= n_eq
  // the m-th smallest row among the ties (all of them when m == n_eq)
  uint32_t rmax = 0xffffffffu;
  if (m < n_eq) {
    uint32_t r = 0u;  // smallest R with #(tie, row <= R) >= m, bit by bit
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = r | ((1u << bit) - 1u);  // rows <= cand with this prefix
      int n = 0;
#pragma unroll
      for (int i = 0; i < PL; ++i)
        n += (i * 32 + lane < c && key[i] == thr && row[i] <= cand) ? 1 : 0;
      if (__reduce_add_sync(0xffffffffu, n) < m) r |= 1u << bit;
    }
    rmax = r;
  }
  int base = 0;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const bool v = i * 32 + lane < c;
    const bool take = v && (key[i] > thr || (key[i] == thr && row[i] <= rmax));
    const unsigned mk = __ballot_sync(0xffffffffu, take);
    if (take) out[base + __popc(mk & lt)] = (uint64_t(key[i]) << 32) | uint64_t(~row[i]);
    base += __popc(mk);
  }
}

}  // namespace sdm
