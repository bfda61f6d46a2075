// select_dev.cuh -- warp-level exact top-k of (score, row) pairs held in
// registers, used by the tensor-core scoring epilogue and the survivor top-k
// kernel.
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

// Scratch of warp_bucket_topk per warp: kSelBuckets words (bucket start << 16
// | cursor), then the staged 64-bit keys.
#ifndef SDM_SEL_BUCKETS
#define SDM_SEL_BUCKETS 128
#endif
constexpr int kSelBuckets = SDM_SEL_BUCKETS;
static_assert(kSelBuckets == 64 || kSelBuckets == 128 || kSelBuckets == 256,
              "64, 128 or 256 buckets");
constexpr int kSelHeadBytes = kSelBuckets * 4;

// The k best of the c valid (key, row) entries held PL per lane (entry i*32 + l
// in lane l; 1 <= k <= c <= 65535; rows distinct), written to out[0..k) in (key
// desc, row asc) order as (value bits, row) pairs, value = ord2f(key).
//   1. The keys are counted into kSelBuckets buckets of the key range, bucket 0
//      holding the largest (bucket = (max - key) >> shift, monotone in the
//      key); each lane owns kSelBuckets / 32 consecutive buckets.
//   2. A warp scan of the counts gives every bucket's start in the output
//      order and the bucket kb that holds the k-th largest.
//   3. The entries of buckets 0..kb are staged, grouped by bucket.
//   4. An entry's rank is its bucket's start plus the number of staged entries
//      of its bucket that precede it; ranks below k are final positions.  The
//      lanes take the staged entries in turn, so the bucket walks scale with
//      the staged count, not with the entries each lane held.
// A bucket holds a few entries unless the keys crowd together, so the rank
// loops are short.  Returns false, writing nothing, if more than `cap` entries
// would be staged (the caller then takes another path).
template <int PL>
__device__ __forceinline__ bool warp_bucket_topk(const uint32_t (&key)[PL],
                                                 const uint32_t (&row)[PL], int c, int k,
                                                 uint32_t* bkt, uint64_t* stage, int cap,
                                                 uint2* out) {
  constexpr int BPL = kSelBuckets / 32;  // buckets per lane
  constexpr int LOGB = kSelBuckets == 64 ? 6 : (kSelBuckets == 128 ? 7 : 8);
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
  const int nbits = 32 - __clz(hi - lo);  // hi - lo < 2^nbits
  const int sh = nbits > LOGB ? nbits - LOGB : 0;
  uint32_t* mine = bkt + lane * BPL;
#pragma unroll
  for (int j = 0; j < BPL; ++j) mine[j] = 0u;
  __syncwarp();
  int b[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    b[i] = i * 32 + lane < c ? int((hi - key[i]) >> sh) : kSelBuckets;
    if (b[i] < kSelBuckets) atomicAdd(&bkt[b[i]], 1u);
  }
  __syncwarp();
  // the lane's buckets: counts and running sums, then the warp scan of the totals
  int cnt[BPL], run[BPL];
  int tot = 0;
#pragma unroll
  for (int j = 0; j < BPL; ++j) {
    cnt[j] = int(mine[j]);
    tot += cnt[j];
    run[j] = tot;
  }
  int incl = tot;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += y;
  }
  const int excl = incl - tot;
  // kb: the first bucket whose end reaches k (lane 31's last end is c >= k)
  int myj = BPL, myend = 0;
#pragma unroll
  for (int j = BPL - 1; j >= 0; --j) {
    if (excl + run[j] >= k) {
      myj = j;
      myend = excl + run[j];
    }
  }
  const int lk = __ffs(__ballot_sync(0xffffffffu, myj < BPL)) - 1;
  const int kb = lk * BPL + __shfl_sync(0xffffffffu, myj, lk);
  const int nst = __shfl_sync(0xffffffffu, myend, lk);  // end of bucket kb
  if (nst > cap) return false;
  __syncwarp();
#pragma unroll
  for (int j = 0; j < BPL; ++j) {
    const uint32_t st = uint32_t(excl + run[j] - cnt[j]);
    mine[j] = (st << 16) | st;  // start, cursor
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    if (b[i] <= kb) {
      const int pos = int(atomicAdd(&bkt[b[i]], 1u) & 0xffffu);
      stage[pos] = (uint64_t(key[i]) << 32) | uint64_t(~row[i]);
    }
  }
  __syncwarp();
  // ranks, by staged position (at most ceil(cap / 32) per lane), so that the
  // warp walks only the buckets of staged entries
  for (int q = lane; q < nst; q += 32) {
    const uint64_t me = stage[q];
    const uint32_t mk = uint32_t(me >> 32);
    const uint32_t w = bkt[(hi - mk) >> sh];
    const int bs = int(w >> 16), be = int(w & 0xffffu);
    int rank = bs;
    for (int j = bs; j < be; ++j) rank += stage[j] > me ? 1 : 0;
    if (rank < k) out[rank] = make_uint2(__float_as_uint(ord2f(mk)), ~uint32_t(me));
  }
  return true;
}

}  // namespace sdm
