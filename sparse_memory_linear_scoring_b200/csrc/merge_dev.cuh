// merge_dev.cuh -- warp-level product-key merge (staircase candidates, exact
// tie handling, quickselect, softmax weights) shared by the merge kernel and
// the single-step kernel.
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central" item 2: the
// top-W write slots (from k') and top-R read slots (from q') are the best of
// the k x k outer-sum candidates of the two halves' top-k lists,
//   topk(s1 (+) s2) = topk(topk(s1) (+) topk(s2)),   slot = i1 * n + i2,
// ordered by (float32 sum descending, slot ascending); w = softmax over the
// selected scores.  See merge_plan.cu for the staircase and its exactness.
#pragma once

#include "sdm_internal.cuh"

namespace sdm {

constexpr uint32_t kEmpty = 0xffffffffu;
constexpr uint32_t kInvalid = 0xffffffffu;

// A sorted half-list entry in shared memory: the float32 score's bits in the
// high word, the codebook row in the low word (only read back, never ordered
// as an integer).
__device__ __forceinline__ float hval(uint64_t e) { return __uint_as_float(uint32_t(e >> 32)); }
__device__ __forceinline__ uint32_t hrow(uint64_t e) { return uint32_t(e); }

__host__ __device__ inline int p2(int x) {
  int p = 2;
  while (p < x) p <<= 1;
  return p;
}

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~size_t(15); }

// k_merge: staircase tables, then per warp: two sorted half lists (h1, h2),
// the selection, the candidate scores and cells, and two select buffers.
struct MergeLayout {
  size_t stair, uni, total, per_warp;
  int Sk, Sc, Ss, warps;
};

__host__ __device__ inline MergeLayout merge_layout(const Plan& p, int warps) {
  MergeLayout L;
  L.Sk = p2(p.k);
  L.Sc = ((p.ncW > p.ncR ? p.ncW : p.ncR) + 31) & ~31;
  L.Ss = p2(p.W > p.R ? p.W : p.R);
  if (L.Ss < 32) L.Ss = 32;  // the register sort of the selection takes 32 keys at least
  L.warps = warps;
  size_t o = 0;
  L.stair = o; o = al16(o + size_t(p.ncW + p.nfW + p.ncR + p.nfR + 2 * p.k) * 4);
  L.uni = o;
  // h1, h2 [Sk], sel [Ss] (64-bit); cand, cell [Sc], select scratch [2 Sc],
  // bucket counts [64] (32-bit)
  L.per_warp = size_t(2 * L.Sk + L.Ss) * 8 + size_t(4 * L.Sc + 64) * 4;
  o += L.per_warp * warps;
  L.total = al16(o);
  return L;
}

// ------------------------------------------------------------------ merge (warp)
// Exact top-n_sel of all k*k candidates by a bitwise search over the 64-bit
// keys, counting by enumeration.  Used only when the staircase is not provably
// sufficient.  Leaves the n_sel best keys, descending, in cand[0..n_sel).
__device__ inline void merge_full(const uint64_t* h1, const uint64_t* h2, int k, int n, int n_sel,
                           uint64_t* cand) {
  const int lane = threadIdx.x & 31;
  const int kk = k * k;
  uint64_t prefix = 0;
  for (int bit = 63; bit >= 0; --bit) {
    const uint64_t probe = prefix | (uint64_t(1) << bit);
    int cnt = 0;
    for (int i = lane; i < kk; i += 32) {
      const int a = i / k, b = i - a * k;
      const float v = hval(h1[a]) + hval(h2[b]);
      const uint32_t slot = hrow(h1[a]) * uint32_t(n) + hrow(h2[b]);
      cnt += make_key(v, slot) >= probe;
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= n_sel) prefix = probe;
  }
  // prefix is the n_sel-th largest key; gather the keys >= prefix (exactly n_sel)
  int base = 0;
  for (int i0 = 0; i0 < kk; i0 += 32) {
    const int i = i0 + lane;
    uint64_t key = 0;
    bool take = false;
    if (i < kk) {
      const int a = i / k, b = i - a * k;
      const float v = hval(h1[a]) + hval(h2[b]);
      const uint32_t slot = hrow(h1[a]) * uint32_t(n) + hrow(h2[b]);
      key = make_key(v, slot);
      take = key >= prefix;
    }
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (take) cand[base + __popc(m & ((1u << lane) - 1u))] = key;
    base += __popc(m);
  }
  __syncwarp();
  const int S = p2(n_sel);
  for (int i = n_sel + lane; i < S; i += 32) cand[i] = 0;
  __syncwarp();
  warp_sort_desc(cand, S);
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Descending bitonic sort of one 64-bit key per lane across the warp.
__device__ __forceinline__ uint64_t warp_sort32_desc(uint64_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t y = __shfl_xor_sync(0xffffffffu, x, stride);
      const bool desc = (lane & size) == 0 || size == 32;
      const bool lower = (lane & stride) == 0;
      x = (lower == desc) ? (x > y ? x : y) : (x < y ? x : y);
    }
  }
  return x;
}

// Descending bitonic sort of one 32-bit key per lane across the warp.
__device__ __forceinline__ uint32_t warp_sort32_desc_u32(uint32_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint32_t y = __shfl_xor_sync(0xffffffffu, x, stride);
      const bool desc = (lane & size) == 0 || size == 32;
      const bool lower = (lane & stride) == 0;
      x = (lower == desc) ? max(x, y) : min(x, y);
    }
  }
  return x;
}

// Descending bitonic sort of 32 NJ 64-bit keys a[0..32 NJ) by one warp, in
// registers: element j*32 + lane is lane's x[j]; partners 32 or more apart
// are in the same lane, nearer ones are exchanged by shuffles.
template <int NJ>
__device__ inline void warp_sort_desc_reg(uint64_t* a) {
  const int lane = threadIdx.x & 31;
  constexpr int S = NJ * 32;
  uint64_t x[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) x[j] = a[j * 32 + lane];
#pragma unroll
  for (int size = 2; size <= S; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32) {
        const int js = stride / 32;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          if ((j & js) == 0) {
            const bool desc = ((j * 32 + lane) & size) == 0;
            const uint64_t lo = x[j], hi = x[j + js];
            if (desc ? (lo < hi) : (lo > hi)) {
              x[j] = hi;
              x[j + js] = lo;
            }
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const uint64_t y = __shfl_xor_sync(0xffffffffu, x[j], stride);
          const bool desc = ((j * 32 + lane) & size) == 0;
          const bool lower = (lane & stride) == 0;
          x[j] = (lower == desc) ? (x[j] > y ? x[j] : y) : (x[j] < y ? x[j] : y);
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < NJ; ++j) a[j * 32 + lane] = x[j];
}

// Ascending bitonic sort of S (power of two) 32-bit keys in shared memory by
// one warp.
__device__ inline void warp_sort_asc_u32(uint32_t* a, int S) {
  const int lane = threadIdx.x & 31;
  for (int size = 2; size <= S; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < (S >> 1); i += 32) {
        const int lo = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));
        const int hi = lo + stride;
        const uint32_t x = a[lo], y = a[hi];
        const bool asc = (lo & size) == 0;
        if (asc ? (x > y) : (x < y)) { a[lo] = y; a[hi] = x; }
      }
      __syncwarp();
    }
  }
}

// The r-th largest (1-based, counting repeats) of the n values in cand[]
// (left intact): quickselect with median-of-3 pivots and a three-way split;
// each round moves the values above / below the pivot into a scratch buffer
// (A and B alternate, each of capacity >= n); at <= 32 values a warp sort
// finishes.
__device__ inline uint32_t warp_select32(const uint32_t* cand, int n, int r, uint32_t* A, uint32_t* B) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = lanemask_lt();
  const uint32_t* src = cand;
  int which = 0;
  for (int iter = 0; iter < 4096; ++iter) {
    if (n <= 32) {
      uint32_t x = lane < n ? src[lane] : 0u;
      __syncwarp();
      x = warp_sort32_desc_u32(x);
      return __shfl_sync(0xffffffffu, x, r - 1);
    }
    const uint32_t a = src[0], b = src[n >> 1], c = src[n - 1];
    const uint32_t piv = max(min(a, b), min(max(a, b), c));
    uint32_t* dst = which ? B : A;
    int front = 0, back = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t x = i < n ? src[i] : 0u;
      const bool gt = (i < n) && x > piv;
      const bool ls = (i < n) && x < piv;
      const unsigned mg = __ballot_sync(0xffffffffu, gt);
      const unsigned ml = __ballot_sync(0xffffffffu, ls);
      if (gt) dst[front + __popc(mg & lt_mask)] = x;
      if (ls) dst[n - 1 - (back + __popc(ml & lt_mask))] = x;
      front += __popc(mg);
      back += __popc(ml);
    }
    __syncwarp();
    const int eq = n - front - back;
    if (r <= front) {
      src = dst;
      n = front;
    } else if (r <= front + eq) {
      return piv;
    } else {
      src = dst + (n - back);
      n = back;
      r -= front + eq;
    }
    which ^= 1;
  }
  return 0u;  // not reached: each round removes at least the pivot's value
}

// Merge of one (step, side): sorted half lists (first k entries of each
// survivor list) -> the n_sel selected slots and their softmax weights.
// Selection order is unspecified unless `sorted` is set (then rank order).
// With sv1 == sv2 == nullptr the lists are already in h1, h2.
__device__ inline void merge_one(const Plan& p, const uint2* sv1, int c1, const uint2* sv2, int c2,
                          int n_sel, const uint32_t* stair, int n_stair, const uint32_t* front,
                          int nf, const int* ediv, uint64_t* h1, uint64_t* h2, uint32_t* cand, uint32_t* cell,
                          uint32_t* alt, int* hist, uint64_t* sel, bool sorted, float* w_out,
                          uint32_t* slot_out, DevStatus* st, int info, bool sigmoid_w = false) {
  const int lane = threadIdx.x & 31;
  if (c1 < p.k || c1 > p.C || c2 < p.k || c2 > p.C) {
    if (lane == 0) dev_flag(st, SDM_DEV_CAPACITY, info);
    for (int i = lane; i < n_sel; i += 32) { w_out[i] = 0.f; slot_out[i] = kInvalid; }
    __syncwarp();
    return;
  }
  if (sv1 != nullptr) {  // else the caller has staged the lists in h1, h2
    for (int i = lane; i < p.k; i += 32) {
      const uint2 a = sv1[i], b = sv2[i];
      h1[i] = (uint64_t(a.x) << 32) | a.y;
      h2[i] = (uint64_t(b.x) << 32) | b.y;
    }
  }
  __syncwarp();
  const uint32_t n = uint32_t(p.n);
  // A lower bound on the n_sel-th best candidate: all d * e >= n_sel cells of
  // the d x e corner score at least s1[d-1] + s2[e-1] (sums fall along rows and
  // columns, and float32 addition is monotone).
  uint32_t lb = 0;
  for (int d = lane + 1; d <= p.k; d += 32) {
    const int e = ediv[d - 1];  // ceil(n_sel / d)
    if (e <= p.k) lb = max(lb, f2ord(hval(h1[d - 1]) + hval(h2[e - 1])));
  }
  lb = __reduce_max_sync(0xffffffffu, lb);
  // candidates: the staircase cells scoring >= lb (ordered 32-bit images of the
  // float32 sums) and their cells; they include every staircase cell that
  // scores >= the n_sel-th best, so nc >= n_sel.  Each is also counted into one
  // of 64 buckets of [lb, hi] (hi: cell (0, 0), the best), bucket 0 the highest.
  const uint32_t hi = f2ord(hval(h1[0]) + hval(h2[0]));
  const int nbits = 32 - __clz(hi - lb);  // hi - lb < 2^nbits
  const int sh = nbits > 6 ? nbits - 6 : 0;
  hist[lane] = 0;
  hist[lane + 32] = 0;
  __syncwarp();
  int nc = 0;
  // two groups of 32 cells per trip, their loads issued together
  for (int i0 = 0; i0 < n_stair; i0 += 64) {
    uint32_t x[2] = {0u, 0u}, ab[2] = {0u, 0u};
    bool keep[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + 32 * u + lane;
      if (i < n_stair) ab[u] = stair[i];
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + 32 * u + lane;
      if (i < n_stair) x[u] = f2ord(hval(h1[ab[u] & 0xffff]) + hval(h2[ab[u] >> 16]));
      keep[u] = i < n_stair && x[u] >= lb;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const unsigned m = __ballot_sync(0xffffffffu, keep[u]);
      if (keep[u]) {
        const int pos = nc + __popc(m & lanemask_lt());
        cand[pos] = x[u];
        cell[pos] = ab[u];
        atomicAdd(&hist[(hi - x[u]) >> sh], 1);
      }
      nc += __popc(m);
    }
  }
  __syncwarp();
  // the n_sel-th best: a warp scan of the bucket counts finds the bucket kb
  // that holds it and its rank r there; a bucket of at most 32 entries is
  // sorted across the warp, a larger one (crowded scores) goes to quickselect
  uint32_t vstar;
  int n_gt = 0, n_eq = 0;  // candidates above / equal to vstar
  bool counted = false;
  {
    const int c0 = hist[2 * lane], c1 = hist[2 * lane + 1];
    int incl = c0 + c1;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += y;
    }
    const int s0 = incl - c0 - c1, s1 = s0 + c0;
    const int lk = __ffs(__ballot_sync(0xffffffffu, incl >= n_sel)) - 1;
    const int odd = __shfl_sync(0xffffffffu, s1 >= n_sel ? 0 : 1, lk);
    const uint32_t kb = uint32_t(2 * lk + odd);
    const int kb0 = __shfl_sync(0xffffffffu, odd ? s1 : s0, lk);
    const int kb1 = __shfl_sync(0xffffffffu, odd ? incl : s1, lk);
    if (kb1 - kb0 <= 32) {
      int nb = 0;
      for (int i0 = 0; i0 < nc; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t x = i < nc ? cand[i] : 0u;
        const bool in = i < nc && ((hi - x) >> sh) == kb;
        const unsigned m = __ballot_sync(0xffffffffu, in);
        if (in) alt[nb + __popc(m & lanemask_lt())] = x;
        nb += __popc(m);
      }
      __syncwarp();
      const bool live = lane < kb1 - kb0;  // the sorted bucket fills lanes 0..m-1
      uint32_t y = live ? alt[lane] : 0u;
      y = warp_sort32_desc_u32(y);
      vstar = __shfl_sync(0xffffffffu, y, n_sel - kb0 - 1);
      // the buckets before kb hold only candidates above vstar, those after it
      // only candidates below; in kb, count from the sorted values
      n_gt = kb0 + __popc(__ballot_sync(0xffffffffu, live && y > vstar));
      n_eq = __popc(__ballot_sync(0xffffffffu, live && y == vstar));
      counted = true;
      __syncwarp();
    } else {
      vstar = warp_select32(cand, nc, n_sel, alt, alt + (nc + 31) / 32 * 32);
    }
  }
  // exact when every candidate outside the staircase scores strictly below the
  // n_sel-th and no other candidate ties it
  if (!counted) {
    for (int i = lane; i < nc; i += 32) {
      const uint32_t x = cand[i];
      n_gt += x > vstar;
      n_eq += x == vstar;
    }
    n_gt = __reduce_add_sync(0xffffffffu, n_gt);
    n_eq = __reduce_add_sync(0xffffffffu, n_eq);
  }
  bool bad = false;
  for (int i = lane; i < nf; i += 32) {
    const uint32_t ab = front[i];
    bad |= f2ord(hval(h1[ab & 0xffff]) + hval(h2[ab >> 16])) >= vstar;
  }
  bool is_sorted = false;
  if (__any_sync(0xffffffffu, bad) || n_gt + n_eq != n_sel) {
    // Ties at vstar.  Every candidate outside the staircase is dominated by at
    // least n_sel staircase candidates, so it scores <= vstar: the selection is
    // the n_gt staircase candidates above vstar plus the lowest slots among all
    // k*k candidates equal to vstar.
    const int kk = p.k * p.k;
    int tcap = 1;  // largest power of two that fits the scratch (2 * Sc entries)
    while (2 * tcap <= 2 * (((p.ncW > p.ncR ? p.ncW : p.ncR) + 31) & ~31)) tcap *= 2;
    int n_tie = 0;
    for (int i0 = 0; i0 < kk; i0 += 32) {
      const int i = i0 + lane;
      bool tie = false;
      uint32_t slot = 0;
      if (i < kk) {
        const int a = i / p.k, b = i - a * p.k;
        tie = f2ord(hval(h1[a]) + hval(h2[b])) == vstar;
        slot = hrow(h1[a]) * n + hrow(h2[b]);
      }
      const unsigned m = __ballot_sync(0xffffffffu, tie);
      const int pos = n_tie + __popc(m & lanemask_lt());
      if (tie && pos < tcap) alt[pos] = slot;
      n_tie += __popc(m);
    }
    __syncwarp();
    if (n_tie > tcap) {
      merge_full(h1, h2, p.k, p.n, n_sel, sel);  // pathological ties only
      is_sorted = true;
    } else {
      const int S = p2(n_tie);
      for (int i = n_tie + lane; i < S; i += 32) alt[i] = 0xffffffffu;
      __syncwarp();
      warp_sort_asc_u32(alt, S);
      int base = 0;
      for (int i0 = 0; i0 < nc; i0 += 32) {
        const int i = i0 + lane;
        const bool take = (i < nc) && cand[i] > vstar;
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (take) {
          const uint32_t ab = cell[i];
          const uint64_t a = h1[ab & 0xffff], b = h2[ab >> 16];
          sel[base + __popc(m & lanemask_lt())] =
              (uint64_t(cand[i]) << 32) | uint64_t(~(hrow(a) * n + hrow(b)));
        }
        base += __popc(m);
      }
      for (int j = lane; j < n_sel - base; j += 32)
        sel[base + j] = (uint64_t(vstar) << 32) | uint64_t(~alt[j]);
    }
  } else {
    int base = 0;
    for (int i0 = 0; i0 < nc; i0 += 32) {
      const int i = i0 + lane;
      const bool take = (i < nc) && cand[i] >= vstar;
      const unsigned m = __ballot_sync(0xffffffffu, take);
      if (take) {
        const uint32_t ab = cell[i];
        const uint64_t a = h1[ab & 0xffff], b = h2[ab >> 16];
        sel[base + __popc(m & lanemask_lt())] =
            (uint64_t(cand[i]) << 32) | uint64_t(~(hrow(a) * n + hrow(b)));
      }
      base += __popc(m);
    }
  }
  __syncwarp();
  if (sorted && !is_sorted) {
    const int S = p2(n_sel) < 32 ? 32 : p2(n_sel);
    for (int i = n_sel + lane; i < S; i += 32) sel[i] = 0;
    __syncwarp();
    if (S == 32) warp_sort_desc_reg<1>(sel);
    else if (S == 64) warp_sort_desc_reg<2>(sel);
    else if (S == 128) warp_sort_desc_reg<4>(sel);
    else warp_sort_desc(sel, S);
    __syncwarp();
  }
  // softmax over the selected float32 scores (the best candidate is (0, 0));
  // with sigmoid_w, the router weights of the selective-decay rule instead:
  // sigmoid of each selected score, normalised to sum 1
  const float m = hval(h1[0]) + hval(h2[0]);
  float* ex = reinterpret_cast<float*>(cand);  // free again (n_sel <= Sc)
  float zs = 0.f;
  for (int i = lane; i < n_sel; i += 32) {
    const float s = key_val(sel[i]);
    const float e = sigmoid_w ? 1.f / (1.f + expf(-s)) : expf(s - m);
    ex[i] = e;
    zs += e;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, off);
  const float inv = 1.f / zs;
  for (int i = lane; i < n_sel; i += 32) {
    w_out[i] = ex[i] * inv;
    slot_out[i] = key_idx(sel[i]);
  }
  __syncwarp();
}

// Staircase rows a < k with bm(a) = min(k, n_sel / (a+1)) columns, and the
// frontier cell (a, bm(a)) of each row that stops short of k (rows past the
// last non-empty one contribute only their first empty cell); and, for the
// corner lower bound, ediv[d-1] = ceil(n_sel / d) for d = 1..k.  One warp.
__device__ inline void build_staircase(int k, int n_sel, uint32_t* stair, uint32_t* front,
                                       int* ediv) {
  const int lane = threadIdx.x & 31;
  for (int d = lane + 1; d <= k; d += 32) ediv[d - 1] = (n_sel + d - 1) / d;  // ceil(n_sel / d)
  int obase = 0, fbase = 0, prev_last = -1;
  for (int a0 = 0; a0 < k; a0 += 32) {
    const int a = a0 + lane;
    const int bm = a < k ? min(k, n_sel / (a + 1)) : 0;
    const int prev = __shfl_up_sync(0xffffffffu, bm, 1);
    const int pbm = lane == 0 ? prev_last : prev;
    const bool fr = a < k && bm < k && !(bm == 0 && pbm == 0);
    int incl = bm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned fm = __ballot_sync(0xffffffffu, fr);
    const int start = obase + incl - bm;
    for (int b = 0; b < bm; ++b) stair[start + b] = uint32_t(a) | (uint32_t(b) << 16);
    if (fr) front[fbase + __popc(fm & lanemask_lt())] = uint32_t(a) | (uint32_t(bm) << 16);
    obase += __shfl_sync(0xffffffffu, incl, 31);
    fbase += __popc(fm);
    prev_last = __shfl_sync(0xffffffffu, bm, 31);
  }
}

}  // namespace sdm
