// merge_plan.cu -- product-key merge, softmax weights, and the recurrence plan.
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central" item 2: the top-W
// write slots (from k') and top-R read slots (from q') are the best of the k x k
// outer-sum candidates of the two halves' top-k lists,
//   topk(s1 (+) s2) = topk(topk(s1) (+) topk(s2)),   slot = i1 * n + i2,
// ordered by (float32 sum descending, slot ascending).  Item 3 weights: w =
// softmax over the W selected write scores, u = softmax over the R read scores.
//
// Merge (one warp per (step, side)): the half lists arrive sorted; evaluate the
// "staircase" candidates (a, b) with (a+1)(b+1) <= n_sel (a, b = ranks in the
// two halves) and select the n_sel best by quickselect.  This is exact when every
// candidate outside the staircase scores strictly below the n_sel-th: the
// largest outside score is attained on the staircase's frontier (row a, column
// bmax(a)), since sums fall along each row; if the frontier check fails, an
// exact search over all k x k candidates runs instead.
//
// The merge kernel writes the lists (slot, weight) of every step; the plan
// kernel reads them back (or a caller's lists) and builds the recurrence plan.
//
// Plan (one CTA per (head, block of P steps)): the block's W+R entries per
// step become records for the recurrence, ordered by (bucket, slot, entry).
// A slot's bucket is a hash of the slot into the head's NB buckets, the same in
// every block, and recurrence stream s owns buckets [s*mb, (s+1)*mb); so every
// record of a slot, in every block, goes to the same stream, and within a
// bucket a slot's records are adjacent and in time order (entry order puts a
// step's write before its read).  A record is
//   int4 {slot, (step_in_chunk << 1) | is_read, f1, f2}
// with, for a write, f1 = alpha_t * (1 - c), f2 = c = beta_t * w_i (the update
// is then M = f1 * M + f2 * v_t); for a read, f1 = u_r.  The per-(head, block)
// bucket starts (NB + 1 of them) go to roff.
#include "sdm_internal.cuh"

namespace sdm {

constexpr uint32_t kEmpty = 0xffffffffu;
constexpr uint32_t kInvalid = 0xffffffffu;

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
  L.warps = warps;
  size_t o = 0;
  L.stair = o; o = al16(o + size_t(p.ncW + p.nfW + p.ncR + p.nfR) * 4);
  L.uni = o;
  // h1, h2 [Sk], sel [Ss] (64-bit); cand, cell [Sc], select scratch [2 Sc] (32-bit)
  L.per_warp = size_t(2 * L.Sk + L.Ss) * 8 + size_t(4 * L.Sc) * 4;
  o += L.per_warp * warps;
  L.total = al16(o);
  return L;
}

size_t merge_smem_bytes(const Plan& p, int warps) { return merge_layout(p, warps).total; }

// k_plan: the block's sort keys (bucket, slot, entry) and the bucket counts /
// starts and running positions.
struct PlanLayout {
  size_t key, cnt, total;
};

__host__ __device__ inline PlanLayout plan_layout(const Plan& p) {
  PlanLayout L;
  size_t o = 0;
  L.key = o; o = al16(o + size_t(p.E) * 8);
  L.cnt = o; o = al16(o + size_t(2 * p.NB + 2) * 4);
  L.total = o;
  return L;
}

size_t plan_smem_bytes(const Plan& p) { return plan_layout(p).total; }

// ------------------------------------------------------------------ merge (warp)
// Exact top-n_sel of all k*k candidates by a bitwise search over the 64-bit
// keys, counting by enumeration.  Used only when the staircase is not provably
// sufficient.  Leaves the n_sel best keys, descending, in cand[0..n_sel).
__device__ void merge_full(const uint64_t* h1, const uint64_t* h2, int k, int n, int n_sel,
                           uint64_t* cand) {
  const int lane = threadIdx.x & 31;
  const int kk = k * k;
  uint64_t prefix = 0;
  for (int bit = 63; bit >= 0; --bit) {
    const uint64_t probe = prefix | (uint64_t(1) << bit);
    int cnt = 0;
    for (int i = lane; i < kk; i += 32) {
      const int a = i / k, b = i - a * k;
      const float v = key_val(h1[a]) + key_val(h2[b]);
      const uint32_t slot = key_idx(h1[a]) * uint32_t(n) + key_idx(h2[b]);
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
      const float v = key_val(h1[a]) + key_val(h2[b]);
      const uint32_t slot = key_idx(h1[a]) * uint32_t(n) + key_idx(h2[b]);
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

// Ascending bitonic sort of S (power of two) 32-bit keys in shared memory by
// one warp.
__device__ void warp_sort_asc_u32(uint32_t* a, int S) {
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
__device__ uint32_t warp_select32(const uint32_t* cand, int n, int r, uint32_t* A, uint32_t* B) {
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
__device__ void merge_one(const Plan& p, const uint2* sv1, int c1, const uint2* sv2, int c2,
                          int n_sel, const uint32_t* stair, int n_stair, const uint32_t* front,
                          int nf, uint64_t* h1, uint64_t* h2, uint32_t* cand, uint32_t* cell,
                          uint32_t* alt, uint64_t* sel, bool sorted, float* w_out,
                          uint32_t* slot_out, DevStatus* st, int info) {
  const int lane = threadIdx.x & 31;
  if (c1 < p.k || c1 > p.C || c2 < p.k || c2 > p.C) {
    if (lane == 0) dev_flag(st, SDM_DEV_CAPACITY, info);
    for (int i = lane; i < n_sel; i += 32) { w_out[i] = 0.f; slot_out[i] = kInvalid; }
    __syncwarp();
    return;
  }
  for (int i = lane; i < p.k; i += 32) {
    const uint2 a = sv1[i], b = sv2[i];
    h1[i] = make_key(__uint_as_float(a.x), a.y);
    h2[i] = make_key(__uint_as_float(b.x), b.y);
  }
  __syncwarp();
  const uint32_t n = uint32_t(p.n);
  // A lower bound on the n_sel-th best candidate: all d * e >= n_sel cells of
  // the d x e corner score at least s1[d-1] + s2[e-1] (sums fall along rows and
  // columns, and float32 addition is monotone).
  uint32_t lb = 0;
  for (int d = lane + 1; d <= p.k; d += 32) {
    const int e = (n_sel + d - 1) / d;
    if (e <= p.k) lb = max(lb, f2ord(key_val(h1[d - 1]) + key_val(h2[e - 1])));
  }
  lb = __reduce_max_sync(0xffffffffu, lb);
  // candidates: the staircase cells scoring >= lb (ordered 32-bit images of the
  // float32 sums) and their cells; they include every staircase cell that
  // scores >= the n_sel-th best
  int nc = 0;
  for (int i0 = 0; i0 < n_stair; i0 += 32) {
    const int i = i0 + lane;
    uint32_t x = 0, ab = 0;
    if (i < n_stair) {
      ab = stair[i];
      x = f2ord(key_val(h1[ab & 0xffff]) + key_val(h2[ab >> 16]));
    }
    const bool keep = i < n_stair && x >= lb;
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int pos = nc + __popc(m & lanemask_lt());
      cand[pos] = x;
      cell[pos] = ab;
    }
    nc += __popc(m);
  }
  __syncwarp();
  const uint32_t vstar = warp_select32(cand, nc, n_sel, alt, alt + (nc + 31) / 32 * 32);
  // exact when every candidate outside the staircase scores strictly below the
  // n_sel-th and no other candidate ties it
  int n_gt = 0, n_eq = 0;
  for (int i = lane; i < nc; i += 32) {
    const uint32_t x = cand[i];
    n_gt += x > vstar;
    n_eq += x == vstar;
  }
  n_gt = __reduce_add_sync(0xffffffffu, n_gt);
  n_eq = __reduce_add_sync(0xffffffffu, n_eq);
  bool bad = false;
  for (int i = lane; i < nf; i += 32) {
    const uint32_t ab = front[i];
    bad |= f2ord(key_val(h1[ab & 0xffff]) + key_val(h2[ab >> 16])) >= vstar;
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
        tie = f2ord(key_val(h1[a]) + key_val(h2[b])) == vstar;
        slot = key_idx(h1[a]) * n + key_idx(h2[b]);
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
              (uint64_t(cand[i]) << 32) | uint64_t(~(key_idx(a) * n + key_idx(b)));
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
            (uint64_t(cand[i]) << 32) | uint64_t(~(key_idx(a) * n + key_idx(b)));
      }
      base += __popc(m);
    }
  }
  __syncwarp();
  if (sorted && !is_sorted) {
    const int S = p2(n_sel);
    for (int i = n_sel + lane; i < S; i += 32) sel[i] = 0;
    __syncwarp();
    warp_sort_desc(sel, S);
  }
  // softmax over the selected float32 scores; the best candidate is (0, 0)
  const float m = key_val(h1[0]) + key_val(h2[0]);
  float* ex = reinterpret_cast<float*>(cand);  // free again (n_sel <= Sc)
  float zs = 0.f;
  for (int i = lane; i < n_sel; i += 32) {
    const float e = expf(key_val(sel[i]) - m);
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

// ------------------------------------------------------------------ kernels
// Staircase rows a < k with bm(a) = min(k, n_sel / (a+1)) columns, and the
// frontier cell (a, bm(a)) of each row that stops short of k (rows past the
// last non-empty one contribute only their first empty cell).  One warp.
__device__ void build_staircase(int k, int n_sel, uint32_t* stair, uint32_t* front) {
  const int lane = threadIdx.x & 31;
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

// One CTA per (head, kMergeSteps steps); one warp per (step, side).  Writes
// the W write and R read (slot, weight) pairs of each step to the lists
// (row = bh * list_T + list_t0 + step), in rank order when `sorted`.
__global__ void __launch_bounds__(kMergeWarps * 32)
k_merge(Plan p, MergeIO io, int t0, int tlen, DevStatus* st) {
  extern __shared__ __align__(16) unsigned char smem[];
  const MergeLayout L = merge_layout(p, kMergeWarps);
  uint32_t* stairW = reinterpret_cast<uint32_t*>(smem + L.stair);
  uint32_t* frontW = stairW + p.ncW;
  uint32_t* stairR = frontW + p.nfW;
  uint32_t* frontR = stairR + p.ncR;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bh = blockIdx.y;
  const int s0 = blockIdx.x * kMergeSteps;
  if (s0 >= tlen) return;
  const int np = min(kMergeSteps, tlen - s0);
  if (warp == 0) build_staircase(p.k, p.W, stairW, frontW);
  if (warp == 1) build_staircase(p.k, p.R, stairR, frontR);
  __syncthreads();
  unsigned char* mine = smem + L.uni + L.per_warp * warp;
  uint64_t* h1 = reinterpret_cast<uint64_t*>(mine);
  uint64_t* h2 = h1 + L.Sk;
  uint64_t* sel = h2 + L.Sk;
  uint32_t* cand = reinterpret_cast<uint32_t*>(sel + L.Ss);
  uint32_t* cell = cand + L.Sc;
  uint32_t* alt = cell + L.Sc;
  for (int pi = warp; pi < 2 * np; pi += kMergeWarps) {
    const int tc = s0 + (pi >> 1), side = pi & 1;
    const size_t hr = (size_t(bh) * p.Tc + tc) * 4 + side * 2;
    const int n_sel = side ? p.R : p.W;
    const size_t row = size_t(bh) * io.list_T + io.list_t0 + tc;
    float* w_out = (side ? io.out_wr : io.out_ww) + row * n_sel;
    uint32_t* s_out = reinterpret_cast<uint32_t*>(side ? io.out_ir : io.out_iw) + row * n_sel;
    merge_one(p, io.surv + hr * p.C, io.surv_cnt[hr], io.surv + (hr + 1) * p.C,
              io.surv_cnt[hr + 1], n_sel, side ? stairR : stairW, side ? p.ncR : p.ncW,
              side ? frontR : frontW, side ? p.nfR : p.nfW, h1, h2, cand, cell, alt, sel,
              io.sorted != 0, w_out, s_out, st, int(hr));
  }
}

// One CTA per (head, block of P steps): sort the block's list entries into
// records by (bucket, slot, entry) (see the file header) and zero the block's
// rows of o.
__global__ void __launch_bounds__(kPlanThreads)
k_plan(Plan p, PlanIO io, int t0, int tlen, DevStatus* st) {
  extern __shared__ __align__(16) unsigned char smem[];
  const PlanLayout L = plan_layout(p);
  uint64_t* key = reinterpret_cast<uint64_t*>(smem + L.key);  // sorted by bucket
  int* start = reinterpret_cast<int*>(smem + L.cnt);          // [NB + 1] counts, then starts
  int* cur = start + p.NB + 1;                                 // [NB] running positions
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int WR = p.W + p.R;
  const int s0 = blk * p.P;
  if (s0 >= tlen) return;
  const int np = min(p.P, tlen - s0);
  const int nent = np * WR;
  const size_t lrow0 = size_t(bh) * io.list_T + io.list_t0 + s0;  // list row of step s0
  const size_t trow0 = size_t(bh) * p.T + t0 + s0;                 // time row of step s0
  // e / WR for e < 2^13 by a multiply-high (exact in that range)
  const uint32_t magic = 0xffffffffu / uint32_t(WR) + 1u;
  auto step_of = [&](int e) { return int(__umulhi(uint32_t(e), magic)); };
  auto slot_of = [&](int e) -> int32_t {
    const int tl = step_of(e), j = e - tl * WR;
    return j < p.W ? io.iw[(lrow0 + tl) * p.W + j] : io.ir[(lrow0 + tl) * p.R + (j - p.W)];
  };
  auto in_range = [&](int32_t s) { return s >= 0 && (long long)s < p.N; };
  constexpr int kB = 8;  // entries per thread whose loads are in flight together
  const int stride = blockDim.x;

  for (int g = tid; g <= p.NB; g += stride) start[g] = 0;
  __syncthreads();
  for (int e0 = tid; e0 < nent; e0 += stride * kB) {
    int32_t sv[kB];
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int e = e0 + i * stride;
      sv[i] = e < nent ? slot_of(e) : 0;
    }
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int e = e0 + i * stride;
      if (e >= nent) break;
      if (!in_range(sv[i])) {
        if (io.validate) dev_flag(st, SDM_DEV_BAD_INDEX, int(trow0 + step_of(e)));
        continue;
      }
      atomicAdd(&start[slot_bucket(uint32_t(sv[i]), p.NB)], 1);
    }
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scan of the bucket counts, one warp
    const int per = (p.NB + 31) / 32;
    const int g0 = min(p.NB, lane * per), g1 = min(p.NB, g0 + per);
    int sum = 0;
    for (int g = g0; g < g1; ++g) sum += start[g];
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    int run = inc - sum;
    for (int g = g0; g < g1; ++g) {
      const int c = start[g];
      start[g] = run;
      cur[g] = run;
      run += c;
    }
    if (lane == 31) start[p.NB] = inc;
  }
  __syncthreads();
  int* roff = io.roff + (size_t(bh) * p.nblk + blk) * (p.NB + 1);
  for (int g = tid; g <= p.NB; g += stride) roff[g] = start[g];
  for (int e0 = tid; e0 < nent; e0 += stride * kB) {
    int32_t sv[kB];
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int e = e0 + i * stride;
      sv[i] = e < nent ? slot_of(e) : 0;
    }
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int e = e0 + i * stride;
      if (e >= nent) break;
      if (!in_range(sv[i])) continue;
      const int g = slot_bucket(uint32_t(sv[i]), p.NB);
      const int pos = atomicAdd(&cur[g], 1);
      key[pos] = (uint64_t(g) << (31 + kEntryBits)) | (uint64_t(uint32_t(sv[i])) << kEntryBits) |
                 uint64_t(e);
    }
  }
  __syncthreads();
  // Each entry's record goes to its bucket's start plus its rank inside the
  // bucket; its predecessor in that order tells whether a slot repeats within
  // one step's list.
  int4* rec = io.rec + (size_t(bh) * p.nblk + blk) * p.E;
  const int total = start[p.NB];
  constexpr uint64_t kEntryMask = (uint64_t(1) << kEntryBits) - 1;
  constexpr int kR = 4;
  for (int p0 = tid; p0 < total; p0 += stride * kR) {
    uint64_t x[kR];
    float w[kR], al[kR], be[kR];
#pragma unroll
    for (int i = 0; i < kR; ++i) {
      const int pos = p0 + i * stride;
      x[i] = pos < total ? key[pos] : 0;
      const int e = int(x[i] & kEntryMask);
      const int tl = step_of(e), j = e - tl * WR;
      w[i] = al[i] = be[i] = 0.f;
      if (pos < total) {
        if (j >= p.W) {
          w[i] = io.wr[(lrow0 + tl) * p.R + (j - p.W)];
        } else {
          w[i] = io.ww[(lrow0 + tl) * p.W + j];
          al[i] = io.alpha[trow0 + tl];
          be[i] = io.beta[trow0 + tl];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kR; ++i) {
      const int pos = p0 + i * stride;
      if (pos >= total) break;
      const int g = int(x[i] >> (31 + kEntryBits));
      const uint32_t s = uint32_t(x[i] >> kEntryBits) & 0x7fffffffu;
      const int e = int(x[i] & kEntryMask);
      const int tl = step_of(e), j = e - tl * WR;
      const bool is_read = j >= p.W;
      const int b0 = start[g], n = start[g + 1] - b0;
      int rank = 0;
      uint64_t pred = 0;
      for (int q = 0; q < n; ++q) {
        const uint64_t y = key[b0 + q];
        const bool lt = y < x[i];
        rank += lt ? 1 : 0;
        pred = (lt && y > pred) ? y : pred;
      }
      if (rank > 0 && (uint32_t(pred >> kEntryBits) & 0x7fffffffu) == s) {
        const int e2 = int(pred & kEntryMask);
        const int tl2 = step_of(e2);
        if (tl2 == tl && ((e2 - tl2 * WR) >= p.W) == is_read)
          dev_flag(st, SDM_DEV_BAD_LIST, int(trow0 + tl));
      }
      int4 r;
      r.x = int(s);
      r.y = ((s0 + tl) << 1) | (is_read ? 1 : 0);
      if (is_read) {
        r.z = __float_as_int(w[i]);
        r.w = 0;
      } else {
        const float c = be[i] * w[i];
        r.z = __float_as_int(al[i] * (1.f - c));
        r.w = __float_as_int(c);
      }
      rec[b0 + rank] = r;
    }
  }
  // the recurrence adds every read into o with reductions: start from zero
  float4* o4 = reinterpret_cast<float4*>(io.o + trow0 * p.dv);
  const int n4 = np * p.dv / 4;
  for (int i = tid; i < n4; i += stride) o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

cudaError_t launch_merge(const Plan& p, const MergeIO& io, int t0, int tlen, DevStatus* st,
                         cudaStream_t s) {
  const size_t smem = merge_smem_bytes(p, kMergeWarps);
  cudaError_t e = cudaFuncSetAttribute(k_merge, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((tlen + kMergeSteps - 1) / kMergeSteps, p.BH);
  k_merge<<<grid, kMergeWarps * 32, smem, s>>>(p, io, t0, tlen, st);
  return cudaGetLastError();
}

cudaError_t launch_plan(const Plan& p, const PlanIO& io, int t0, int tlen, DevStatus* st,
                        cudaStream_t s) {
  const size_t smem = plan_smem_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(k_plan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((tlen + p.P - 1) / p.P, p.BH);
  k_plan<<<grid, kPlanThreads, smem, s>>>(p, io, t0, tlen, st);
  return cudaGetLastError();
}

}  // namespace sdm
