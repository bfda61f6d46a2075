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
// Plan (one CTA per (head, block of P steps)): the block's W+R entries per step
// are grouped for the recurrence kernel.  Each slot belongs to one of G parts
// (a hash of the slot); records are laid out part by part: the writes of slots
// used once in the block, the reads of slots used once, then the slots used
// several times, grouped by slot in time order (write before read within a
// step).  A record is
//   int4 {slot, (step_in_block << 1) | is_read, weight bits, chain length},
// chain length = number of records of that slot in the block on its first
// record, 0 on the others.
#include "sdm_internal.cuh"

namespace sdm {

constexpr uint32_t kEmpty = 0xffffffffu;
constexpr uint32_t kInvalid = 0xffffffffu;

struct MergeLayout {
  size_t ent_slot, ent_w, stair, misc, uni, total;
  int Sk, Sc, Ss, HS, warps;
  size_t per_warp, phase2;
};

__host__ __device__ inline int p2(int x) {
  int p = 2;
  while (p < x) p <<= 1;
  return p;
}

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~size_t(15); }

__host__ __device__ inline MergeLayout merge_layout(const Plan& p, int warps) {
  MergeLayout L;
  L.Sk = p2(p.k);
  L.Sc = ((p.ncW > p.ncR ? p.ncW : p.ncR) + 31) & ~31;
  L.Ss = p2(p.W > p.R ? p.W : p.R);
  if (L.Ss < L.Sc) L.Ss = L.Sc;
  L.HS = p2(2 * p.E);
  L.warps = warps;
  size_t o = 0;
  L.ent_slot = o; o = al16(o + size_t(p.E) * 4);
  L.ent_w = o; o = al16(o + size_t(p.E) * 4);
  L.stair = o; o = al16(o + size_t(p.ncW + p.nfW + p.ncR + p.nfR) * 4);
  L.misc = o; o = al16(o + size_t(8 * (kMaxParts + 1) + 8) * 4);
  L.uni = o;
  L.per_warp = size_t(2 * L.Sk + 2 * L.Sc + L.Ss) * 8;
  L.phase2 = al16(size_t(L.HS) * 4) + al16(size_t(L.HS)) + al16(size_t(p2(p.E)) * 2);
  const size_t ph1 = L.per_warp * warps;
  o += (ph1 > L.phase2 ? ph1 : L.phase2);
  L.total = al16(o);
  return L;
}

size_t merge_smem_bytes(const Plan& p, int warps) { return merge_layout(p, warps).total; }

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

// The r-th largest (1-based) of the n distinct, nonzero keys in cand[]
// (left intact): quickselect with median-of-3 pivots; each round splits the
// live keys around the pivot into a scratch buffer (A and B alternate, each
// of capacity >= n) and keeps the side holding the answer; at <= 32 keys a
// warp sort finishes.
__device__ uint64_t warp_select(const uint64_t* cand, int n, int r, uint64_t* A, uint64_t* B) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = lanemask_lt();
  const uint64_t* src = cand;
  uint64_t* bufs[2] = {A, B};
  int which = 0;
  for (int iter = 0; iter < 4096; ++iter) {
    if (n <= 32) {
      uint64_t x = lane < n ? src[lane] : 0;
      __syncwarp();
      x = warp_sort32_desc(x);
      return __shfl_sync(0xffffffffu, x, r - 1);
    }
    const uint64_t a = src[0], b = src[n >> 1], c = src[n - 1];
    const uint64_t lo = a < b ? a : b, hi = a < b ? b : a;
    const uint64_t piv = c < lo ? lo : (c > hi ? hi : c);
    uint64_t* dst = bufs[which];
    int front = 0, back = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + lane;
      const uint64_t x = i < n ? src[i] : 0;
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
    const int ge = front + 1;
    if (ge == r) return piv;
    if (ge > r) {
      src = dst;
      n = front;
    } else {
      src = dst + (n - back);
      n = back;
      r -= ge;
    }
    which ^= 1;
  }
  return 0;  // not reached: each round removes at least the pivot
}

// Merge of one (step, side): sorted half lists (first k entries of each
// survivor list) -> the n_sel selected slots and their softmax weights.
// Selection order is unspecified unless `sorted` is set (then rank order).
__device__ void merge_one(const Plan& p, const uint2* sv1, int c1, const uint2* sv2, int c2,
                          int n_sel, const uint32_t* stair, int nc, const uint32_t* front, int nf,
                          uint64_t* h1, uint64_t* h2, uint64_t* cand, uint64_t* alt,
                          uint64_t* sel, bool sorted, float* w_out, uint32_t* slot_out,
                          DevStatus* st, int info) {
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
  for (int i = lane; i < nc; i += 32) {
    const uint32_t ab = stair[i];
    const int a = ab & 0xffff, b = ab >> 16;
    const float v = key_val(h1[a]) + key_val(h2[b]);
    cand[i] = make_key(v, key_idx(h1[a]) * n + key_idx(h2[b]));
  }
  __syncwarp();
  const uint64_t kth = warp_select(cand, nc, n_sel, alt, sel);
  // every candidate outside the staircase must score strictly below the kth
  const uint32_t tau = uint32_t(kth >> 32);
  bool bad = false;
  for (int i = lane; i < nf; i += 32) {
    const uint32_t ab = front[i];
    const int a = ab & 0xffff, b = ab >> 16;
    bad |= f2ord(key_val(h1[a]) + key_val(h2[b])) >= tau;
  }
  bool is_sorted = false;
  if (__any_sync(0xffffffffu, bad)) {
    merge_full(h1, h2, p.k, p.n, n_sel, sel);
    is_sorted = true;
  } else {
    int base = 0;
    for (int i0 = 0; i0 < nc; i0 += 32) {
      const int i = i0 + lane;
      const uint64_t x = i < nc ? cand[i] : 0;
      const bool take = (i < nc) && x >= kth;
      const unsigned m = __ballot_sync(0xffffffffu, take);
      if (take) sel[base + __popc(m & lanemask_lt())] = x;
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
  float zs = 0.f;
  for (int i = lane; i < n_sel; i += 32) zs += expf(key_val(sel[i]) - m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, off);
  const float inv = 1.f / zs;
  for (int i = lane; i < n_sel; i += 32) {
    w_out[i] = expf(key_val(sel[i]) - m) * inv;
    slot_out[i] = key_idx(sel[i]);
  }
  __syncwarp();
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(kMergeThreads)
k_merge_plan(Plan p, MergeIO io, int t0, int tlen, DevStatus* st) {
  extern __shared__ __align__(16) unsigned char smem[];
  const MergeLayout L = merge_layout(p, p.merge_warps);
  uint32_t* ent_slot = reinterpret_cast<uint32_t*>(smem + L.ent_slot);
  float* ent_w = reinterpret_cast<float*>(smem + L.ent_w);
  uint32_t* stairW = reinterpret_cast<uint32_t*>(smem + L.stair);
  uint32_t* frontW = stairW + p.ncW;
  uint32_t* stairR = frontW + p.nfW;
  uint32_t* frontR = stairR + p.ncR;
  int* cnt_w = reinterpret_cast<int*>(smem + L.misc);  // single-use writes per part
  int* cnt_r = cnt_w + (kMaxParts + 1);                  // single-use reads per part
  int* cnt_m = cnt_r + (kMaxParts + 1);                  // multi-use entries per part
  int* base = cnt_m + (kMaxParts + 1);
  int* mbase = base + (kMaxParts + 1);
  int* fill_w = mbase + (kMaxParts + 1);
  int* fill_r = fill_w + (kMaxParts + 1);
  int* misc = fill_r + (kMaxParts + 1);  // [0] n_multi
  unsigned char* uni = smem + L.uni;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int WR = p.W + p.R;
  const int s0 = blk * p.P;                 // first step of the block within the chunk
  if (s0 >= tlen) return;
  const int np = min(p.P, tlen - s0);
  const int nent = np * WR;

  if (io.mode != 2) {
    // staircase tables: row a holds columns b < min(k, n_sel / (a+1))
    if (tid == 0) {
      int oc = 0, of = 0, prev = -1;
      for (int a = 0; a < p.k; ++a) {
        const int bm = min(p.k, p.W / (a + 1));
        for (int b = 0; b < bm; ++b) stairW[oc++] = uint32_t(a) | (uint32_t(b) << 16);
        if (bm < p.k && !(bm == 0 && prev == 0)) frontW[of++] = uint32_t(a) | (uint32_t(bm) << 16);
        prev = bm;
      }
    } else if (tid == 32) {
      int oc = 0, of = 0, prev = -1;
      for (int a = 0; a < p.k; ++a) {
        const int bm = min(p.k, p.R / (a + 1));
        for (int b = 0; b < bm; ++b) stairR[oc++] = uint32_t(a) | (uint32_t(b) << 16);
        if (bm < p.k && !(bm == 0 && prev == 0)) frontR[of++] = uint32_t(a) | (uint32_t(bm) << 16);
        prev = bm;
      }
    }
    __syncthreads();
    // ---- phase 1: merges, one warp per (step, side)
    if (warp < p.merge_warps) {
      uint64_t* h1 = reinterpret_cast<uint64_t*>(uni + L.per_warp * warp);
      uint64_t* h2 = h1 + L.Sk;
      uint64_t* cand = h2 + L.Sk;
      uint64_t* alt = cand + L.Sc;
      uint64_t* sel = alt + L.Sc;
      for (int pi = warp; pi < 2 * np; pi += p.merge_warps) {
        const int tl = pi >> 1, side = pi & 1;
        const int tc = s0 + tl;                       // step within the chunk
        const size_t hr = (size_t(bh) * p.Tc + tc) * 4 + side * 2;
        const int n_sel = side ? p.R : p.W;
        float* w_out = ent_w + tl * WR + (side ? p.W : 0);
        uint32_t* s_out = ent_slot + tl * WR + (side ? p.W : 0);
        merge_one(p, io.surv + hr * p.C, io.surv_cnt[hr], io.surv + (hr + 1) * p.C,
                  io.surv_cnt[hr + 1], n_sel, side ? stairR : stairW, side ? p.ncR : p.ncW,
                  side ? frontR : frontW, side ? p.nfR : p.nfW, h1, h2, cand, alt, sel,
                  io.mode == 1, w_out, s_out, st, int(hr));
        if (io.mode == 1) {
          const size_t t = size_t(bh) * p.T + t0 + tc;
          int32_t* oi = side ? io.out_ir : io.out_iw;
          float* ow = side ? io.out_wr : io.out_ww;
          for (int i = lane; i < n_sel; i += 32) {
            oi[t * n_sel + i] = int32_t(s_out[i]);
            ow[t * n_sel + i] = w_out[i];
          }
        }
      }
    }
    if (io.mode == 1) return;
  } else {
    // ---- lists given: validate and copy
    for (int e = tid; e < nent; e += blockDim.x) {
      const int tl = e / WR, j = e - tl * WR;
      const size_t t = size_t(bh) * p.T + t0 + s0 + tl;
      int32_t s;
      float w;
      if (j < p.W) { s = io.in_iw[t * p.W + j]; w = io.in_ww[t * p.W + j]; }
      else { s = io.in_ir[t * p.R + (j - p.W)]; w = io.in_wr[t * p.R + (j - p.W)]; }
      if (s < 0 || (long long)s >= p.N) {
        dev_flag(st, SDM_DEV_BAD_INDEX, int(t));
        ent_slot[e] = kInvalid;
      } else {
        ent_slot[e] = uint32_t(s);
      }
      ent_w[e] = w;
    }
  }
  __syncthreads();

  // ---- phase 2: plan.  Hash table of the block's slots -> used once or more.
  uint32_t* hkey = reinterpret_cast<uint32_t*>(uni);
  unsigned char* hflag = uni + al16(size_t(L.HS) * 4);
  uint16_t* mlist = reinterpret_cast<uint16_t*>(uni + al16(size_t(L.HS) * 4) + al16(size_t(L.HS)));
  const uint32_t hmask = uint32_t(L.HS - 1);
  for (int i = tid; i < L.HS; i += blockDim.x) { hkey[i] = kEmpty; hflag[i] = 0; }
  for (int i = tid; i <= p.G; i += blockDim.x) {
    cnt_w[i] = 0; cnt_r[i] = 0; cnt_m[i] = 0; fill_w[i] = 0; fill_r[i] = 0;
  }
  if (tid == 0) misc[0] = 0;
  __syncthreads();
  for (int e = tid; e < nent; e += blockDim.x) {
    const uint32_t s = ent_slot[e];
    if (s == kInvalid) continue;
    uint32_t h = mix32(s) & hmask;
    for (;;) {
      const uint32_t old = atomicCAS(&hkey[h], kEmpty, s);
      if (old == kEmpty) break;
      if (old == s) { hflag[h] = 1; break; }
      h = (h + 1) & hmask;
    }
  }
  __syncthreads();
  for (int e = tid; e < nent; e += blockDim.x) {
    const uint32_t s = ent_slot[e];
    if (s == kInvalid) continue;
    uint32_t h = mix32(s) & hmask;
    while (hkey[h] != s) h = (h + 1) & hmask;
    const int part = slot_part(s, p.G);
    if (hflag[h]) {
      mlist[atomicAdd(&misc[0], 1)] = uint16_t(e);
      atomicAdd(&cnt_m[part], 1);
    } else if ((e % WR) < p.W) {
      atomicAdd(&cnt_w[part], 1);
    } else {
      atomicAdd(&cnt_r[part], 1);
    }
  }
  __syncthreads();
  const int n_multi = misc[0];
  if (tid == 0) {
    int acc = 0, macc = 0;
    for (int g = 0; g < p.G; ++g) {
      base[g] = acc;
      mbase[g] = macc;
      acc += cnt_w[g] + cnt_r[g] + cnt_m[g];
      macc += cnt_m[g];
    }
    base[p.G] = acc;
  }
  // sort the multi-use entries by (part, slot, entry) -- ascending bitonic
  {
    const int S = n_multi > 1 ? p2(n_multi) : 1;
    for (int i = n_multi + tid; i < S; i += blockDim.x) mlist[i] = 0xffff;
    __syncthreads();
    auto mkey = [&](uint16_t e) -> uint64_t {
      if (e == 0xffff) return ~uint64_t(0);
      const uint32_t s = ent_slot[e];
      return (uint64_t(slot_part(s, p.G)) << 46) | (uint64_t(s) << 14) | uint64_t(e);
    };
    for (int size = 2; size <= S; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < (S >> 1); i += blockDim.x) {
          const int lo = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));
          const int hi = lo + stride;
          const uint16_t x = mlist[lo], y = mlist[hi];
          const uint64_t kx = mkey(x), ky = mkey(y);
          const bool asc = (lo & size) == 0;
          if (asc ? (kx > ky) : (kx < ky)) { mlist[lo] = y; mlist[hi] = x; }
        }
        __syncthreads();
      }
    }
  }
  __syncthreads();
  int4* rec = io.rec + (size_t(bh) * p.nblk + blk) * p.E;
  auto meta_of = [&](int e) -> int {
    const int tl = e / WR;
    return (tl << 1) | ((e - tl * WR) >= p.W ? 1 : 0);
  };
  for (int e = tid; e < nent; e += blockDim.x) {
    const uint32_t s = ent_slot[e];
    if (s == kInvalid) continue;
    uint32_t h = mix32(s) & hmask;
    while (hkey[h] != s) h = (h + 1) & hmask;
    if (hflag[h]) continue;
    const int part = slot_part(s, p.G);
    const bool is_read = (e % WR) >= p.W;
    const int pos = is_read ? base[part] + cnt_w[part] + atomicAdd(&fill_r[part], 1)
                            : base[part] + atomicAdd(&fill_w[part], 1);
    rec[pos] = make_int4(int(s), meta_of(e), __float_as_int(ent_w[e]), 1);
  }
  for (int i = tid; i < n_multi; i += blockDim.x) {
    const int e = mlist[i];
    const uint32_t s = ent_slot[e];
    const int part = slot_part(s, p.G);
    const int pos = base[part] + cnt_w[part] + cnt_r[part] + (i - mbase[part]);
    int len = 0;
    if (i == 0 || ent_slot[mlist[i - 1]] != s) {
      int j = i + 1;
      while (j < n_multi && ent_slot[mlist[j]] == s) ++j;
      len = j - i;
    } else if (meta_of(mlist[i - 1]) == meta_of(e)) {
      dev_flag(st, SDM_DEV_BAD_LIST, int(size_t(bh) * p.T + t0 + s0 + e / WR));
    }
    rec[pos] = make_int4(int(s), meta_of(e), __float_as_int(ent_w[e]), len);
  }
  // per part g: single writes [3g, 3g+1), single reads [3g+1, 3g+2), multi-use
  // chains [3g+2, 3g+3); entry 3G = end
  int* roff = io.roff + (size_t(bh) * p.nblk + blk) * (3 * p.G + 1);
  for (int g = tid; g < p.G; g += blockDim.x) {
    roff[3 * g] = base[g];
    roff[3 * g + 1] = base[g] + cnt_w[g];
    roff[3 * g + 2] = base[g] + cnt_w[g] + cnt_r[g];
  }
  if (tid == 0) roff[3 * p.G] = base[p.G];
  // the recurrence adds every read into o with reductions: start from zero
  float4* o4 = reinterpret_cast<float4*>(io.o + (size_t(bh) * p.T + t0 + s0) * p.dv);
  const int n4 = np * p.dv / 4;
  for (int i = tid; i < n4; i += blockDim.x) o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

cudaError_t launch_merge_plan(const Plan& p, const MergeIO& io, int t0, int tlen, DevStatus* st,
                              cudaStream_t s) {
  const size_t smem = merge_smem_bytes(p, p.merge_warps);
  cudaError_t e = cudaFuncSetAttribute(k_merge_plan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  const int nb = (tlen + p.P - 1) / p.P;
  dim3 grid(nb, p.BH);
  k_merge_plan<<<grid, kMergeThreads, smem, s>>>(p, io, t0, tlen, st);
  return cudaGetLastError();
}

}  // namespace sdm
