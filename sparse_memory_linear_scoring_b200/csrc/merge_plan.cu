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
// two halves) and select the n_sel best (64 buckets of the score range, then a
// warp sort of the bucket that holds the n_sel-th, or quickselect).  This is exact when every
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
// is then M = f1 * M + f2 * v_t); for a read, f1 = u_r.  Under the selective-
// decay write rule (the Raven page, section 2.2: router weight r_i, decay
// rate a_t), f1 = exp(a_t r_i) and f2 = 1 - f1.  The per-(head, block)
// bucket starts (NB + 1 of them) go to roff.
#include "merge_dev.cuh"

namespace sdm {

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

// ------------------------------------------------------------------ kernels
// One CTA per (head, kMergeSteps steps); one warp per (step, side).  Writes
// the W write and R read (slot, weight) pairs of each step to the lists
// (row = bh * list_T + list_t0 + step), in rank order when `sorted`.  A warp
// loads the half lists of its next (step, side) into registers (KPL entries
// per lane, k <= 32 KPL) while it merges the current one; KPL = 0 leaves the
// loads to merge_one.  The launch bounds keep the k <= 64 kernels at 64
// registers (four CTAs per SM, the shared-memory limit too) and give the wider
// ones room for their lists without spilling.
template <int KPL>
__global__ void __launch_bounds__(kMergeWarps * 32, KPL >= 4 ? 3 : 4)
k_merge(Plan p, MergeIO io, int t0, int tlen, DevStatus* st) {
  extern __shared__ __align__(16) unsigned char smem[];
  const MergeLayout L = merge_layout(p, kMergeWarps);
  uint32_t* stairW = reinterpret_cast<uint32_t*>(smem + L.stair);
  uint32_t* frontW = stairW + p.ncW;
  uint32_t* stairR = frontW + p.nfW;
  uint32_t* frontR = stairR + p.ncR;
  int* edivW = reinterpret_cast<int*>(frontR + p.nfR);
  int* edivR = edivW + p.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bh = blockIdx.y;
  const int s0 = blockIdx.x * kMergeSteps;
  if (s0 >= tlen) return;
  const int np = min(kMergeSteps, tlen - s0);
  if (warp == 0) build_staircase(p.k, p.W, stairW, frontW, edivW);
  if (warp == 1) build_staircase(p.k, p.R, stairR, frontR, edivR);
  __syncthreads();
  unsigned char* mine = smem + L.uni + L.per_warp * warp;
  uint64_t* h1 = reinterpret_cast<uint64_t*>(mine);
  uint64_t* h2 = h1 + L.Sk;
  uint64_t* sel = h2 + L.Sk;
  uint32_t* cand = reinterpret_cast<uint32_t*>(sel + L.Ss);
  uint32_t* cell = cand + L.Sc;
  uint32_t* alt = cell + L.Sc;
  int* hist = reinterpret_cast<int*>(alt + 2 * L.Sc);
  auto task_hr = [&](int pi) { return (size_t(bh) * p.Tc + s0 + (pi >> 1)) * 4 + (pi & 1) * 2; };
  uint2 pa[KPL > 0 ? KPL : 1], pb[KPL > 0 ? KPL : 1];
  int pc1 = 0, pc2 = 0;
  auto prefetch = [&](int pi) {
    const size_t hr = task_hr(pi);
    pc1 = io.surv_cnt[hr];
    pc2 = io.surv_cnt[hr + 1];
    const uint2* l1 = io.surv + hr * p.C;
    const uint2* l2 = l1 + p.C;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = j * 32 + lane;
      if (i < p.k) {
        pa[j] = l1[i];
        pb[j] = l2[i];
      }
    }
  };
  if (KPL > 0 && warp < 2 * np) prefetch(warp);
  for (int pi = warp; pi < 2 * np; pi += kMergeWarps) {
    const int tc = s0 + (pi >> 1), side = pi & 1;
    const size_t hr = task_hr(pi);
    const int n_sel = side ? p.R : p.W;
    const size_t row = size_t(bh) * io.list_T + io.list_t0 + tc;
    float* w_out = (side ? io.out_wr : io.out_ww) + row * n_sel;
    uint32_t* s_out = reinterpret_cast<uint32_t*>(side ? io.out_ir : io.out_iw) + row * n_sel;
    const uint2* l1 = nullptr;
    const uint2* l2 = nullptr;
    int c1, c2;
    if (KPL > 0) {
#pragma unroll
      for (int j = 0; j < KPL; ++j) {
        const int i = j * 32 + lane;
        if (i < p.k) {
          h1[i] = (uint64_t(pa[j].x) << 32) | pa[j].y;
          h2[i] = (uint64_t(pb[j].x) << 32) | pb[j].y;
        }
      }
      c1 = pc1;
      c2 = pc2;
      if (pi + kMergeWarps < 2 * np) prefetch(pi + kMergeWarps);
    } else {
      l1 = io.surv + hr * p.C;
      l2 = l1 + p.C;
      c1 = io.surv_cnt[hr];
      c2 = io.surv_cnt[hr + 1];
    }
    merge_one(p, l1, c1, l2, c2, n_sel, side ? stairR : stairW, side ? p.ncR : p.ncW,
              side ? frontR : frontW, side ? p.nfR : p.nfW, side ? edivR : edivW, h1, h2, cand,
              cell, alt, hist, sel,
              io.sorted != 0, w_out, s_out, st, int(hr), p.rule == 1 && side == 0);
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
  {
    // exclusive scan of the bucket counts over the whole CTA: each thread sums
    // a run of buckets, a warp scan and a scan of the warp totals give its base
    __shared__ int wtot[kPlanThreads / 32];
    const int per = (p.NB + stride - 1) / stride;
    const int g0 = min(p.NB, tid * per), g1 = min(p.NB, g0 + per);
    int sum = 0;
    for (int g = g0; g < g1; ++g) sum += start[g];
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) wtot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const int x = lane < kPlanThreads / 32 ? wtot[lane] : 0;
      int wi = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      if (lane < kPlanThreads / 32) wtot[lane] = wi - x;  // exclusive
      if (lane == 31) start[p.NB] = wi;                   // all entries in range
    }
    __syncthreads();
    int run = wtot[warp] + inc - sum;
    for (int g = g0; g < g1; ++g) {
      const int c = start[g];
      start[g] = run;
      cur[g] = run;
      run += c;
    }
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
          be[i] = p.rule == 1 ? 0.f : io.beta[trow0 + tl];
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
      } else if (p.rule == 1) {
        // selective decay: M = e^{a r} M + (1 - e^{a r}) v, with a in alpha
        const float d = expf(al[i] * w[i]);
        r.z = __float_as_int(d);
        r.w = __float_as_int(1.f - d);
      } else {
        const float c = be[i] * w[i];
        r.z = __float_as_int(al[i] * (1.f - c));
        r.w = __float_as_int(c);
      }
      rec[b0 + rank] = r;
      if (io.rent) io.rent[(size_t(bh) * p.nblk + blk) * p.E + b0 + rank] = e;
    }
  }
  // the recurrence adds every read into o with reductions: start from zero
  if (io.o) {
    float4* o4 = reinterpret_cast<float4*>(io.o + trow0 * p.dv);
    const int n4 = np * p.dv / 4;
    for (int i = tid; i < n4; i += stride) o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int KPL>
static cudaError_t launch_merge_t(const Plan& p, const MergeIO& io, int t0, int tlen,
                                  DevStatus* st, size_t smem, dim3 grid, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(k_merge<KPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  k_merge<KPL><<<grid, kMergeWarps * 32, smem, s>>>(p, io, t0, tlen, st);
  return cudaGetLastError();
}

cudaError_t launch_merge(const Plan& p, const MergeIO& io, int t0, int tlen, DevStatus* st,
                         cudaStream_t s) {
  const size_t smem = merge_smem_bytes(p, kMergeWarps);
  dim3 grid((tlen + kMergeSteps - 1) / kMergeSteps, p.BH);
  if (p.k <= 32) return launch_merge_t<1>(p, io, t0, tlen, st, smem, grid, s);
  if (p.k <= 64) return launch_merge_t<2>(p, io, t0, tlen, st, smem, grid, s);
  if (p.k <= 128) return launch_merge_t<4>(p, io, t0, tlen, st, smem, grid, s);
  return launch_merge_t<0>(p, io, t0, tlen, st, smem, grid, s);
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
