// step.cu -- the SDM forward pass for short calls (decoding), fused into one
// kernel: one CTA per (b,h) head runs the call's steps in order, and every
// phase of a step stays on chip (no workspace).
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central" items 1-4, per
// step t (the same method as sdm_forward):
//   1. scoring (item 2): the two halves of k'_t and q'_t against C1 and C2, on
//      CUDA cores (float32 FMA), into shared memory: 4 x n scores;
//   2. per-half top-k (item 2): four warps per (side, half) find the k-th
//      largest score by a bitwise search over order-preserving images (their
//      counts added through shared memory), and the k best are sorted by
//      (score desc, row asc);
//   3. merge (item 2): one warp per side takes the top-W (k') / top-R (q') of
//      the k x k outer-sum candidates with the staircase merge of sdm_forward,
//      and their softmax weights;
//   4. write (item 3): each write slot is gated and delta-updated,
//      M[i] = f1 * M[i] + f2 * v_t with f2 = c = beta_t * w_i and
//      f1 = alpha_t * (1 - c);
//   5. read (item 4), after the write: o_t = sum_r u_r M_t[r], reduced in a
//      fixed order (run to run reproducible).
// A step's phases are separated by CTA barriers; global writes of step t are
// visible to the reads of step t and to the writes of step t + 1 of the same
// CTA, which owns its head's table.
#include "merge_dev.cuh"
#include "select_dev.cuh"

namespace sdm {

constexpr int kStepThreads = 512;
constexpr int kStepWarps = kStepThreads / 32;
constexpr int kStepMaxN = 1024;   // scores of a half-row held 32 per lane
constexpr int kStepMaxK = 256;

struct StepLayout {
  size_t x, sc, tk, hl, merge, selw, sels, opart, st, xch, total;
  int K2;
  MergeLayout ML;
};

__host__ __device__ inline StepLayout step_layout(const Plan& p) {
  StepLayout L;
  L.K2 = p2(p.k);
  L.ML = merge_layout(p, 2);
  size_t o = 0;
  L.x = o; o = al16(o + size_t(2) * p.dqk * 4);          // k'_t, q'_t as float
  L.sc = o; o = al16(o + size_t(4) * p.n * 4);           // scores [side*2 + half][n]
  L.tk = o; o = al16(o + size_t(4) * L.K2 * 8);          // top-k keys per half-row
  L.hl = o; o = al16(o + size_t(4) * L.K2 * 8);          // sorted (score, row) lists
  L.merge = o; o = al16(o + L.ML.total);                 // staircases + 2 warps' scratch
  L.selw = o; o = al16(o + size_t(p.W + p.R) * 4);       // weights: write, then read
  L.sels = o; o = al16(o + size_t(p.W + p.R) * 4);       // slots: write, then read
  L.opart = o; o = al16(o + size_t(kStepWarps) * p.dv * 4);
  L.st = o; o = al16(o + sizeof(DevStatus));
  L.xch = o; o = al16(o + size_t(4) * 8 * 4);              // top-k count exchange

  L.total = o;
  return L;
}

// Elements of a 16-byte load, and the lanes that cover one codebook row half.
template <typename Tin>
__host__ __device__ constexpr int step_epl() { return int(16 / sizeof(Tin)); }

template <typename Tin>
__device__ __forceinline__ void ld16(const Tin* ptr, float* out);
template <>
__device__ __forceinline__ void ld16<float>(const float* ptr, float* out) {
  const float4 v = __ldg(reinterpret_cast<const float4*>(ptr));
  out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}
template <>
__device__ __forceinline__ void ld16<__nv_bfloat16>(const __nv_bfloat16* ptr, float* out) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(ptr));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(w[i] << 16);
    out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float4 ldcg4(const float* ptr) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(ptr));
  return v;
}

template <typename Tin>
__device__ __forceinline__ float4 ld_v4(const Tin* ptr);
template <>
__device__ __forceinline__ float4 ld_v4<float>(const float* ptr) {
  return __ldg(reinterpret_cast<const float4*>(ptr));
}
template <>
__device__ __forceinline__ float4 ld_v4<__nv_bfloat16>(const __nv_bfloat16* ptr) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(ptr));
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

// The k best of one half-row's n <= 1024 scores (sc), found by the four warps of
// a group: warp `part` holds entries [256 part, 256 part + 256), 8 per lane,
// in row order.  The k-th largest order-preserving image comes from a bitwise
// search whose per-bit counts the four warps add through shared memory (xch,
// [2][4] ints, double-buffered by bit parity) behind the group's named barrier
// `bar` (128 threads); the k best -- ties at the threshold to the lowest rows,
// i.e. in warp then lane order -- are written to out[0..k) as 64-bit keys.
__device__ __forceinline__ void group_bar(int bar) {
  asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
}

__device__ void group_topk(const float* sc, int n, int k, int part, int bar, int* xch,
                           uint64_t* out) {
  const int lane = threadIdx.x & 31;
  uint32_t key[8];
  uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int j = part * 256 + u * 32 + lane;
    key[u] = j < n ? f2ord(sc[j]) : 0u;  // 0: below every valid image
    if (j < n) {
      lo = min(lo, key[u]);
      hi = max(hi, key[u]);
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    xch[part] = int(lo);
    xch[4 + part] = int(hi);
  }
  group_bar(bar);
  lo = min(min(uint32_t(xch[0]), uint32_t(xch[1])), min(uint32_t(xch[2]), uint32_t(xch[3])));
  hi = max(max(uint32_t(xch[4]), uint32_t(xch[5])), max(uint32_t(xch[6]), uint32_t(xch[7])));
  group_bar(bar);  // everyone has read lo/hi before the slots are reused
  uint32_t thr = hi;
  const uint32_t diff = lo ^ hi;
  if (diff != 0u) {
    const int top = 31 - __clz(diff);
    thr = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t cand = thr | (1u << bit);
      int c = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) c += key[u] >= cand ? 1 : 0;
      c = __reduce_add_sync(0xffffffffu, c);
      int* slot = xch + (bit & 1) * 4;
      if (lane == 0) slot[part] = c;
      group_bar(bar);
      if (slot[0] + slot[1] + slot[2] + slot[3] >= k) thr = cand;
    }
  }
  // the entries above thr, then the lowest rows equal to it
  int ngt = 0, neq = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    ngt += key[u] > thr ? 1 : 0;
    neq += (key[u] == thr && part * 256 + u * 32 + lane < n) ? 1 : 0;
  }
  ngt = __reduce_add_sync(0xffffffffu, ngt);
  neq = __reduce_add_sync(0xffffffffu, neq);
  group_bar(bar);  // the last bit's counts have been read
  if (lane == 0) {
    xch[part] = ngt;
    xch[4 + part] = neq;
  }
  group_bar(bar);
  int gt_all = 0, eq_before = 0, gt_before = 0;
  for (int w = 0; w < 4; ++w) {
    gt_all += xch[w];
    if (w < part) {
      eq_before += xch[4 + w];
      gt_before += xch[w];
    }
  }
  const int m = k - gt_all;  // ties to take overall, lowest rows first
  int ties_here = min(max(m - eq_before, 0), neq);
  int eq_taken_before = min(max(m, 0), eq_before);
  int base = gt_before + eq_taken_before;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int j = part * 256 + u * 32 + lane;
    const bool above = key[u] > thr;
    const bool tie = key[u] == thr && j < n;
    const unsigned mt = __ballot_sync(0xffffffffu, tie);
    const int trank = __popc(mt & lt);
    const bool take = above || (tie && trank < ties_here);
    const unsigned mk = __ballot_sync(0xffffffffu, take);
    if (take) out[base + __popc(mk & lt)] = (uint64_t(key[u]) << 32) | uint64_t(~uint32_t(j));
    base += __popc(mk);
    ties_here -= min(ties_here, __popc(mt));
  }
}

struct StepIO {
  const void *q, *k, *v;
  const float *alpha, *beta;
  const void *C1, *C2;
  float *M, *o;
  int32_t* idx_w; float* w_w; int32_t* idx_r; float* w_r;  // optional lists (rank order)
};

template <typename Tin, int LPRW>
__global__ void __launch_bounds__(kStepThreads, 1) k_step(Plan p, StepIO io) {
  extern __shared__ __align__(16) unsigned char smem[];
  const StepLayout L = step_layout(p);
  float* xs = reinterpret_cast<float*>(smem + L.x);
  float* sc = reinterpret_cast<float*>(smem + L.sc);
  uint64_t* tk = reinterpret_cast<uint64_t*>(smem + L.tk);
  uint2* hl = reinterpret_cast<uint2*>(smem + L.hl);
  unsigned char* msm = smem + L.merge;
  float* selw = reinterpret_cast<float*>(smem + L.selw);
  uint32_t* sels = reinterpret_cast<uint32_t*>(smem + L.sels);
  float* opart = reinterpret_cast<float*>(smem + L.opart);
  DevStatus* st = reinterpret_cast<DevStatus*>(smem + L.st);
  int* xch = reinterpret_cast<int*>(smem + L.xch);
  constexpr int EPL = step_epl<Tin>();
  constexpr int RPW = 32 / LPRW;  // codebook rows per warp and iteration
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, h = bh % p.H;
  const int n = p.n, dh = p.dh, dqk = p.dqk, dv = p.dv, k = p.k;
  const int K2 = L.K2;
  const Tin* qg = static_cast<const Tin*>(io.q);
  const Tin* kg = static_cast<const Tin*>(io.k);
  const Tin* vg = static_cast<const Tin*>(io.v);
  const Tin* c1 = static_cast<const Tin*>(io.C1) + size_t(h) * n * dh;
  const Tin* c2 = static_cast<const Tin*>(io.C2) + size_t(h) * n * dh;
  float* Mh = io.M + size_t(bh) * size_t(p.N) * dv;
  const bool lists = io.idx_w != nullptr;

  // staircase tables of the merge, once (warp 0: write side, warp 1: read side)
  uint32_t* stairW = reinterpret_cast<uint32_t*>(msm + L.ML.stair);
  uint32_t* frontW = stairW + p.ncW;
  uint32_t* stairR = frontW + p.nfW;
  uint32_t* frontR = stairR + p.ncR;
  int* edivW = reinterpret_cast<int*>(frontR + p.nfR);
  int* edivR = edivW + p.k;
  if (warp == 0) build_staircase(k, p.W, stairW, frontW, edivW);
  if (warp == 1) build_staircase(k, p.R, stairR, frontR, edivR);
  if (tid == 0) {
    st->flags = 0;
    st->info = -1;
  }

  for (int t = 0; t < p.T; ++t) {
    const size_t row = size_t(bh) * p.T + t;
    // ---- 1. k'_t and q'_t as float
    for (int i = tid; i < 2 * dqk; i += kStepThreads) {
      const Tin* src = i < dqk ? kg + row * dqk + i : qg + row * dqk + (i - dqk);
      xs[i] = to_f32(*src);
    }
    __syncthreads();
    // ---- 2. scores of both halves, both sides: RPW codebook rows per warp
    // load, LPRW lanes per row, EPL elements per lane; kUnr loads in flight
    // per warp before their products; each codebook row serves k' and q'
    {
      constexpr int kUnr = 4;
      const int sub = lane / LPRW, part = lane % LPRW;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float xk[EPL], xq[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          xk[e] = xs[half * dh + part * EPL + e];
          xq[e] = xs[dqk + half * dh + part * EPL + e];
        }
        const Tin* cbh = (half ? c2 : c1) + part * EPL;
        for (int j0 = warp * RPW * kUnr; j0 < n; j0 += kStepWarps * RPW * kUnr) {
          float cb[kUnr][EPL];
#pragma unroll
          for (int u = 0; u < kUnr; ++u) {
            const int j = j0 + u * RPW + sub;
            if (j < n) {
              ld16<Tin>(cbh + size_t(j) * dh, cb[u]);
            } else {
#pragma unroll
              for (int e = 0; e < EPL; ++e) cb[u][e] = 0.f;
            }
          }
#pragma unroll
          for (int u = 0; u < kUnr; ++u) {
            float pk = 0.f, pq = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
              pk = fmaf(xk[e], cb[u][e], pk);
              pq = fmaf(xq[e], cb[u][e], pq);
            }
#pragma unroll
            for (int off = LPRW / 2; off > 0; off >>= 1) {
              pk += __shfl_xor_sync(0xffffffffu, pk, off);
              pq += __shfl_xor_sync(0xffffffffu, pq, off);
            }
            const int j = j0 + u * RPW + sub;
            if (j < n && part == 0) {
              sc[(0 * 2 + half) * n + j] = pk;
              sc[(1 * 2 + half) * n + j] = pq;
            }
          }
        }
      }
    }
    __syncthreads();
    // ---- 3. exact sorted top-k of each of the four half-rows, four warps each
    {
      const int hrw = warp >> 2, part = warp & 3;
      uint64_t* out = tk + size_t(hrw) * K2;
      group_topk(sc + size_t(hrw) * n, n, k, part, 1 + hrw, xch + hrw * 8, out);
      group_bar(1 + hrw);
      if (part == 0) {
        for (int i = k + lane; i < K2; i += 32) out[i] = 0;
        __syncwarp();
        warp_sort_desc(out, K2);
        uint2* hw = hl + size_t(hrw) * K2;
        for (int i = lane; i < k; i += 32)
          hw[i] = make_uint2(__float_as_uint(key_val(out[i])), key_idx(out[i]));
      }
    }
    __syncthreads();
    // ---- 4. merge: warp 0 the write slots (k'), warp 1 the read slots (q')
    if (warp < 2) {
      const int side = warp;
      const int n_sel = side ? p.R : p.W;
      unsigned char* mine = msm + L.ML.uni + L.ML.per_warp * warp;
      uint64_t* h1 = reinterpret_cast<uint64_t*>(mine);
      uint64_t* h2 = h1 + L.ML.Sk;
      uint64_t* sel = h2 + L.ML.Sk;
      uint32_t* cand = reinterpret_cast<uint32_t*>(sel + L.ML.Ss);
      uint32_t* cell = cand + L.ML.Sc;
      uint32_t* alt = cell + L.ML.Sc;
      int* hist = reinterpret_cast<int*>(alt + 2 * L.ML.Sc);
      float* w_out = selw + (side ? p.W : 0);
      uint32_t* s_out = sels + (side ? p.W : 0);
      merge_one(p, hl + size_t(side * 2) * K2, k, hl + size_t(side * 2 + 1) * K2, k, n_sel,
                side ? stairR : stairW, side ? p.ncR : p.ncW, side ? frontR : frontW,
                side ? p.nfR : p.nfW, side ? edivR : edivW, h1, h2, cand, cell, alt, hist, sel, lists,
                w_out, s_out, st, t);
      if (lists) {
        int32_t* gi = (side ? io.idx_r : io.idx_w) + row * n_sel;
        float* gw = (side ? io.w_r : io.w_w) + row * n_sel;
        for (int i = lane; i < n_sel; i += 32) {
          gi[i] = int32_t(s_out[i]);
          gw[i] = w_out[i];
        }
      }
    }
    __syncthreads();
    // ---- 5. gated delta write of the W slots (float4 columns, rows in order)
    const int dv4 = dv / 4;
    {
      const float al = __ldg(io.alpha + row), be = __ldg(io.beta + row);
      for (int i = tid; i < p.W * dv4; i += kStepThreads) {
        const int r = i / dv4, c4 = i - r * dv4;
        const uint32_t slot = sels[r];
        if (slot >= uint32_t(p.N)) continue;  // an invalid list (flagged by the merge)
        const float c = be * selw[r];
        const float f1 = al * (1.f - c);
        float* mp = Mh + size_t(slot) * dv + c4 * 4;
        const float4 m = ldcg4(mp);
        const float4 x = ld_v4<Tin>(vg + row * dv + c4 * 4);
        float4 y;
        y.x = fmaf(f1, m.x, c * x.x);
        y.y = fmaf(f1, m.y, c * x.y);
        y.z = fmaf(f1, m.z, c * x.z);
        y.w = fmaf(f1, m.w, c * x.w);
        *reinterpret_cast<float4*>(mp) = y;
      }
    }
    __syncthreads();
    // ---- 6. read after the write: thread tid sums the float4 column
    // c4 = tid % dv4 over its rows, then a fixed-order tree over threads
    {
      const int c4 = tid % dv4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int r = tid / dv4; r < p.R; r += kStepThreads / dv4) {
        const uint32_t slot = sels[p.W + r];
        if (slot >= uint32_t(p.N)) continue;
        const float u = selw[p.W + r];
        const float4 m = ldcg4(Mh + size_t(slot) * dv + c4 * 4);
        acc.x = fmaf(u, m.x, acc.x);
        acc.y = fmaf(u, m.y, acc.y);
        acc.z = fmaf(u, m.z, acc.z);
        acc.w = fmaf(u, m.w, acc.w);
      }
      for (int off = 16; off >= dv4; off >>= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
      }
      // lanes [0, dv4) now hold the warp's sums of columns 4 c4 .. 4 c4 + 3
      // (dv4 <= 32: every warp covers all dv columns)
      if (lane < dv4) {
        float* op = opart + size_t(warp) * dv + c4 * 4;
        op[0] = acc.x; op[1] = acc.y; op[2] = acc.z; op[3] = acc.w;
      }
    }
    __syncthreads();
    for (int c = tid; c < dv; c += kStepThreads) {
      float s = 0.f;
      for (int w = 0; w < kStepWarps; ++w) s += opart[size_t(w) * dv + c];
      io.o[row * dv + c] = s;
    }
    __syncthreads();
  }
}

bool step_supported(const Plan& p, size_t* smem) {
  const int epl = p.dtype == SDM_DTYPE_BF16 ? 8 : 4;
  if (p.n > kStepMaxN || p.k > kStepMaxK || p.dh % epl != 0) return false;
  const int lprw = p.dh / epl;
  if (lprw < 1 || lprw > 32 || (lprw & (lprw - 1))) return false;
  if (p.dv < 4 || p.dv > 128) return false;  // dv4 <= 32
  const size_t s = step_layout(p).total;
  if (smem) *smem = s;
  return s <= 227 * 1024;
}

template <typename Tin, int LPRW>
static cudaError_t launch_step_t(const Plan& p, const StepIO& io, size_t smem, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(k_step<Tin, LPRW>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_step<Tin, LPRW><<<p.BH, kStepThreads, smem, s>>>(p, io);
  return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_step_dt(const Plan& p, const StepIO& io, size_t smem, cudaStream_t s) {
  switch (p.dh / step_epl<Tin>()) {
    case 1: return launch_step_t<Tin, 1>(p, io, smem, s);
    case 2: return launch_step_t<Tin, 2>(p, io, smem, s);
    case 4: return launch_step_t<Tin, 4>(p, io, smem, s);
    case 8: return launch_step_t<Tin, 8>(p, io, smem, s);
    case 16: return launch_step_t<Tin, 16>(p, io, smem, s);
    case 32: return launch_step_t<Tin, 32>(p, io, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sdm

using namespace sdm;

extern "C" int sdm_step(const void* q, const void* k, const void* v, const float* alpha,
                        const float* beta, const void* C1, const void* C2, float* M_inout,
                        float* o_out, int32_t* idx_w, float* w_w, int32_t* idx_r, float* w_r,
                        const sdm_dims* dims, void* stream) {
  Plan p;
  int rc = make_plan(dims, &p);
  if (rc != SDM_OK) return rc;
  p.C = p.k;  // the half lists hold exactly k entries
  size_t smem = 0;
  if (!step_supported(p, &smem)) return SDM_ERR_UNSUPPORTED;
  if (p.T == 0) return SDM_OK;  // nothing to do; no pointer is read
  const void* ps[] = {q, k, v, C1, C2, M_inout, o_out};
  for (const void* x : ps) {
    if (!x) return SDM_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) & 15) return SDM_ERR_ALIGN;
  }
  for (const void* x : {static_cast<const void*>(alpha), static_cast<const void*>(beta)}) {
    if (!x) return SDM_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) & 3) return SDM_ERR_ALIGN;  // per-step scalars
  }
  const int nl = (idx_w != nullptr) + (w_w != nullptr) + (idx_r != nullptr) + (w_r != nullptr);
  if (nl != 0 && nl != 4) return SDM_ERR_NULL;
  StepIO io;
  io.q = q; io.k = k; io.v = v; io.alpha = alpha; io.beta = beta; io.C1 = C1; io.C2 = C2;
  io.M = M_inout; io.o = o_out;
  io.idx_w = idx_w; io.w_w = w_w; io.idx_r = idx_r; io.w_r = w_r;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = p.dtype == SDM_DTYPE_BF16
                            ? launch_step_dt<__nv_bfloat16>(p, io, smem, s)
                            : launch_step_dt<float>(p, io, smem, s);
  return e == cudaSuccess ? SDM_OK : SDM_ERR_CUDA;
}
