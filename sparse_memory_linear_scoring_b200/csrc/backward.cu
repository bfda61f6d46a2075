// backward.cu -- gradients of the SDM forward pass (training; the pages make the
// initial table M_0 a learned parameter, "Estado Inicial Aprendido").
//
// The pages give no backward pass.  The gradient is the derivative of the
// forward ("Mecanismo Central" items 2-4) with the discrete choices -- each
// half's top-k, the top-W / top-R candidates -- held at the ones the forward
// made (they are piecewise constant in the inputs).  Given do = dL/do and
// dM_T = dL/dM_T, for L a function of o and M_T:
//
//  * reverse recurrence, per slot, its records taken backward in time with
//    g = dL/dM[slot] (g starts at dM_T[slot]):
//      read  (u_r, step t):      g += u_r do_t;       du_r = M_t[slot] . do_t
//      write (c = beta_t w_i):   with m = M_{t-1}[slot] and M_t = alpha (1 - c) m + c v_t,
//                                dv_t += c g;   dc_i = g . (v_t - alpha_t m);
//                                dalpha_t += (1 - c) g . m;   g = alpha_t (1 - c) g;
//    and the g left after a slot's first record is dM_0[slot] (dM_T elsewhere);
//  * softmax: write side dw_i = beta_t dc_i, dbeta_t = sum_i w_i dc_i,
//    dscore_i = w_i (dw_i - sum_j w_j dw_j); read side dscore_r = u_r (du_r - sum u du);
//  * scores: a selected slot i1 * n + i2 scores s1[i1] + s2[i2], so its dscore
//    goes to row i1 of half 1 and row i2 of half 2; s_h[j] = x_h . C_h[j] gives
//    dx_h = sum_j ds_h[j] C_h[j] (into dk' or dq') and dC_h[j] += ds_h[j] x_h.
//
// The reverse recurrence needs the row values the forward saw (m, M_t[slot]).
// They are recomputed: the forward recurrence runs again from M_0, in the mode
// that stores, per record, the row it finds (launch_recur with snap); it reads
// a row from M_0 until it first writes the row into its working table, so M_0
// is never copied.  The plan's records already sort every slot's accesses by time inside
// a block, so the reverse kernel walks the same per-slot streams: blocks from
// last to first, each block's records from last to first, carrying g between
// blocks in dM_0's row.
#include <string.h>

#include "sdm_internal.cuh"

namespace sdm {

constexpr int kBwdThreads = 256;

struct BwdLayout {
  size_t off_status, off_rec, off_roff, off_rent, off_snap, off_g, off_ga, off_mw, off_touch,
      total;
};

static BwdLayout bwd_layout(const Plan& p) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  BwdLayout L;
  const size_t recs = size_t(p.BH) * p.nblk * p.E;
  const size_t ents = size_t(p.BH) * p.T * (p.W + p.R);
  size_t o = 0;
  L.off_status = o; o = al(o + sizeof(DevStatus));
  L.off_rec = o; o = al(o + recs * 16);
  L.off_roff = o; o = al(o + size_t(p.BH) * p.nblk * (p.NB + 1) * 4);
  L.off_rent = o; o = al(o + recs * 4);
  L.off_snap = o; o = al(o + recs * p.dv * 4);
  L.off_g = o; o = al(o + ents * 4);
  L.off_ga = o; o = al(o + ents * 4);
  L.off_mw = o; o = al(o + size_t(p.BH) * size_t(p.N) * p.dv * 4);
  L.off_touch = o; o = al(o + size_t(p.BH) * size_t(p.N));
  L.total = o;
  return L;
}

// the whole sequence is one time chunk of the plan
static int bwd_plan(const sdm_dims* d, Plan* p) {
  int rc = make_plan(d, p, ~size_t(0) >> 2);
  if (rc != SDM_OK) return rc;
  if (p->nchunks > 1) return SDM_ERR_UNSUPPORTED;
  return SDM_OK;
}

__global__ void k_bwd_init(const float4* __restrict__ dMT, float4* __restrict__ dM0,
                           size_t n4, float4* __restrict__ dv, size_t nv4,
                           float4* __restrict__ dC1, float4* __restrict__ dC2, size_t nc4) {
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride)
    dM0[i] = dMT ? dMT[i] : z;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nv4; i += stride) dv[i] = z;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nc4; i += stride) {
    dC1[i] = z;
    dC2[i] = z;
  }
}

template <typename Tv>
__device__ __forceinline__ float ldv(const Tv* p) { return to_f32(__ldg(p)); }

// two consecutive elements (the first at an even index) as float
__device__ __forceinline__ void ld2(const float* p, float& a, float& b) {
  const float2 v = __ldg(reinterpret_cast<const float2*>(p));
  a = v.x;
  b = v.y;
}
__device__ __forceinline__ void ld2(const __nv_bfloat16* p, float& a, float& b) {
  const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
  a = __uint_as_float(u << 16);
  b = __uint_as_float(u & 0xffff0000u);
}

// One stream (LPR lanes, F floats of a row each) per group of buckets, as in
// the forward recurrence; records backward.
template <typename Tv, int LPR, int F>
__global__ void __launch_bounds__(kBwdThreads)
k_recur_bwd(Plan p, const Tv* __restrict__ v, const float* __restrict__ alpha,
            const float* __restrict__ d_o, float* __restrict__ dv, float* __restrict__ dM,
            const int4* __restrict__ rec, const int* __restrict__ roff,
            const int* __restrict__ rent, const float* __restrict__ snap,
            float* __restrict__ gent, float* __restrict__ gal) {
  constexpr int dvw = LPR * F;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int stream = tid / LPR, sl = threadIdx.x % LPR;
  const unsigned gmask =
      LPR == 32 ? 0xffffffffu : (((1u << LPR) - 1u) << ((threadIdx.x & 31) / LPR * LPR));
  const int bh = stream / p.S, s = stream % p.S;
  if (bh >= p.BH) return;
  const int WR = p.W + p.R;
  const int g0 = s * p.mb, g1 = g0 + p.mb;
  float* dMh = dM + size_t(bh) * size_t(p.N) * dvw + sl * F;
  const size_t trow = size_t(bh) * p.T;
  auto reduce = [&](float x) {
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) x += __shfl_xor_sync(gmask, x, off, LPR);
    return x;
  };
  for (int blk = p.nblk - 1; blk >= 0; --blk) {
    const int* rr = roff + (size_t(bh) * p.nblk + blk) * (p.NB + 1);
    const int lo = __ldg(rr + g0), hi = __ldg(rr + g1);
    const size_t base = (size_t(bh) * p.nblk + blk) * p.E;
    float g[F];
    int cur_slot = -1;
    for (int pos = hi - 1; pos >= lo; --pos) {
      const int4 r = __ldg(rec + base + pos);
      if (r.x != cur_slot) {  // the last record of a slot run in this block
        cur_slot = r.x;
#pragma unroll
        for (int j = 0; j < F; ++j) g[j] = dMh[size_t(unsigned(r.x)) * dvw + j];
      }
      const int t = r.y >> 1;  // step within the (single) chunk
      const int e = __ldg(rent + base + pos);
      const int jj = e % WR;
      const size_t ent = (trow + t) * WR + jj;
      const float* m = snap + (base + pos) * dvw + sl * F;
      if (r.y & 1) {
        // read: g += u do_t; du = M_t[slot] . do_t
        const float u = __int_as_float(r.z);
        const float* dot = d_o + (trow + t) * dvw + sl * F;
        float du = 0.f;
#pragma unroll
        for (int j = 0; j < F; ++j) {
          const float dj = __ldg(dot + j);
          du = fmaf(__ldg(m + j), dj, du);
          g[j] = fmaf(u, dj, g[j]);
        }
        du = reduce(du);
        if (sl == 0) gent[ent] = du;
      } else {
        // write: M_t = f1 m + c v_t with f1 = alpha (1 - c)
        const float f1 = __int_as_float(r.z), c = __int_as_float(r.w);
        const float al = __ldg(alpha + trow + t);
        const Tv* vt = v + (trow + t) * dvw + sl * F;
        float* dvt = dv + (trow + t) * dvw + sl * F;
        float dc = 0.f, gm = 0.f;
#pragma unroll
        for (int j = 0; j < F; ++j) {
          const float mj = __ldg(m + j), vj = ldv(vt + j);
          dc = fmaf(g[j], vj - al * mj, dc);
          gm = fmaf(g[j], mj, gm);
          atomicAdd(dvt + j, c * g[j]);
          g[j] *= f1;
        }
        dc = reduce(dc);
        gm = reduce(gm);
        if (sl == 0) {
          gent[ent] = dc;
          gal[ent] = (1.f - c) * gm;
        }
      }
      // the first record of the slot's run in this block: g goes back to the row
      const int prev = pos > lo ? __ldg(&rec[base + pos - 1].x) : -1;
      if (prev != r.x) {
#pragma unroll
        for (int j = 0; j < F; ++j) dMh[size_t(unsigned(r.x)) * dvw + j] = g[j];
        cur_slot = -1;
      }
    }
  }
}

// One warp per (step, side): softmax backward, then the half scores' gradients
// into dk' / dq' and the codebooks.
template <typename Tin>
__global__ void __launch_bounds__(kBwdThreads)
k_sel_bwd(Plan p, const Tin* __restrict__ q, const Tin* __restrict__ k,
          const Tin* __restrict__ C1, const Tin* __restrict__ C2, const float* __restrict__ beta,
          const int32_t* __restrict__ idx_w, const float* __restrict__ w_w,
          const int32_t* __restrict__ idx_r, const float* __restrict__ w_r,
          const float* __restrict__ gent, const float* __restrict__ gal, float* __restrict__ dq,
          float* __restrict__ dk, float* __restrict__ dalpha, float* __restrict__ dbeta,
          float* __restrict__ dC1, float* __restrict__ dC2) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = kBwdThreads / 32;
  const int WR = p.W + p.R;
  const int Smax = p.W > p.R ? p.W : p.R;
  float* ds = reinterpret_cast<float*>(smem) + size_t(warp) * 2 * Smax;  // dscore, then merged
  int* rows = reinterpret_cast<int*>(ds + Smax);
  const size_t total = size_t(p.BH) * p.T * 2;
  for (size_t task = size_t(blockIdx.x) * nw + warp; task < total; task += size_t(gridDim.x) * nw) {
    const int side = int(task & 1);
    const size_t row = task >> 1;  // bh * T + t
    const int bh = int(row / p.T), h = bh % p.H;
    const int n_sel = side ? p.R : p.W;
    const int32_t* idx = (side ? idx_r : idx_w) + row * n_sel;
    const float* wt = (side ? w_r : w_w) + row * n_sel;
    const float* gg = gent + row * WR + (side ? p.W : 0);
    // softmax backward
    float sgw = 0.f, sdb = 0.f, sda = 0.f;
    const float be = side ? 0.f : beta[row];
    for (int j = lane; j < n_sel; j += 32) {
      const float dw = side ? gg[j] : be * gg[j];
      sgw = fmaf(wt[j], dw, sgw);
      if (!side) {
        sdb = fmaf(wt[j], gg[j], sdb);
        sda += gal[row * WR + j];
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      sgw += __shfl_xor_sync(0xffffffffu, sgw, off);
      sdb += __shfl_xor_sync(0xffffffffu, sdb, off);
      sda += __shfl_xor_sync(0xffffffffu, sda, off);
    }
    if (!side && lane == 0) {
      dbeta[row] = sdb;
      dalpha[row] = sda;
    }
    for (int j = lane; j < n_sel; j += 32) {
      const float dw = side ? gg[j] : be * gg[j];
      ds[j] = wt[j] * (dw - sgw);
    }
    __syncwarp();
    const Tin* x = (side ? q : k) + row * p.dqk;
    float* dx = (side ? dq : dk) + row * p.dqk;
    for (int half = 0; half < 2; ++half) {
      const Tin* C = (half ? C2 : C1) + size_t(h) * p.n * p.dh;
      float* dC = (half ? dC2 : dC1) + size_t(h) * p.n * p.dh;
      for (int j = lane; j < n_sel; j += 32) {
        const uint32_t slot = uint32_t(idx[j]);
        rows[j] = int(half ? slot % uint32_t(p.n) : slot / uint32_t(p.n));
      }
      __syncwarp();
      // dx_h = sum_j ds_j C_h[row_j] (two columns per lane when d_h is even)
      if ((p.dh & 1) == 0) {
        for (int c = 2 * lane; c < p.dh; c += 64) {
          float a0 = 0.f, a1 = 0.f;
          for (int j = 0; j < n_sel; ++j) {
            float c0, c1;
            ld2(C + size_t(rows[j]) * p.dh + c, c0, c1);
            a0 = fmaf(ds[j], c0, a0);
            a1 = fmaf(ds[j], c1, a1);
          }
          dx[half * p.dh + c] = a0;
          dx[half * p.dh + c + 1] = a1;
        }
      } else {
        for (int c = lane; c < p.dh; c += 32) {
          float acc = 0.f;
          for (int j = 0; j < n_sel; ++j)
            acc = fmaf(ds[j], to_f32(C[size_t(rows[j]) * p.dh + c]), acc);
          dx[half * p.dh + c] = acc;
        }
      }
      // dC_h[row] += (sum of ds over the entries on that row) x_h: within each
      // group of 32 entries, one update per distinct row (its lowest lane sums
      // the group's entries on that row)
      for (int j0 = 0; j0 < n_sel; j0 += 32) {
        const int j = j0 + lane;
        const bool valid = j < n_sel;
        const int rj = valid ? rows[j] : -1 - lane;
        const unsigned peers = __match_any_sync(0xffffffffu, rj);
        const bool lead = valid && __ffs(peers) - 1 == lane;
        float sum = 0.f;
        if (lead) {
          for (unsigned m = peers; m; m &= m - 1) sum += ds[j0 + __ffs(m) - 1];
        }
        unsigned m = __ballot_sync(0xffffffffu, lead);
        while (m) {
          const int src = __ffs(m) - 1;
          m &= m - 1;
          const int rs = __shfl_sync(0xffffffffu, rj, src);
          const float sj = __shfl_sync(0xffffffffu, sum, src);
          for (int c = lane; c < p.dh; c += 32)
            atomicAdd(dC + size_t(rs) * p.dh + c, sj * to_f32(x[half * p.dh + c]));
        }
      }
      __syncwarp();
    }
  }
}

template <typename Tv, int DV>
static cudaError_t launch_bwd_w(const Plan& p, const void* v, const float* alpha,
                                const float* d_o, float* dv, float* dM, const int4* rec,
                                const int* roff, const int* rent, const float* snap, float* gent,
                                float* gal, cudaStream_t s) {
#ifndef SDM_BWD_LANE_FLOATS
#define SDM_BWD_LANE_FLOATS 2  // floats per lane = this x d_v / 32: two streams per warp at d_v = 64
#endif
  constexpr int F0 = SDM_BWD_LANE_FLOATS * DV / 32;
  constexpr int F = F0 >= 1 ? (F0 > 8 ? 8 : F0) : 1;
  constexpr int LPR = DV / F;
  static_assert(LPR <= 32 && (32 % LPR) == 0, "lanes per row");
  const long long threads = (long long)p.BH * p.S * LPR;
  const int grid = int((threads + kBwdThreads - 1) / kBwdThreads);
  k_recur_bwd<Tv, LPR, F><<<grid, kBwdThreads, 0, s>>>(p, (const Tv*)v, alpha, d_o, dv, dM, rec,
                                                       roff, rent, snap, gent, gal);
  return cudaGetLastError();
}

template <typename Tv>
static cudaError_t launch_bwd_dt(const Plan& p, const void* v, const float* alpha,
                                 const float* d_o, float* dv, float* dM, const int4* rec,
                                 const int* roff, const int* rent, const float* snap,
                                 float* gent, float* gal, cudaStream_t s) {
  switch (p.dv) {
    case 4: return launch_bwd_w<Tv, 4>(p, v, alpha, d_o, dv, dM, rec, roff, rent, snap, gent, gal, s);
    case 8: return launch_bwd_w<Tv, 8>(p, v, alpha, d_o, dv, dM, rec, roff, rent, snap, gent, gal, s);
    case 16: return launch_bwd_w<Tv, 16>(p, v, alpha, d_o, dv, dM, rec, roff, rent, snap, gent, gal, s);
    case 32: return launch_bwd_w<Tv, 32>(p, v, alpha, d_o, dv, dM, rec, roff, rent, snap, gent, gal, s);
    case 64: return launch_bwd_w<Tv, 64>(p, v, alpha, d_o, dv, dM, rec, roff, rent, snap, gent, gal, s);
    case 128: return launch_bwd_w<Tv, 128>(p, v, alpha, d_o, dv, dM, rec, roff, rent, snap, gent, gal, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sdm

using namespace sdm;

extern "C" size_t sdm_backward_workspace_bytes(const sdm_dims* dims) {
  Plan p;
  if (bwd_plan(dims, &p) != SDM_OK) return 0;
  return bwd_layout(p).total;
}

extern "C" int sdm_backward(const void* q, const void* k, const void* v, const float* alpha,
                            const float* beta, const void* C1, const void* C2, const float* M0,
                            const int32_t* idx_w, const float* w_w, const int32_t* idx_r,
                            const float* w_r, const float* d_o, const float* dM_T, float* dq,
                            float* dk, float* dv, float* dalpha, float* dbeta, float* dC1,
                            float* dC2, float* dM0, const sdm_dims* dims, void* workspace,
                            size_t ws_bytes, void* stream) {
  Plan p;
  int rc = bwd_plan(dims, &p);
  if (rc != SDM_OK) return rc;
  if (p.T == 0) return SDM_OK;
  const void* need16[] = {q, k, v, C1, C2, M0, idx_w, w_w, idx_r, w_r, d_o,
                          dq, dk, dv, dC1, dC2, dM0, workspace};
  for (const void* x : need16) {
    if (!x) return x == workspace ? SDM_ERR_WORKSPACE : SDM_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) & 15) return SDM_ERR_ALIGN;
  }
  if (dM_T && (reinterpret_cast<uintptr_t>(dM_T) & 15)) return SDM_ERR_ALIGN;
  for (const void* x : {static_cast<const void*>(alpha), static_cast<const void*>(beta),
                        static_cast<const void*>(dalpha), static_cast<const void*>(dbeta)}) {
    if (!x) return SDM_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) & 3) return SDM_ERR_ALIGN;
  }
  const BwdLayout L = bwd_layout(p);
  if (ws_bytes < L.total) return SDM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(workspace);
  DevStatus* st = reinterpret_cast<DevStatus*>(w + L.off_status);
  int4* rec = reinterpret_cast<int4*>(w + L.off_rec);
  int* roff = reinterpret_cast<int*>(w + L.off_roff);
  int* rent = reinterpret_cast<int*>(w + L.off_rent);
  float* snap = reinterpret_cast<float*>(w + L.off_snap);
  float* gent = reinterpret_cast<float*>(w + L.off_g);
  float* gal = reinterpret_cast<float*>(w + L.off_ga);
  float* Mw = reinterpret_cast<float*>(w + L.off_mw);
  uint8_t* touched = reinterpret_cast<uint8_t*>(w + L.off_touch);
  if (launch_init(p, st, s) != cudaSuccess) return SDM_ERR_CUDA;
  // dM_0 = dM_T (or 0; nothing to copy when dM0 is dM_T itself), dv = dC = 0,
  // no row of the working table written yet
  if (cudaMemsetAsync(touched, 0, size_t(p.BH) * size_t(p.N), s) != cudaSuccess)
    return SDM_ERR_CUDA;
  {
    const size_t n4 = size_t(p.BH) * size_t(p.N) * p.dv / 4;
    const size_t nv4 = size_t(p.BH) * p.T * p.dv / 4;
    const size_t nc4 = size_t(p.H) * p.n * p.dh / 4;
    k_bwd_init<<<148 * 8, 256, 0, s>>>(
        reinterpret_cast<const float4*>(dM_T), reinterpret_cast<float4*>(dM0),
        static_cast<const void*>(dM_T) == static_cast<const void*>(dM0) ? 0 : n4,
        reinterpret_cast<float4*>(dv), nv4, reinterpret_cast<float4*>(dC1),
        reinterpret_cast<float4*>(dC2), p.dh % 4 == 0 ? nc4 : 0);
    if (cudaGetLastError() != cudaSuccess) return SDM_ERR_CUDA;
    if (p.dh % 4 != 0) {
      if (cudaMemsetAsync(dC1, 0, size_t(p.H) * p.n * p.dh * 4, s) != cudaSuccess ||
          cudaMemsetAsync(dC2, 0, size_t(p.H) * p.n * p.dh * 4, s) != cudaSuccess)
        return SDM_ERR_CUDA;
    }
  }
  // plan of the whole sequence from the given lists, with each record's entry
  PlanIO pio;
  memset(&pio, 0, sizeof(pio));
  pio.iw = idx_w; pio.ww = w_w; pio.ir = idx_r; pio.wr = w_r;
  pio.list_T = p.T;
  pio.list_t0 = 0;
  pio.validate = 1;
  pio.alpha = alpha;
  pio.beta = beta;
  pio.rec = rec;
  pio.roff = roff;
  pio.o = nullptr;
  pio.rent = rent;
  if (launch_plan(p, pio, 0, p.T, st, s) != cudaSuccess) return SDM_ERR_CUDA;
  // the forward recurrence again from M_0, saving the rows each record sees
  if (launch_recur(p, v, Mw, nullptr, rec, roff, 0, p.T, s,
                   SaveIO{snap, static_cast<const float*>(M0), touched}) != cudaSuccess)
    return SDM_ERR_CUDA;
  // reverse recurrence
  cudaError_t e = p.dtype == SDM_DTYPE_F32
                      ? launch_bwd_dt<float>(p, v, alpha, d_o, dv, dM0, rec, roff, rent, snap,
                                             gent, gal, s)
                      : launch_bwd_dt<__nv_bfloat16>(p, v, alpha, d_o, dv, dM0, rec, roff, rent,
                                                     snap, gent, gal, s);
  if (e != cudaSuccess) return SDM_ERR_CUDA;
  // selection and scores
  {
    const int Smax = p.W > p.R ? p.W : p.R;
    const size_t smem = size_t(kBwdThreads / 32) * 2 * Smax * 4;
    if (smem > 227 * 1024) return SDM_ERR_UNSUPPORTED;
    const size_t tasks = size_t(p.BH) * p.T * 2;
    long long grid = (long long)((tasks + 7) / 8);
    if (grid > 148 * 16) grid = 148 * 16;
    if (p.dtype == SDM_DTYPE_F32) {
      if (cudaFuncSetAttribute(k_sel_bwd<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem)) != cudaSuccess)
        return SDM_ERR_CUDA;
      k_sel_bwd<float><<<int(grid), kBwdThreads, smem, s>>>(
          p, (const float*)q, (const float*)k, (const float*)C1, (const float*)C2, beta, idx_w,
          w_w, idx_r, w_r, gent, gal, dq, dk, dalpha, dbeta, dC1, dC2);
    } else {
      if (cudaFuncSetAttribute(k_sel_bwd<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem)) != cudaSuccess)
        return SDM_ERR_CUDA;
      k_sel_bwd<__nv_bfloat16><<<int(grid), kBwdThreads, smem, s>>>(
          p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)C1,
          (const __nv_bfloat16*)C2, beta, idx_w, w_w, idx_r, w_r, gent, gal, dq, dk, dalpha,
          dbeta, dC1, dC2);
    }
    if (cudaGetLastError() != cudaSuccess) return SDM_ERR_CUDA;
  }
  return SDM_OK;
}
