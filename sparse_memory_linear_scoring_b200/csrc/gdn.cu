// gdn.cu -- the dense Gated DeltaNet (GDN) recurrence, the baseline the SDM
// pages compare against ("Resultados": SDM trains 1.49x slower than GDN,
// attributed to HBM against SRAM traffic), at matched sizes.
//
// The rule (the SDM summaries' "Mecanismo Central" item 3 applied to a dense
// state; the delta-mem page, section 2.A, writes the same dense delta rule),
// per (b,h) head with S in R^{d_v x d_k}:
//     S~ = alpha_t S_{t-1};   S_t = S~ + beta_t (v_t - S~ k_t) k_t^T;   o_t = S_t q_t.
//
// Chunked evaluation (chunks of C = 64 steps).  Within a chunk let g_t be the
// running sum of log alpha from the chunk's first step (so alpha_1...alpha_t =
// exp(g_t)).  Row i of S evolves as s_t = alpha_t s_{t-1} + u_t k_t^T with the
// delta error u_t = beta_t (v_t - alpha_t s_{t-1} k_t); unrolling,
//     u_t = beta_t v_t - beta_t exp(g_t) (S_0 k_t) - sum_{j<t} A_tj u_j,
//     A_tj = beta_t exp(g_t - g_j) (k_t . k_j),
// so, for all rows at once, U = U~ - W S_0^T with (I + A) U~ = diag(beta) V and
// (I + A) W = diag(beta exp(g)) K (unit lower triangular solves), and
//     O = diag(exp(g)) Q S_0^T + P U,   P_tj = exp(g_t - g_j) (q_t . k_j), j <= t,
//     S_C = exp(g_last) S_0 + U^T diag(exp(g_last - g)) K.
// k_gdn_prep computes, per (head, chunk) and in parallel, everything that does
// not depend on S_0 (U~, W, P, Q~ = diag(exp(g)) Q, K~ = diag(exp(g_last - g)) K,
// exp(g_last)); rows past a partial last chunk are zero.  W, Q~ and P are
// stored transposed (step index fastest), which is how the scan reads them.
// k_gdn_scan then walks the chunks of one head in order for a block of RB = 4
// rows of S -- rows are independent under this rule -- and writes o and the
// final S.  Everything is float32 on CUDA cores; the state stays in shared memory.
#include <string.h>

#include "sdm_internal.cuh"

namespace sdm {

constexpr int kGdnC = 64;          // steps per chunk
constexpr int kGdnThreads = 256;
constexpr int kGdnRB = 4;          // rows of S per scan CTA (two warps per row)

struct GdnPlan {
  int B, H, T, dk, dv, dtype, BH, nch;
  size_t per_chunk;   // floats of prep output per (head, chunk)
  size_t oU, oW, oP, oQ, oK, oG;  // float offsets within a chunk's block
  size_t total;       // workspace bytes
};

static int gdn_plan(const sdm_gdn_dims* d, GdnPlan* p) {
  if (!d) return SDM_ERR_NULL;
  memset(p, 0, sizeof(*p));
  if (d->B < 1 || d->H < 1 || d->T < 0 ||
      (d->in_dtype != SDM_DTYPE_F32 && d->in_dtype != SDM_DTYPE_BF16))
    return SDM_ERR_DIMS;
  if ((long long)d->B * d->H > (1 << 24) || (long long)d->B * d->H * (long long)d->T > (1LL << 40))
    return SDM_ERR_DIMS;
  auto ok = [](int x) { return x == 16 || x == 32 || x == 64 || x == 128; };
  if (d->d_k < 1 || d->d_v < 1) return SDM_ERR_DIMS;
  if (!ok(d->d_k) || !ok(d->d_v)) return SDM_ERR_UNSUPPORTED;
  p->B = d->B; p->H = d->H; p->T = d->T; p->dk = d->d_k; p->dv = d->d_v;
  p->dtype = d->in_dtype;
  p->BH = d->B * d->H;
  p->nch = (d->T + kGdnC - 1) / kGdnC;
  const size_t C = kGdnC;
  size_t o = 0;
  p->oU = o; o += C * p->dv;
  p->oW = o; o += C * p->dk;
  p->oP = o; o += C * C;
  p->oQ = o; o += C * p->dk;
  p->oK = o; o += C * p->dk;
  p->oG = o; o += 4;
  p->per_chunk = (o + 3) & ~size_t(3);  // 16-byte blocks
  p->total = size_t(p->BH) * p->nch * p->per_chunk * 4;
  return SDM_OK;
}

template <typename Tin>
__device__ __forceinline__ float ldin(const Tin* p) { return to_f32(*p); }

// ---------------------------------------------------------------- prep
// smem: K, Q [C][dk+1], X [C][dv+dk] (U~ | W), A [C][C+1], g, beta [C]
__host__ __device__ inline size_t gdn_prep_smem(int dk, int dv) {
  return size_t(4) * (2 * kGdnC * (dk + 1) + kGdnC * (dv + dk) + kGdnC * (kGdnC + 1) + 2 * kGdnC);
}

template <typename Tin, int DK>
__global__ void __launch_bounds__(kGdnThreads)
k_gdn_prep(GdnPlan p, const Tin* __restrict__ q, const Tin* __restrict__ k,
           const Tin* __restrict__ v, const float* __restrict__ alpha,
           const float* __restrict__ beta, float* __restrict__ ws) {
  extern __shared__ __align__(16) float sm[];
  constexpr int dk = DK, dkp = DK + 1;
  const int dv = p.dv, Cp = kGdnC + 1, dx = dv + dk;
  float* Ks = sm;
  float* Qs = Ks + kGdnC * dkp;
  float* X = Qs + kGdnC * dkp;
  float* A = X + kGdnC * dx;
  float* g = A + kGdnC * Cp;
  float* bs = g + kGdnC;
  const int tid = threadIdx.x;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int t0 = c * kGdnC;
  const int L = min(kGdnC, p.T - t0);
  const size_t r0 = size_t(bh) * p.T + t0;
  float* out = ws + (size_t(bh) * p.nch + c) * p.per_chunk;
  // inputs; rows past L are zero
  for (int i = tid; i < kGdnC * dk; i += kGdnThreads) {
    const int t = i / dk, e = i - t * dk;
    Ks[t * dkp + e] = t < L ? ldin(k + (r0 + t) * dk + e) : 0.f;
    Qs[t * dkp + e] = t < L ? ldin(q + (r0 + t) * dk + e) : 0.f;
  }
  if (tid < kGdnC) {
    bs[tid] = tid < L ? beta[r0 + tid] : 0.f;
    g[tid] = tid < L ? logf(alpha[r0 + tid]) : 0.f;
  }
  __syncthreads();
  if (tid < 32) {  // inclusive running sum of log alpha (one warp, 2 per lane)
    float a0 = g[2 * tid], a1 = g[2 * tid + 1];
    float s = a0 + a1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, s, off);
      if (tid >= off) s += y;
    }
    const float ex = s - a0 - a1;  // sum over earlier lanes
    g[2 * tid] = ex + a0;
    g[2 * tid + 1] = ex + a0 + a1;
  }
  __syncthreads();
  // right-hand sides: X = [beta v | beta exp(g) k]
  for (int i = tid; i < kGdnC * dx; i += kGdnThreads) {
    const int t = i / dx, e = i - t * dx;
    float x = 0.f;
    if (t < L) {
      x = e < dv ? bs[t] * ldin(v + (r0 + t) * dv + e) : bs[t] * __expf(g[t]) * Ks[t * dkp + (e - dv)];
    }
    X[t * dx + e] = x;
  }
  // A (strictly lower) and P (lower with diagonal), one entry per thread
  for (int i = tid; i < kGdnC * kGdnC; i += kGdnThreads) {
    const int t = i / kGdnC, j = i - t * kGdnC;
    float a = 0.f, pq = 0.f;
    if (j <= t && t < L) {
      float skk = 0.f, sqk = 0.f;
#pragma unroll 16
      for (int e = 0; e < dk; ++e) {
        const float kj = Ks[j * dkp + e];
        skk = fmaf(Ks[t * dkp + e], kj, skk);
        sqk = fmaf(Qs[t * dkp + e], kj, sqk);
      }
      const float dec = __expf(g[t] - g[j]);
      a = j < t ? bs[t] * dec * skk : 0.f;
      pq = dec * sqk;
    }
    A[t * Cp + j] = a;
    out[p.oP + size_t(j) * kGdnC + t] = pq;  // transposed: [j][t]
  }
  __syncthreads();
  // (I + A) X = rhs by forward substitution, one thread per column
  for (int e = tid; e < dx; e += kGdnThreads) {
    for (int t = 1; t < L; ++t) {
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
      int j = 0;
      for (; j + 4 <= t; j += 4) {
        s0 = fmaf(A[t * Cp + j], X[j * dx + e], s0);
        s1 = fmaf(A[t * Cp + j + 1], X[(j + 1) * dx + e], s1);
        s2 = fmaf(A[t * Cp + j + 2], X[(j + 2) * dx + e], s2);
        s3 = fmaf(A[t * Cp + j + 3], X[(j + 3) * dx + e], s3);
      }
      for (; j < t; ++j) s0 = fmaf(A[t * Cp + j], X[j * dx + e], s0);
      X[t * dx + e] -= (s0 + s1) + (s2 + s3);
    }
  }
  __syncthreads();
  const float glast = L > 0 ? g[L - 1] : 0.f;
  for (int i = tid; i < kGdnC * dv; i += kGdnThreads) {
    const int t = i / dv, e = i - t * dv;
    out[p.oU + i] = X[t * dx + e];
  }
  for (int i = tid; i < kGdnC * dk; i += kGdnThreads) {
    const int t = i / dk, e = i - t * dk;
    out[p.oK + i] = t < L ? __expf(glast - g[t]) * Ks[t * dkp + e] : 0.f;  // [t][e]
    const int e2 = i / kGdnC, t2 = i - e2 * kGdnC;                           // [e][t]
    out[p.oW + i] = X[t2 * dx + dv + e2];
    out[p.oQ + i] = t2 < L ? __expf(g[t2]) * Qs[t2 * dkp + e2] : 0.f;
  }
  if (tid == 0) out[p.oG] = __expf(glast);
}

// ---------------------------------------------------------------- scan
// smem: S rows [RB][dk], U and o [C][RB], then one chunk's W^T, Q~^T [dk][C],
// K~ [C][dk], P^T [C][C], U~ rows [C][RB] (staged with cp.async, two stages
// when they fit).  One warp per row of the block (RB = 8 warps).
__host__ __device__ inline size_t gdn_stage_floats(int dk) {
  return size_t(3) * kGdnC * dk + size_t(kGdnC) * kGdnC + size_t(kGdnC) * kGdnRB + 4;
}
__host__ __device__ inline size_t gdn_scan_smem(int dk, int stages) {
  return size_t(4) * (kGdnRB * dk + 2 * kGdnC * kGdnRB + stages * gdn_stage_floats(dk));
}

__device__ __forceinline__ void cp16(float* dst, const float* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

template <int DK, int STAGES>
__global__ void __launch_bounds__(kGdnThreads)
k_gdn_scan(GdnPlan p, const float* __restrict__ ws, float* __restrict__ S, float* __restrict__ o) {
  extern __shared__ __align__(16) float sm[];
  constexpr int dk = DK;
  const int dv = p.dv;
  const int tid = threadIdx.x;
  const int rb = blockIdx.x, bh = blockIdx.y;
  const int i0 = rb * kGdnRB;  // first row of S
  float* Ss = sm;                      // [RB][dk]
  float* Us = Ss + kGdnRB * dk;        // [C][RB]
  float* Os = Us + kGdnC * kGdnRB;     // [C][RB]
  float* stg = Os + kGdnC * kGdnRB;    // STAGES x stage
  const size_t sf = gdn_stage_floats(dk);
  float* Sg = S + (size_t(bh) * dv + i0) * dk;
  for (int i = tid; i < kGdnRB * dk; i += kGdnThreads) Ss[i] = Sg[i];
  const float* wsh = ws + size_t(bh) * p.nch * p.per_chunk;
  // stage layout: W^T | Q~^T [dk][C], K~ [C][dk], P^T [C][C], U~ rows [C][RB], glast
  auto load = [&](int c, float* st) {
    const float* src = wsh + size_t(c) * p.per_chunk;
    const int n4 = kGdnC * dk / 4;
    for (int i = tid; i < n4; i += kGdnThreads) {
      cp16(st + 4 * i, src + p.oW + 4 * i);
      cp16(st + kGdnC * dk + 4 * i, src + p.oQ + 4 * i);
      cp16(st + 2 * kGdnC * dk + 4 * i, src + p.oK + 4 * i);
    }
    for (int i = tid; i < kGdnC * kGdnC / 4; i += kGdnThreads)
      cp16(st + 3 * kGdnC * dk + 4 * i, src + p.oP + 4 * i);
    // U~ columns i0 .. i0 + RB of every row: RB floats in 16-byte pieces
    for (int i = tid; i < kGdnC * (kGdnRB / 4); i += kGdnThreads) {
      const int t = i / (kGdnRB / 4), h4 = i - t * (kGdnRB / 4);
      cp16(st + 3 * kGdnC * dk + kGdnC * kGdnC + t * kGdnRB + 4 * h4,
           src + p.oU + size_t(t) * dv + i0 + 4 * h4);
    }
    if (tid == 0) cp16(st + 3 * kGdnC * dk + kGdnC * kGdnC + kGdnC * kGdnRB, src + p.oG);
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (p.nch > 0) load(0, stg);
  for (int c = 0; c < p.nch; ++c) {
    float* st = stg + (STAGES == 2 ? (c & 1) : 0) * sf;
    if (STAGES == 2 && c + 1 < p.nch) {
      // the other stage was last read in iteration c - 1, before its final barrier
      load(c + 1, stg + ((c + 1) & 1) * sf);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      // one stage: chunk c is loaded here, after iteration c - 1's final
      // barrier (chunk 0 was loaded above)
      if (STAGES == 1 && c > 0) load(c, stg);
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const float* Wt = st;                   // [dk][C]
    const float* Qt = st + kGdnC * dk;      // [dk][C]
    const float* Kt = st + 2 * kGdnC * dk;  // [C][dk]
    const float* Pt = st + 3 * kGdnC * dk;  // [C (j)][C (t)]
    const float* Ut = Pt + kGdnC * kGdnC;   // [C][RB]
    const float gl = Ut[kGdnC * kGdnRB];
    // warps 2r and 2r + 1 take row r of the block; each lane one step t.
    // U[t][r] = U~[t][r] - W[t] . S[r];  o[t][r] = Q~[t] . S[r] + sum_{j<=t} P[t][j] U[j][r]
    const int lane = tid & 31, r = tid >> 6, ts = ((tid >> 5) & 1) * 32 + lane;
    float su = 0.f, sq = 0.f;
#pragma unroll 16
    for (int e = 0; e < dk; ++e) {
      const float sv = Ss[r * dk + e];
      su = fmaf(Wt[e * kGdnC + ts], sv, su);
      sq = fmaf(Qt[e * kGdnC + ts], sv, sq);
    }
    Us[ts * kGdnRB + r] = Ut[ts * kGdnRB + r] - su;
    __syncthreads();
    // P is zero above its diagonal: lanes of the first warp of a row stop at 32
    if (ts < 32) {
#pragma unroll 16
      for (int jj = 0; jj < 32; ++jj) sq = fmaf(Pt[jj * kGdnC + ts], Us[jj * kGdnRB + r], sq);
    } else {
#pragma unroll 16
      for (int jj = 0; jj < kGdnC; ++jj) sq = fmaf(Pt[jj * kGdnC + ts], Us[jj * kGdnRB + r], sq);
    }
    Os[ts * kGdnRB + r] = sq;
    // S[r] = exp(g_last) S[r] + sum_t U[t][r] K~[t]
    for (int i = tid; i < kGdnRB * dk; i += kGdnThreads) {
      const int rr = i / dk, e = i - rr * dk;
      float acc = gl * Ss[i];
#pragma unroll 16
      for (int t = 0; t < kGdnC; ++t) acc = fmaf(Us[t * kGdnRB + rr], Kt[t * dk + e], acc);
      Ss[i] = acc;
    }
    __syncthreads();
    // o rows of the chunk: RB consecutive floats of each step
    const int t0 = c * kGdnC;
    for (int i = tid; i < kGdnC * kGdnRB; i += kGdnThreads) {
      const int t = i / kGdnRB, rr = i - t * kGdnRB;
      if (t0 + t < p.T) o[(size_t(bh) * p.T + t0 + t) * dv + i0 + rr] = Os[i];
    }
  }
  for (int i = tid; i < kGdnRB * dk; i += kGdnThreads) Sg[i] = Ss[i];
}

template <int DK>
static cudaError_t launch_gdn_dk(const GdnPlan& p, const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta, float* S, float* o,
                                 float* ws, size_t sp, size_t ss, int stages, dim3 gp, dim3 gs,
                                 cudaStream_t s) {
  cudaError_t e;
  if (p.dtype == SDM_DTYPE_BF16) {
    if ((e = cudaFuncSetAttribute(k_gdn_prep<__nv_bfloat16, DK>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, int(sp))) !=
        cudaSuccess)
      return e;
    k_gdn_prep<__nv_bfloat16, DK><<<gp, kGdnThreads, sp, s>>>(
        p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, alpha,
        beta, ws);
  } else {
    if ((e = cudaFuncSetAttribute(k_gdn_prep<float, DK>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, int(sp))) !=
        cudaSuccess)
      return e;
    k_gdn_prep<float, DK><<<gp, kGdnThreads, sp, s>>>(p, (const float*)q, (const float*)k,
                                                      (const float*)v, alpha, beta, ws);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (stages == 2) {
    if ((e = cudaFuncSetAttribute(k_gdn_scan<DK, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(ss))) != cudaSuccess)
      return e;
    k_gdn_scan<DK, 2><<<gs, kGdnThreads, ss, s>>>(p, ws, S, o);
  } else {
    if ((e = cudaFuncSetAttribute(k_gdn_scan<DK, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(ss))) != cudaSuccess)
      return e;
    k_gdn_scan<DK, 1><<<gs, kGdnThreads, ss, s>>>(p, ws, S, o);
  }
  return cudaGetLastError();
}

}  // namespace sdm

using namespace sdm;

extern "C" size_t sdm_gdn_workspace_bytes(const sdm_gdn_dims* dims) {
  GdnPlan p;
  if (gdn_plan(dims, &p) != SDM_OK) return 0;
  return p.total > 0 ? p.total : 16;
}

extern "C" int sdm_gdn_forward(const void* q, const void* k, const void* v, const float* alpha,
                               const float* beta, float* S_inout, float* o_out,
                               const sdm_gdn_dims* dims, void* workspace, size_t ws_bytes,
                               void* stream) {
  GdnPlan p;
  int rc = gdn_plan(dims, &p);
  if (rc != SDM_OK) return rc;
  if (p.T == 0) return SDM_OK;
  const void* ps[] = {q, k, v, S_inout, o_out, workspace};
  for (const void* x : ps) {
    if (!x) return x == workspace ? SDM_ERR_WORKSPACE : SDM_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) & 15) return SDM_ERR_ALIGN;
  }
  for (const void* x : {static_cast<const void*>(alpha), static_cast<const void*>(beta)}) {
    if (!x) return SDM_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) & 3) return SDM_ERR_ALIGN;  // per-step scalars
  }
  if (ws_bytes < p.total) return SDM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  const size_t sp = gdn_prep_smem(p.dk, p.dv);
  const int stages = gdn_scan_smem(p.dk, 2) <= 227 * 1024 ? 2 : 1;
  const size_t ss = gdn_scan_smem(p.dk, stages);
  if (sp > 227 * 1024 || ss > 227 * 1024) return SDM_ERR_UNSUPPORTED;
  dim3 gp(p.nch, p.BH);
  dim3 gs(p.dv / kGdnRB, p.BH);
  cudaError_t e;
  switch (p.dk) {
    case 16: e = launch_gdn_dk<16>(p, q, k, v, alpha, beta, S_inout, o_out, ws, sp, ss, stages, gp, gs, s); break;
    case 32: e = launch_gdn_dk<32>(p, q, k, v, alpha, beta, S_inout, o_out, ws, sp, ss, stages, gp, gs, s); break;
    case 64: e = launch_gdn_dk<64>(p, q, k, v, alpha, beta, S_inout, o_out, ws, sp, ss, stages, gp, gs, s); break;
    case 128: e = launch_gdn_dk<128>(p, q, k, v, alpha, beta, S_inout, o_out, ws, sp, ss, stages, gp, gs, s); break;
    default: return SDM_ERR_UNSUPPORTED;
  }
  if (e != cudaSuccess) return SDM_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SDM_OK : SDM_ERR_CUDA;
}
