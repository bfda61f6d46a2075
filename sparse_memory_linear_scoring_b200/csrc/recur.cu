// recur.cu -- the gated delta recurrence over the slot table (gather -> gate ->
// delta update -> scatter, and the sparse read).
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central":
//   item 3  for each write slot i of step t:  M~[i] = alpha_t * M[i];
//           M[i] = M~[i] + beta_t * w_i * (v_t - M~[i]), evaluated as
//           (1 - c) * M~[i] + c * v_t with c = beta_t * w_i;
//           all other slots are untouched;
//   item 4  o_t = sum_r u_r * M_t[r], read after step t's write.
//
// Work split.  Each (b,h) head is served by G CTAs; CTA g owns the slots whose
// hash falls in part g, so no two CTAs ever touch the same row.  A CTA walks
// the time blocks of the plan in order; inside a block its records are
// independent except for slots used several times, whose records form one
// chain handled in time order by a single thread group.  A slot row (d_v fp32)
// is moved whole by L = d_v/4 threads, 16 bytes each.  Read contributions are
// summed into a per-block shared accumulator and added to o once per block
// (with vector reductions when G > 1; o was zeroed by the plan kernel).
//
// Between blocks a CTA barrier orders this CTA's row stores before its next
// row loads; rows of other parts are never touched, so nothing else is needed.
#include "sdm_internal.cuh"

namespace sdm {

constexpr int kUnroll = 4;

__device__ __forceinline__ float4 ld_cg4(const float* ptr) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(ptr));
  return v;
}
__device__ __forceinline__ void st4(float* ptr, float4 v) {
  asm volatile("st.global.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(ptr), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void red_add4(float* ptr, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(ptr), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

template <typename Tv>
__device__ __forceinline__ void load_v4(const Tv* src, float* dst, int n);
template <>
__device__ __forceinline__ void load_v4<float>(const float* src, float* dst, int n) {
  for (int i = threadIdx.x; i < n / 4; i += blockDim.x)
    reinterpret_cast<float4*>(dst)[i] = __ldg(reinterpret_cast<const float4*>(src) + i);
}
template <>
__device__ __forceinline__ void load_v4<__nv_bfloat16>(const __nv_bfloat16* src, float* dst,
                                                       int n) {
  for (int i = threadIdx.x; i < n / 4; i += blockDim.x) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(src) + i);
    reinterpret_cast<float4*>(dst)[i] =
        make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                    __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
  }
}

__device__ __forceinline__ float4 gate_delta(float4 m, float alpha, float c, float4 v) {
  const float omc = 1.f - c;
  m.x = fmaf(c, v.x, omc * (alpha * m.x));
  m.y = fmaf(c, v.y, omc * (alpha * m.y));
  m.z = fmaf(c, v.z, omc * (alpha * m.z));
  m.w = fmaf(c, v.w, omc * (alpha * m.w));
  return m;
}

template <typename Tv, int L>
__global__ void __launch_bounds__(kRecurThreads)
k_recur(Plan p, const Tv* __restrict__ v, const float* __restrict__ alpha,
        const float* __restrict__ beta, float* __restrict__ M, float* __restrict__ o,
        const int4* __restrict__ rec, const int* __restrict__ roff, int t0, int tlen,
        DevStatus* st) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int dv = 4 * L;
  float* v_s = reinterpret_cast<float*>(smem);              // [P][dv]
  float* oacc = v_s + size_t(p.P) * dv;                       // [P][dv]
  float* al_s = oacc + size_t(p.P) * dv;                      // [P]
  float* be_s = al_s + p.P;                                   // [P]
  int* touched = reinterpret_cast<int*>(be_s + p.P);          // [P]

  const int part = blockIdx.x, bh = blockIdx.y;
  const int NG = kRecurThreads / L;
  const int grp = threadIdx.x / L, lg = threadIdx.x % L;
  float* Mh = M + size_t(bh) * size_t(p.N) * dv;
  const int nb = (tlen + p.P - 1) / p.P;

  for (int i = threadIdx.x; i < p.P * dv; i += blockDim.x) oacc[i] = 0.f;
  for (int i = threadIdx.x; i < p.P; i += blockDim.x) touched[i] = 0;

  for (int b = 0; b < nb; ++b) {
    const int s0 = b * p.P;
    const int np = min(p.P, tlen - s0);
    const size_t trow = size_t(bh) * p.T + t0 + s0;
    load_v4<Tv>(v + trow * dv, v_s, np * dv);
    for (int i = threadIdx.x; i < np; i += blockDim.x) {
      al_s[i] = __ldg(alpha + trow + i);
      be_s[i] = __ldg(beta + trow + i);
    }
    __syncthreads();
    const size_t blk = size_t(bh) * p.nblk + b;
    const int4* rb = rec + blk * p.E;
    const int r0 = __ldg(roff + blk * (p.G + 1) + part);
    const int r1 = __ldg(roff + blk * (p.G + 1) + part + 1);
    for (int i0 = r0 + grp; i0 < r1; i0 += NG * kUnroll) {
      int4 rc[kUnroll];
      float4 m[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = i0 + u * NG;
        rc[u] = (i < r1) ? __ldg(rb + i) : make_int4(0, 0, 0, 0);
        if (rc[u].w > 0 && (unsigned long long)(unsigned)rc[u].x >= (unsigned long long)p.N) {
          if (lg == 0) dev_flag(st, SDM_DEV_BAD_INDEX, rc[u].x);
          rc[u].w = 0;
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (rc[u].w > 0) m[u] = ld_cg4(Mh + size_t(unsigned(rc[u].x)) * dv + 4 * lg);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (rc[u].w <= 0) continue;
        const int i = i0 + u * NG;
        const int len = rc[u].w;
        bool wrote = false;
        float4 mv = m[u];
        for (int c = 0; c < len; ++c) {
          const int4 r = (c == 0) ? rc[u] : __ldg(rb + i + c);
          const int tl = r.y >> 1;
          const float wt = __int_as_float(r.z);
          if ((r.y & 1) == 0) {
            const float4 vv = *reinterpret_cast<const float4*>(v_s + tl * dv + 4 * lg);
            mv = gate_delta(mv, al_s[tl], be_s[tl] * wt, vv);
            wrote = true;
          } else {
            float* oa = oacc + tl * dv + 4 * lg;
            atomicAdd(oa + 0, wt * mv.x);
            atomicAdd(oa + 1, wt * mv.y);
            atomicAdd(oa + 2, wt * mv.z);
            atomicAdd(oa + 3, wt * mv.w);
            touched[tl] = 1;
          }
        }
        if (wrote) st4(Mh + size_t(unsigned(rc[u].x)) * dv + 4 * lg, mv);
      }
    }
    __syncthreads();
    // add this part's read contributions of the block into o
    float* ob = o + trow * dv;
    const int n4 = np * L;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) {
      const int tl = i / L;
      float4* a4 = reinterpret_cast<float4*>(oacc) + i;
      if (p.G == 1) {
        st4(ob + 4 * i, *a4);
      } else if (touched[tl]) {
        red_add4(ob + 4 * i, *a4);
      }
      *a4 = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < np; i += blockDim.x) touched[i] = 0;
  }
}

size_t recur_smem_bytes(const Plan& p) {
  return size_t(p.P) * p.dv * 4 * 2 + size_t(p.P) * 4 * 3;
}

template <typename Tv, int L>
static cudaError_t launch_recur_t(const Plan& p, const void* v, const float* alpha,
                                  const float* beta, float* M, float* o, const int4* rec,
                                  const int* roff, int t0, int tlen, DevStatus* st,
                                  cudaStream_t s) {
  const size_t smem = recur_smem_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(k_recur<Tv, L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(p.G, p.BH);
  k_recur<Tv, L><<<grid, kRecurThreads, smem, s>>>(p, (const Tv*)v, alpha, beta, M, o, rec, roff,
                                                    t0, tlen, st);
  return cudaGetLastError();
}

template <typename Tv>
static cudaError_t launch_recur_dt(const Plan& p, const void* v, const float* alpha,
                                   const float* beta, float* M, float* o, const int4* rec,
                                   const int* roff, int t0, int tlen, DevStatus* st,
                                   cudaStream_t s) {
  switch (p.dv) {
    case 4: return launch_recur_t<Tv, 1>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 8: return launch_recur_t<Tv, 2>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 16: return launch_recur_t<Tv, 4>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 32: return launch_recur_t<Tv, 8>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 64: return launch_recur_t<Tv, 16>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 128: return launch_recur_t<Tv, 32>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_recur(const Plan& p, const void* v, const float* alpha, const float* beta,
                         float* M, float* o, const int4* rec, const int* roff, int t0, int tlen,
                         DevStatus* st, cudaStream_t s) {
  if (p.dtype == SDM_DTYPE_F32)
    return launch_recur_dt<float>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
  return launch_recur_dt<__nv_bfloat16>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
}

}  // namespace sdm
