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
// is moved whole by L threads holding F = 4 or 8 floats each.  A block's
// records come in three runs: writes of slots used once in the block, reads of
// slots used once, and chains of slots used several times; the two single-use
// runs are branch-free gathers (write: gate + delta + scatter; read: weight +
// vector reduction into o, which the plan kernel zeroed).  The next block's
// records, v rows and gates are prefetched with cp.async while a block runs.
//
// Between blocks a CTA barrier orders this CTA's row stores before its next
// row loads; rows of other parts are never touched, so nothing else is needed.
#include "sdm_internal.cuh"

namespace sdm {


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

// cp.async of n bytes (a multiple of 4) from global to shared memory, in 16-,
// 8- or 4-byte pieces as the alignment of both ends allows.
__device__ __forceinline__ void async_copy(void* dst, const void* src, int nbytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  const uintptr_t sa = reinterpret_cast<uintptr_t>(src);
  const int al = int((sa | d | uintptr_t(nbytes)) & 15);
  if (al == 0) {
    for (int i = threadIdx.x * 16; i < nbytes; i += blockDim.x * 16)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + i), "l"(sa + i)
                   : "memory");
  } else if ((al & 7) == 0) {
    for (int i = threadIdx.x * 8; i < nbytes; i += blockDim.x * 8)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d + i), "l"(sa + i)
                   : "memory");
  } else {
    for (int i = threadIdx.x * 4; i < nbytes; i += blockDim.x * 4)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d + i), "l"(sa + i)
                   : "memory");
  }
}
__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void async_wait_prev() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

template <typename Tv>
__device__ __forceinline__ float4 v4_of(const Tv* row);
template <>
__device__ __forceinline__ float4 v4_of<float>(const float* row) {
  return *reinterpret_cast<const float4*>(row);
}
template <>
__device__ __forceinline__ float4 v4_of<__nv_bfloat16>(const __nv_bfloat16* row) {
  const uint2 u = *reinterpret_cast<const uint2*>(row);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

// F consecutive floats of a staged v row as fp32
template <typename Tv, int F>
__device__ __forceinline__ void v_row(const Tv* row, float* out);
template <>
__device__ __forceinline__ void v_row<float, 4>(const float* row, float* out) {
  const float4 a = *reinterpret_cast<const float4*>(row);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
}
template <>
__device__ __forceinline__ void v_row<float, 8>(const float* row, float* out) {
  const float4 a = reinterpret_cast<const float4*>(row)[0];
  const float4 b = reinterpret_cast<const float4*>(row)[1];
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}
__device__ __forceinline__ void bf16x2(uint32_t u, float* out) {
  out[0] = __uint_as_float(u << 16);
  out[1] = __uint_as_float(u & 0xffff0000u);
}
template <>
__device__ __forceinline__ void v_row<__nv_bfloat16, 4>(const __nv_bfloat16* row, float* out) {
  const uint2 u = *reinterpret_cast<const uint2*>(row);
  bf16x2(u.x, out);
  bf16x2(u.y, out + 2);
}
template <>
__device__ __forceinline__ void v_row<__nv_bfloat16, 8>(const __nv_bfloat16* row, float* out) {
  const uint4 u = *reinterpret_cast<const uint4*>(row);
  bf16x2(u.x, out);
  bf16x2(u.y, out + 2);
  bf16x2(u.z, out + 4);
  bf16x2(u.w, out + 6);
}

template <int F>
__device__ __forceinline__ void ld_row(const float* ptr, float* m) {
#pragma unroll
  for (int j = 0; j < F / 4; ++j) {
    const float4 x = ld_cg4(ptr + 4 * j);
    m[4 * j] = x.x; m[4 * j + 1] = x.y; m[4 * j + 2] = x.z; m[4 * j + 3] = x.w;
  }
}
template <int F>
__device__ __forceinline__ void st_row(float* ptr, const float* m) {
#pragma unroll
  for (int j = 0; j < F / 4; ++j)
    st4(ptr + 4 * j, make_float4(m[4 * j], m[4 * j + 1], m[4 * j + 2], m[4 * j + 3]));
}
template <int F>
__device__ __forceinline__ void red_row(float* ptr, const float* m, float u) {
#pragma unroll
  for (int j = 0; j < F / 4; ++j)
    red_add4(ptr + 4 * j, make_float4(u * m[4 * j], u * m[4 * j + 1], u * m[4 * j + 2],
                                      u * m[4 * j + 3]));
}
// M~ = alpha m;  M = (1 - c) M~ + c v,  c = beta w  (as alpha (1 - c) m + c v)
template <int F>
__device__ __forceinline__ void gate_delta(float* m, float alpha, float c, const float* vv) {
  const float a = alpha * (1.f - c);
#pragma unroll
  for (int j = 0; j < F; ++j) m[j] = fmaf(a, m[j], c * vv[j]);
}

struct RecurLayout {
  size_t roff, rec, v, ab, total;
};

// Records of one (block, part) staged in shared memory; a part with more
// records in a block reads the rest from global memory.
constexpr int kRecStage = 512;

__host__ __device__ inline RecurLayout recur_layout(const Plan& p) {
  RecurLayout L;
  const size_t vb = (p.dtype == SDM_DTYPE_F32 ? 4 : 2);
  size_t o = 0;
  L.roff = o; o += ((size_t(p.nblk) + 1) * 16 + 15) & ~size_t(15);
  L.rec = o; o += size_t(2) * kRecStage * 16;
  L.v = o; o += (size_t(2) * p.P * p.dv * vb + 15) & ~size_t(15);
  L.ab = o; o += size_t(2) * 2 * p.P * 4;
  L.total = o;
  return L;
}

template <typename Tv, int F, int L>
__global__ void __launch_bounds__(kRecurThreads, 2)
k_recur(Plan p, const Tv* __restrict__ v, const float* __restrict__ alpha,
        const float* __restrict__ beta, float* __restrict__ M, float* __restrict__ o,
        const int4* __restrict__ rec, const int* __restrict__ roff, int t0, int tlen,
        DevStatus* st) {
  extern __shared__ __align__(16) unsigned char smem[];
  const RecurLayout Y = recur_layout(p);
  constexpr int dv = F * L;
  int* roff_s = reinterpret_cast<int*>(smem + Y.roff);   // [nb][4]
  int4* rec_s = reinterpret_cast<int4*>(smem + Y.rec);   // [2][kRecStage]
  Tv* v_s = reinterpret_cast<Tv*>(smem + Y.v);           // [2][P][dv]
  float* ab_s = reinterpret_cast<float*>(smem + Y.ab);   // [2][alpha P | beta P]

  const int part = blockIdx.x, bh = blockIdx.y;
  constexpr int NG = kRecurThreads / L;
  constexpr int kUnroll = kRecurUnroll * 4 / F;  // rows in flight per thread: 4*kRecurUnroll floats
  const int grp = threadIdx.x / L, lg = threadIdx.x % L;
  float* Mh = M + size_t(bh) * size_t(p.N) * dv + lg * F;
  const int nb = (tlen + p.P - 1) / p.P;

  // this part's [writes, reads, chains, end) record offsets in every block
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    const int* ro = roff + (size_t(bh) * p.nblk + b) * (3 * p.G + 1) + 3 * part;
#pragma unroll
    for (int j = 0; j < 4; ++j) roff_s[4 * b + j] = __ldg(ro + j);
  }
  __syncthreads();

  auto prefetch = [&](int b) {
    const int buf = b & 1;
    const int s0 = b * p.P;
    const int np = min(p.P, tlen - s0);
    const size_t trow = size_t(bh) * p.T + t0 + s0;
    const size_t blk = size_t(bh) * p.nblk + b;
    const int w0 = roff_s[4 * b];
    const int nr = min(roff_s[4 * b + 3] - w0, kRecStage);
    if (nr > 0) async_copy(rec_s + buf * kRecStage, rec + blk * p.E + w0, nr * 16);
    async_copy(v_s + size_t(buf) * p.P * dv, v + trow * dv, int(np * dv * sizeof(Tv)));
    async_copy(ab_s + buf * 2 * p.P, alpha + trow, np * 4);
    async_copy(ab_s + buf * 2 * p.P + p.P, beta + trow, np * 4);
  };

  prefetch(0);
  async_commit();
  for (int b = 0; b < nb; ++b) {
    if (b + 1 < nb) prefetch(b + 1);
    async_commit();
    async_wait_prev();
    __syncthreads();
    const int buf = b & 1;
    const size_t trow = size_t(bh) * p.T + t0 + size_t(b) * p.P;
    const int w0 = roff_s[4 * b];
    const int nw = roff_s[4 * b + 1] - w0;   // single-use writes [0, nw)
    const int nr = roff_s[4 * b + 2] - w0;   // single-use reads  [nw, nr)
    const int ne = roff_s[4 * b + 3] - w0;   // chains            [nr, ne)
    const int4* rg = rec + (size_t(bh) * p.nblk + b) * p.E + w0;
    const int4* rs = rec_s + buf * kRecStage;
    const Tv* vb = v_s + size_t(buf) * p.P * dv + lg * F;
    const float* al_s = ab_s + buf * 2 * p.P;
    const float* be_s = al_s + p.P;
    float* ob = o + trow * dv + lg * F;
    auto get_rec = [&](int i) -> int4 { return i < kRecStage ? rs[i] : __ldg(rg + i); };
    auto slot_ok = [&](int s) -> bool {
      if ((unsigned long long)(unsigned)s < (unsigned long long)p.N) return true;
      if (lg == 0) dev_flag(st, SDM_DEV_BAD_INDEX, s);
      return false;
    };

    // single-use writes: gather, gate, delta, scatter
    for (int i0 = grp; i0 < nw; i0 += NG * kUnroll) {
      int slot[kUnroll], meta[kUnroll];
      float wt[kUnroll], m[kUnroll][F];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = i0 + u * NG;
        slot[u] = -1;
        if (i < nw) {
          const int4 r = get_rec(i);
          if (slot_ok(r.x)) { slot[u] = r.x; meta[u] = r.y; wt[u] = __int_as_float(r.z); }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (slot[u] >= 0) ld_row<F>(Mh + size_t(unsigned(slot[u])) * dv, m[u]);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (slot[u] < 0) continue;
        const int tl = meta[u] >> 1;
        float vv[F];
        v_row<Tv, F>(vb + tl * dv, vv);
        gate_delta<F>(m[u], al_s[tl], be_s[tl] * wt[u], vv);
        st_row<F>(Mh + size_t(unsigned(slot[u])) * dv, m[u]);
      }
    }
    // single-use reads: gather, weight, reduce into o
    for (int i0 = nw + grp; i0 < nr; i0 += NG * kUnroll) {
      int slot[kUnroll], meta[kUnroll];
      float wt[kUnroll], m[kUnroll][F];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = i0 + u * NG;
        slot[u] = -1;
        if (i < nr) {
          const int4 r = get_rec(i);
          if (slot_ok(r.x)) { slot[u] = r.x; meta[u] = r.y; wt[u] = __int_as_float(r.z); }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (slot[u] >= 0) ld_row<F>(Mh + size_t(unsigned(slot[u])) * dv, m[u]);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (slot[u] >= 0) red_row<F>(ob + size_t(meta[u] >> 1) * dv, m[u], wt[u]);
    }
    // slots used several times in the block: one chain each, in time order
    for (int i = nr + grp; i < ne; i += NG) {
      const int4 r0 = get_rec(i);
      if (r0.w <= 0 || !slot_ok(r0.x)) continue;
      float m[F];
      ld_row<F>(Mh + size_t(unsigned(r0.x)) * dv, m);
      bool wrote = false;
      for (int c = 0; c < r0.w; ++c) {
        const int4 r = c == 0 ? r0 : get_rec(i + c);
        const int tl = r.y >> 1;
        const float w = __int_as_float(r.z);
        if ((r.y & 1) == 0) {
          float vv[F];
          v_row<Tv, F>(vb + tl * dv, vv);
          gate_delta<F>(m, al_s[tl], be_s[tl] * w, vv);
          wrote = true;
        } else {
          red_row<F>(ob + size_t(tl) * dv, m, w);
        }
      }
      if (wrote) st_row<F>(Mh + size_t(unsigned(r0.x)) * dv, m);
    }
    __syncthreads();
  }
  async_wait_prev();
}

size_t recur_smem_bytes(const Plan& p) { return recur_layout(p).total; }

template <typename Tv, int F, int L>
static cudaError_t launch_recur_t(const Plan& p, const void* v, const float* alpha,
                                  const float* beta, float* M, float* o, const int4* rec,
                                  const int* roff, int t0, int tlen, DevStatus* st,
                                  cudaStream_t s) {
  const size_t smem = recur_smem_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(k_recur<Tv, F, L>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(p.G, p.BH);
  k_recur<Tv, F, L><<<grid, kRecurThreads, smem, s>>>(p, (const Tv*)v, alpha, beta, M, o, rec,
                                                       roff, t0, tlen, st);
  return cudaGetLastError();
}

// A row of d_v floats is moved by L threads holding F = 4 or 8 floats each.
template <typename Tv>
static cudaError_t launch_recur_dt(const Plan& p, const void* v, const float* alpha,
                                   const float* beta, float* M, float* o, const int4* rec,
                                   const int* roff, int t0, int tlen, DevStatus* st,
                                   cudaStream_t s) {
  switch (p.dv) {
    case 4: return launch_recur_t<Tv, 4, 1>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 8: return launch_recur_t<Tv, 4, 2>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 16: return launch_recur_t<Tv, 4, 4>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 32: return launch_recur_t<Tv, 8, 4>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 64: return launch_recur_t<Tv, 8, 8>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
    case 128: return launch_recur_t<Tv, 8, 16>(p, v, alpha, beta, M, o, rec, roff, t0, tlen, st, s);
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
