// score_simt.cu -- sub-key scoring with CUDA cores and an exact per-half top-k.
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central" item 2: each half
// of k'_t / q'_t is scored against its sub-key codebook and keeps its top-k.
// This is the general path: any d_qk, n_sub <= 4096, float32 or bf16 inputs,
// float32 FMA accumulation.  It also serves the tensor-core path as its exact
// fallback for rows whose threshold filter did not bracket the k-th score.
//
// One warp per half-row.  Half-row r of a time chunk is
//   r = ((bh * Tc + tl) * 2 + side) * 2 + half,
// side 0 = key (write selection), 1 = query (read selection); half 0 = first
// d_qk/2 entries against C1, half 1 = last d_qk/2 against C2.  Output: the k
// best (score, row) pairs in descending (score, -row) order, count = k.
#include "sdm_internal.cuh"

namespace sdm {

constexpr int kScoreWarps = 4;

template <typename Tin>
__device__ __forceinline__ float dot_row(const float* __restrict__ xs, const Tin* __restrict__ row,
                                         int dh);

template <>
__device__ __forceinline__ float dot_row<float>(const float* __restrict__ xs,
                                                const float* __restrict__ row, int dh) {
  float acc = 0.f;
  if ((dh & 3) == 0) {
    const float4* r4 = reinterpret_cast<const float4*>(row);
    for (int c = 0; c < dh / 4; ++c) {
      const float4 v = __ldg(r4 + c);
      acc = fmaf(xs[4 * c + 0], v.x, acc);
      acc = fmaf(xs[4 * c + 1], v.y, acc);
      acc = fmaf(xs[4 * c + 2], v.z, acc);
      acc = fmaf(xs[4 * c + 3], v.w, acc);
    }
  } else {
    for (int c = 0; c < dh; ++c) acc = fmaf(xs[c], __ldg(row + c), acc);
  }
  return acc;
}

template <>
__device__ __forceinline__ float dot_row<__nv_bfloat16>(const float* __restrict__ xs,
                                                        const __nv_bfloat16* __restrict__ row,
                                                        int dh) {
  float acc = 0.f;
  if ((dh & 7) == 0) {
    const uint4* r8 = reinterpret_cast<const uint4*>(row);
    for (int c = 0; c < dh / 8; ++c) {
      const uint4 u = __ldg(r8 + c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(w[i] << 16);
        const float hi = __uint_as_float(w[i] & 0xffff0000u);
        acc = fmaf(xs[8 * c + 2 * i], lo, acc);
        acc = fmaf(xs[8 * c + 2 * i + 1], hi, acc);
      }
    }
  } else {
    for (int c = 0; c < dh; ++c) acc = fmaf(xs[c], __bfloat162float(row[c]), acc);
  }
  return acc;
}

__device__ __forceinline__ int pow2_at_least(int x) {
  int p = 2;
  while (p < x) p <<= 1;
  return p;
}

template <typename Tin>
__global__ void __launch_bounds__(kScoreWarps * 32)
k_score_simt(const Tin* __restrict__ q, const Tin* __restrict__ kk, const Tin* __restrict__ C1,
             const Tin* __restrict__ C2, Plan p, int t0, int tlen, const int* __restrict__ rows,
             const DevStatus* __restrict__ st_rows, int nrows, int* __restrict__ surv_cnt,
             uint2* __restrict__ surv) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = pow2_at_least(p.n);
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem) + size_t(warp) * S;
  float* xs = reinterpret_cast<float*>(reinterpret_cast<uint64_t*>(smem) + size_t(kScoreWarps) * S) +
              size_t(warp) * p.dh;
  const int count = rows ? st_rows->redo : nrows;
  for (int w = blockIdx.x * kScoreWarps + warp; w < count; w += gridDim.x * kScoreWarps) {
    const int r = rows ? rows[w] : w;
    const int half = r & 1, side = (r >> 1) & 1;
    const int tl = (r >> 2) % p.Tc, bh = (r >> 2) / p.Tc;
    if (tl >= tlen) continue;
    const int h = bh % p.H;
    const size_t t = size_t(bh) * p.T + t0 + tl;
    const Tin* x = (side ? q : kk) + t * p.dqk + size_t(half) * p.dh;
    const Tin* cb = (half ? C2 : C1) + size_t(h) * p.n * p.dh;
    for (int c = lane; c < p.dh; c += 32) xs[c] = to_f32(x[c]);
    __syncwarp();
    for (int j = lane; j < S; j += 32)
      keys[j] = (j < p.n) ? make_key(dot_row<Tin>(xs, cb + size_t(j) * p.dh, p.dh), uint32_t(j))
                          : uint64_t(0);
    __syncwarp();
    warp_sort_desc(keys, S);
    uint2* out = surv + size_t(r) * p.C;
    for (int i = lane; i < p.k; i += 32) {
      const uint64_t key = keys[i];
      out[i] = make_uint2(__float_as_uint(key_val(key)), key_idx(key));
    }
    if (lane == 0) surv_cnt[r] = p.k;
    __syncwarp();
  }
}

size_t score_simt_smem(const Plan& p) {
  int S = 2;
  while (S < p.n) S <<= 1;
  return size_t(kScoreWarps) * (size_t(S) * 8 + size_t(p.dh) * 4);
}

cudaError_t launch_score_simt(const Plan& p, const void* q, const void* k, const void* C1,
                              const void* C2, int t0, int tlen, const int* rows,
                              const DevStatus* st_rows, int* surv_cnt, uint2* surv,
                              DevStatus* st, cudaStream_t s) {
  (void)st;
  const size_t smem = score_simt_smem(p);
  const int nrows = p.BH * p.Tc * 4;
  int grid = rows ? 148 * 8 : (nrows + kScoreWarps - 1) / kScoreWarps;
  if (grid < 1) grid = 1;
  cudaError_t e;
  if (p.dtype == SDM_DTYPE_F32) {
    e = cudaFuncSetAttribute(k_score_simt<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    k_score_simt<float><<<grid, kScoreWarps * 32, smem, s>>>(
        (const float*)q, (const float*)k, (const float*)C1, (const float*)C2, p, t0, tlen, rows,
        st_rows, nrows, surv_cnt, surv);
  } else {
    e = cudaFuncSetAttribute(k_score_simt<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    k_score_simt<__nv_bfloat16><<<grid, kScoreWarps * 32, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)C1,
        (const __nv_bfloat16*)C2, p, t0, tlen, rows, st_rows, nrows, surv_cnt, surv);
  }
  return cudaGetLastError();
}

}  // namespace sdm
