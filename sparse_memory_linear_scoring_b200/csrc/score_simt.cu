// score_simt.cu -- sub-key scoring with CUDA cores and an exact per-half top-k.
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central" item 2: each half
// of k'_t / q'_t is scored against its sub-key codebook and keeps its top-k.
// This is the general path: any d_qk, n_sub <= 4096, float32 or bf16 inputs,
// float32 FMA accumulation.  It also serves the tensor-core path as its exact
// fallback for rows whose threshold filter did not bracket the k-th score.
//
// One warp per half-row (two kernels: k_score_warp for d_h = 32, 64, 128 or 256
// and n_sub <= 1024, k_score_simt for everything else).  Half-row r of a time
// chunk is
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

__host__ __device__ __forceinline__ int pow2_at_least(int x) {
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

// ---- k_score_warp: the half-row's x and the scores stay in registers.
// Lane l holds dims [l*DPL, (l+1)*DPL) of x; codebook rows are read whole by
// the warp (one coalesced load per row), 32 rows at a time, and a butterfly
// across lanes leaves row g*32 + l's score in lane l (register g).  The k-th
// largest score is found by a most-significant-bit-first search over the
// order-preserving 32-bit images; the k best (ties: lower row first) are then
// sorted in shared memory.
template <typename Tin, int DPL>
__device__ __forceinline__ void load_slice(const Tin* __restrict__ p, float* out) {
  if constexpr (sizeof(Tin) == 4) {
#pragma unroll
    for (int i = 0; i < DPL; i += 4) {
      if constexpr (DPL >= 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p + i));
        out[i] = v.x; out[i + 1] = v.y; out[i + 2] = v.z; out[i + 3] = v.w;
      }
    }
    if constexpr (DPL == 2) {
      const float2 v = __ldg(reinterpret_cast<const float2*>(p));
      out[0] = v.x; out[1] = v.y;
    } else if constexpr (DPL == 1) {
      out[0] = __ldg(reinterpret_cast<const float*>(p));
    }
  } else {
    if constexpr (DPL == 8) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(w[i] << 16);
        out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    } else if constexpr (DPL == 4) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
      out[0] = __uint_as_float(u.x << 16); out[1] = __uint_as_float(u.x & 0xffff0000u);
      out[2] = __uint_as_float(u.y << 16); out[3] = __uint_as_float(u.y & 0xffff0000u);
    } else if constexpr (DPL == 2) {
      const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
      out[0] = __uint_as_float(u << 16); out[1] = __uint_as_float(u & 0xffff0000u);
    } else {
      out[0] = __bfloat162float(*p);
    }
  }
}

template <typename Tin, int DPL>
__global__ void __launch_bounds__(kScoreWarps * 32)
k_score_warp(const Tin* __restrict__ q, const Tin* __restrict__ kk, const Tin* __restrict__ C1,
             const Tin* __restrict__ C2, Plan p, int t0, int tlen, const int* __restrict__ rows,
             const DevStatus* __restrict__ st_rows, int nrows, int* __restrict__ surv_cnt,
             uint2* __restrict__ surv) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K2 = pow2_at_least(p.k);
  uint64_t* sel = reinterpret_cast<uint64_t*>(smem) + size_t(warp) * K2;
  const int n = p.n, k = p.k;
  const int ng = (n + 31) / 32;
  const int count = rows ? st_rows->redo : nrows;
  for (int w = blockIdx.x * kScoreWarps + warp; w < count; w += gridDim.x * kScoreWarps) {
    const int r = rows ? rows[w] : w;
    const int half = r & 1, side = (r >> 1) & 1;
    const int tl = (r >> 2) % p.Tc, bh = (r >> 2) / p.Tc;
    if (tl >= tlen) continue;
    const int h = bh % p.H;
    const size_t t = size_t(bh) * p.T + t0 + tl;
    const Tin* x = (side ? q : kk) + t * p.dqk + size_t(half) * p.dh;
    const Tin* cb = (half ? C2 : C1) + size_t(h) * n * p.dh + lane * DPL;
    float xr[DPL];
    load_slice<Tin, DPL>(x + lane * DPL, xr);
    uint32_t key[32];  // order-preserving image of the score of row g * 32 + lane
#pragma unroll
    for (int g = 0; g < 32; ++g) {
      key[g] = 0u;
      if (g < ng) {
        float part[32];
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int row = min(g * 32 + jj, n - 1);
          float c[DPL];
          load_slice<Tin, DPL>(cb + size_t(row) * p.dh, c);
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc = fmaf(xr[i], c[i], acc);
          part[jj] = acc;
        }
        // butterfly: lane l ends with the sum over lanes of part[l]
#pragma unroll
        for (int sft = 16; sft >= 1; sft >>= 1) {
          const bool up = (lane & sft) != 0;
#pragma unroll
          for (int i = 0; i < sft; ++i) {
            const float send = up ? part[i] : part[i + sft];
            const float keep = up ? part[i + sft] : part[i];
            part[i] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
          }
        }
        if (g * 32 + lane < n) key[g] = f2ord(part[0]);
      }
    }
    // the k-th largest image (counting repeats): most significant bit first
    uint32_t thr = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = thr | (1u << bit);
      int c = 0;
#pragma unroll
      for (int g = 0; g < 32; ++g) c += (g < ng && key[g] >= cand) ? 1 : 0;
      if (__reduce_add_sync(0xffffffffu, c) >= k) thr = cand;
    }
    int gt = 0;
#pragma unroll
    for (int g = 0; g < 32; ++g) gt += (g < ng && key[g] > thr) ? 1 : 0;
    const int n_gt = __reduce_add_sync(0xffffffffu, gt);
    // the rows above the threshold, then the lowest rows at it, in row order
    int base = 0, ties_left = k - n_gt;
#pragma unroll
    for (int g = 0; g < 32; ++g) {
      if (g < ng) {
        const bool valid = g * 32 + lane < n;
        const bool above = valid && key[g] > thr;
        const bool tie = valid && key[g] == thr;
        const unsigned ma = __ballot_sync(0xffffffffu, above);
        const unsigned mt = __ballot_sync(0xffffffffu, tie);
        const int tie_rank = __popc(mt & ((1u << lane) - 1u));
        const bool take = above || (tie && tie_rank < ties_left);
        const unsigned mk = __ballot_sync(0xffffffffu, take);
        if (take)
          sel[base + __popc(mk & ((1u << lane) - 1u))] =
              (uint64_t(key[g]) << 32) | uint64_t(~uint32_t(g * 32 + lane));
        base += __popc(mk);
        ties_left -= min(ties_left, __popc(mt));
      }
    }
    for (int i = k + lane; i < K2; i += 32) sel[i] = 0;
    __syncwarp();
    warp_sort_desc(sel, K2);
    uint2* out = surv + size_t(r) * p.C;
    for (int i = lane; i < k; i += 32) {
      const uint64_t kv = sel[i];
      out[i] = make_uint2(__float_as_uint(key_val(kv)), key_idx(kv));
    }
    if (lane == 0) surv_cnt[r] = k;
    __syncwarp();
  }
}

int score_warp_dpl(const Plan& p) {
  if (p.n > 1024 || p.dh % 32 != 0) return 0;
  const int dpl = p.dh / 32;
  return (dpl == 1 || dpl == 2 || dpl == 4 || dpl == 8) ? dpl : 0;
}

size_t score_simt_smem(const Plan& p) {
  if (score_warp_dpl(p)) return size_t(kScoreWarps) * size_t(pow2_at_least(p.k)) * 8;
  int S = 2;
  while (S < p.n) S <<= 1;
  return size_t(kScoreWarps) * (size_t(S) * 8 + size_t(p.dh) * 4);
}

template <typename Tin, int DPL>
static cudaError_t launch_warp_t(const Plan& p, const void* q, const void* k, const void* C1,
                                 const void* C2, int t0, int tlen, const int* rows,
                                 const DevStatus* st_rows, int nrows, int grid, size_t smem,
                                 int* surv_cnt, uint2* surv, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(k_score_warp<Tin, DPL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_score_warp<Tin, DPL><<<grid, kScoreWarps * 32, smem, s>>>(
      (const Tin*)q, (const Tin*)k, (const Tin*)C1, (const Tin*)C2, p, t0, tlen, rows, st_rows,
      nrows, surv_cnt, surv);
  return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_warp_dt(const Plan& p, int dpl, const void* q, const void* k,
                                  const void* C1, const void* C2, int t0, int tlen,
                                  const int* rows, const DevStatus* st_rows, int nrows, int grid,
                                  size_t smem, int* surv_cnt, uint2* surv, cudaStream_t s) {
  switch (dpl) {
    case 1: return launch_warp_t<Tin, 1>(p, q, k, C1, C2, t0, tlen, rows, st_rows, nrows, grid, smem, surv_cnt, surv, s);
    case 2: return launch_warp_t<Tin, 2>(p, q, k, C1, C2, t0, tlen, rows, st_rows, nrows, grid, smem, surv_cnt, surv, s);
    case 4: return launch_warp_t<Tin, 4>(p, q, k, C1, C2, t0, tlen, rows, st_rows, nrows, grid, smem, surv_cnt, surv, s);
    case 8: return launch_warp_t<Tin, 8>(p, q, k, C1, C2, t0, tlen, rows, st_rows, nrows, grid, smem, surv_cnt, surv, s);
    default: return cudaErrorInvalidValue;
  }
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
  if (const int dpl = score_warp_dpl(p)) {
    if (p.dtype == SDM_DTYPE_F32)
      return launch_warp_dt<float>(p, dpl, q, k, C1, C2, t0, tlen, rows, st_rows, nrows, grid,
                                   smem, surv_cnt, surv, s);
    return launch_warp_dt<__nv_bfloat16>(p, dpl, q, k, C1, C2, t0, tlen, rows, st_rows, nrows,
                                         grid, smem, surv_cnt, surv, s);
  }
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
