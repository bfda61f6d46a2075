// topk_surv.cu -- exact sorted top-k of each half-row's survivor list.
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central" item 2: each
// half keeps its top-k codebook rows.  After the filter-only tensor-core
// scoring kernel, a half-row's survivor list holds, unsorted, every score at
// or above the row's threshold (between k and C entries); rows the filter could
// not settle were re-scored exactly by the CUDA-core kernel (k entries, already
// sorted).  One warp per half-row loads its list into registers and takes the
// exact top-k of it by buckets of the key range (warp_bucket_topk), or, when
// the buckets down to the k-th hold more entries than the staging area, by a
// bitwise search for the k-th largest, a gather of the k best and a warp sort.
// The k best are written back in place, sorted by (score desc, row asc), so
// that the merge reads the first k entries of every list, sorted, as it does
// after the other scoring kernels.
#include "select_dev.cuh"

namespace sdm {

constexpr int kTopkWarps = 8;

template <int PL>
__global__ void __launch_bounds__(kTopkWarps * 32)
k_topk_surv(Plan p, int tlen, int* __restrict__ cnt, uint2* __restrict__ surv, DevStatus* st) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K2 = next_pow2(p.k < 2 ? 2 : p.k);
  const int cap = p.C > K2 ? p.C : K2;
  unsigned char* wscr = smem + size_t(warp) * (kSelHeadBytes + 8 * size_t(cap));
  uint32_t* scr = reinterpret_cast<uint32_t*>(wscr);
  uint64_t* sel = reinterpret_cast<uint64_t*>(wscr + kSelHeadBytes);
  const int nrows = p.BH * tlen * 4;
  for (int w = blockIdx.x * kTopkWarps + warp; w < nrows; w += gridDim.x * kTopkWarps) {
    // w -> half-row (bh, tl, side, half) of the chunk
    const int bh = w / (tlen * 4), rem = w - bh * tlen * 4;
    const size_t hr = size_t(bh) * p.Tc * 4 + rem;
    const int c = cnt[hr];
    if (c < p.k || c > p.C || c > PL * 32) {
      if (lane == 0) dev_flag(st, SDM_DEV_CAPACITY, int(hr));
      continue;  // the merge sees the bad count and flags it too
    }
    uint2* list = surv + hr * p.C;
    uint32_t key[PL], row[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      const int j = i * 32 + lane;
      uint2 e = make_uint2(0u, 0u);
      if (j < c) e = list[j];
      key[i] = f2ord(__uint_as_float(e.x));
      row[i] = e.y;
    }
    __syncwarp();  // every lane has read the list before it is overwritten
    if (!warp_bucket_topk<PL>(key, row, c, p.k, scr, sel, cap, list)) {
      const uint32_t thr = warp_kth_key<PL>(key, c, p.k);
      warp_gather_topk<PL>(key, row, c, p.k, thr, sel);
      __syncwarp();
      for (int i = p.k + lane; i < K2; i += 32) sel[i] = 0;
      __syncwarp();
      warp_sort_desc(sel, K2);
      for (int i = lane; i < p.k; i += 32) {
        const uint64_t kv = sel[i];
        list[i] = make_uint2(__float_as_uint(key_val(kv)), key_idx(kv));
      }
    }
    if (lane == 0) cnt[hr] = p.k;
    __syncwarp();
  }
}

size_t topk_surv_smem(const Plan& p) {
  const int K2 = next_pow2(p.k < 2 ? 2 : p.k);
  const int cap = p.C > K2 ? p.C : K2;
  return size_t(kTopkWarps) * (kSelHeadBytes + 8 * size_t(cap));
}

template <int PL>
static cudaError_t launch_topk_t(const Plan& p, int tlen, int* cnt, uint2* surv, DevStatus* st,
                                 cudaStream_t s) {
  const size_t smem = topk_surv_smem(p);
  cudaError_t e = cudaFuncSetAttribute(k_topk_surv<PL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const long long nrows = (long long)p.BH * tlen * 4;
  long long grid = (nrows + kTopkWarps - 1) / kTopkWarps;
  if (grid > 148 * 32) grid = 148 * 32;
  k_topk_surv<PL><<<int(grid), kTopkWarps * 32, smem, s>>>(p, tlen, cnt, surv, st);
  return cudaGetLastError();
}

// Survivor capacities up to 512 entries (16 per lane).
bool topk_surv_supported(int C) { return C <= 16 * 32; }

cudaError_t launch_topk_surv(const Plan& p, int tlen, int* cnt, uint2* surv, DevStatus* st,
                             cudaStream_t s) {
  if (p.C <= 4 * 32) return launch_topk_t<4>(p, tlen, cnt, surv, st, s);
  if (p.C <= 8 * 32) return launch_topk_t<8>(p, tlen, cnt, surv, st, s);
  if (p.C <= 12 * 32) return launch_topk_t<12>(p, tlen, cnt, surv, st, s);
  if (p.C <= 16 * 32) return launch_topk_t<16>(p, tlen, cnt, surv, st, s);
  return cudaErrorInvalidValue;
}

}  // namespace sdm
