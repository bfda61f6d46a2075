// sdm_internal.cuh -- shared definitions of the CUDA path (not part of the C ABI).
//
// The forward pass is split into three kernel families, launched per time
// chunk on the caller's stream:
//   1. scoring + per-half candidate lists   (score_simt.cu, score_tc.cu)
//   2. merge of the two halves into the top-W / top-R lists and softmax
//      weights, then the write/read plan of the recurrence (merge_plan.cu)
//   3. the gated delta recurrence over the slot table     (recur.cu)
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sdm.h"

namespace sdm {

// Fixed launch targets (depend on nothing but the problem sizes, so the
// workspace size is a function of the dims alone).
#ifndef SDM_RECUR_WARPS
#define SDM_RECUR_WARPS 2368  // recurrence warps aimed for: 148 SMs x 16 resident warps
#endif
#ifndef SDM_RECUR_CHUNK
#define SDM_RECUR_CHUNK 8  // records of a recurrence stream whose rows are in flight at once
#endif
#ifndef SDM_RECUR_MAX_F
#define SDM_RECUR_MAX_F 8  // floats of a row per lane, at most
#endif
constexpr int kRecurMaxF = SDM_RECUR_MAX_F;
constexpr int kRecurWarps = SDM_RECUR_WARPS;
constexpr int kRecurChunk = SDM_RECUR_CHUNK;
constexpr int kRecurThreads = 256;
constexpr int kMaxBlockEntries = 8192;  // list entries per (head, block) in a plan
constexpr int kEntryBits = 13;          // entry index within a block: < 2^13
static_assert(kMaxBlockEntries <= (1 << kEntryBits), "entry index must fit its key field");
#ifndef SDM_BUCKET_TARGET
#define SDM_BUCKET_TARGET 4
#endif
constexpr int kBucketTarget = SDM_BUCKET_TARGET;  // mean plan records per bucket aimed for
constexpr int kStreamMin = 4;           // mean records per stream and block, at least
constexpr size_t kChunkBudget = size_t(4) << 30;  // workspace bytes per time chunk
#ifndef SDM_RECUR_GROUP_BYTES
#define SDM_RECUR_GROUP_BYTES (size_t(8) << 30)  // slot-table bytes per recurrence launch
#endif
constexpr size_t kRecurGroupBytes = SDM_RECUR_GROUP_BYTES;
#ifndef SDM_PLAN_THREADS
#define SDM_PLAN_THREADS 512
#endif
#ifndef SDM_MERGE_WARPS
#define SDM_MERGE_WARPS 8
#endif
constexpr int kPlanThreads = SDM_PLAN_THREADS;
constexpr int kMergeWarps = SDM_MERGE_WARPS;  // merge kernel: warps per CTA
constexpr int kMergeSteps = 2 * SDM_MERGE_WARPS;  // merge kernel: steps per CTA

// Everything the kernels need to know about one call.
struct Plan {
  int B, H, T, dqk, dh, dv, n, k, W, R, dtype;
  int BH;
  long long N;
  int rule;    // write rule: 0 gated delta (alpha, beta), 1 selective decay (a)
  int tc;      // scoring mode: 0 CUDA cores, 1 tensor cores + in-kernel selection,
               // 2 tensor-core filter + survivor top-k (score_tc_mode)
  int C;       // survivor capacity per half-row
  int Tc;      // steps per chunk
  int nchunks;
  int P;       // steps per plan block
  int nblk;    // plan blocks per chunk
  int E;       // list entries per plan block = P * (W + R)
  int S;       // recurrence streams per head (one warp, or a lane group for d_v < 32)
  int NB;      // slot buckets per head = S * mb; stream s owns buckets [s*mb, (s+1)*mb)
  int mb;
  int HG;      // heads per recurrence launch
  int ncW, nfW, ncR, nfR;  // staircase / frontier sizes of the merge
  size_t merge_smem, plan_smem, recur_smem, score_smem;
  // workspace byte offsets
  size_t off_status, off_cnt, off_surv, off_redo, off_lists, off_rec, off_roff, total;
};

// Workspace status words.
struct DevStatus {
  int32_t flags;  // SDM_DEV_* bits
  int32_t info;   // first offending index, -1 if none
  int32_t redo;   // number of half-rows queued for the exact SIMT path
  int32_t pad[13];
};

// SDM_OK or an error code.  chunk_budget bounds the workspace bytes of one
// time chunk (the default, kChunkBudget, keeps it near 4 GiB); a smaller budget
// gives shorter chunks and the same results.
int make_plan(const sdm_dims* d, Plan* p, size_t chunk_budget = kChunkBudget);

// The forward pass of sdm_forward / sdm_forward_timed on a caller workspace
// laid out by make_plan(d, &p, chunk_budget) (same budget).
int forward_with_budget(const void* q, const void* k, const void* v, const float* alpha,
                        const float* beta, const void* C1, const void* C2, float* M_inout,
                        float* o_out, const sdm_dims* dims, void* workspace, size_t ws_bytes,
                        void* stream, void* const* events, int n_events, size_t chunk_budget,
                        int rule = 0);

// ---- device helpers ---------------------------------------------------------
__device__ __forceinline__ uint32_t f2ord(float v) {
  if (v == 0.0f) v = 0.0f;  // -0 and +0 compare equal: give them one key
  uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t o) {
  uint32_t b = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
  return __uint_as_float(b);
}
// Larger key = larger value, then smaller index.
__device__ __forceinline__ uint64_t make_key(float v, uint32_t idx) {
  return (uint64_t(f2ord(v)) << 32) | uint64_t(~idx);
}
__device__ __forceinline__ float key_val(uint64_t key) { return ord2f(uint32_t(key >> 32)); }
__device__ __forceinline__ uint32_t key_idx(uint64_t key) { return ~uint32_t(key); }

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  x ^= x >> 16; x *= 0x85ebca6bu;
  x ^= x >> 13; x *= 0xc2b2ae35u;
  x ^= x >> 16;
  return x;
}
// Which of a head's NB buckets holds a slot (multiply-shift of a hash).
__device__ __forceinline__ int slot_bucket(uint32_t slot, int NB) {
  return int((uint64_t(mix32(slot ^ 0x9e3779b9u)) * uint64_t(uint32_t(NB))) >> 32);
}

__device__ __forceinline__ void dev_flag(DevStatus* st, int bits, int info) {
  atomicOr(&st->flags, bits);
  atomicCAS(&st->info, -1, info);
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// Descending bitonic sort of S (power of two) 64-bit keys in shared memory by
// one warp.
__device__ __forceinline__ void warp_sort_desc(uint64_t* a, int S) {
  const int lane = threadIdx.x & 31;
  for (int size = 2; size <= S; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < (S >> 1); i += 32) {
        const int lo = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));
        const int hi = lo + stride;
        const uint64_t x = a[lo], y = a[hi];
        const bool desc = (lo & size) == 0;
        if (desc ? (x < y) : (x > y)) { a[lo] = y; a[hi] = x; }
      }
      __syncwarp();
    }
  }
}

__host__ __device__ inline int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// ---- launchers (one per kernel family) --------------------------------------
cudaError_t launch_init(const Plan& p, DevStatus* st, cudaStream_t s);
cudaError_t launch_score_simt(const Plan& p, const void* q, const void* k, const void* C1,
                              const void* C2, int t0, int tlen, const int* rows,
                              const DevStatus* st_rows, int* surv_cnt, uint2* surv,
                              DevStatus* st, cudaStream_t s);
cudaError_t launch_score_tc(const Plan& p, const void* q, const void* k, const void* C1,
                            const void* C2, int t0, int tlen, int* surv_cnt, uint2* surv,
                            int* redo_rows, DevStatus* st, cudaStream_t s);
// 0: CUDA-core scoring; 1: k_score_tc (in-kernel exact selection); 2:
// k_score_tc_filter (unsorted survivor lists), then k_topk_surv.
int score_tc_mode(const sdm_dims* d);
int score_tc_capacity(const sdm_dims* d, int mode);
size_t score_tc_smem(const Plan& p);
bool topk_surv_supported(int C);
size_t topk_surv_smem(const Plan& p);
// In place: the exact sorted top-k of every half-row's survivor list of the
// chunk's first tlen steps (counts become k).
cudaError_t launch_topk_surv(const Plan& p, int tlen, int* cnt, uint2* surv, DevStatus* st,
                             cudaStream_t s);

// Lists of (slot, weight) pairs: iw/ww [rows][W], ir/wr [rows][R]; a step's
// row is bh * list_T + list_t0 + (step within the chunk).
struct MergeIO {
  const int* surv_cnt;
  const uint2* surv;
  int32_t* out_iw; float* out_ww; int32_t* out_ir; float* out_wr;
  int list_T, list_t0;
  int sorted;  // write each list in rank order
};
cudaError_t launch_merge(const Plan& p, const MergeIO& io, int t0, int tlen, DevStatus* st,
                         cudaStream_t s);

struct PlanIO {
  const int32_t* iw; const float* ww; const int32_t* ir; const float* wr;
  int list_T, list_t0;
  int validate;  // flag out-of-range slots and repeated slots (caller lists)
  const float* alpha; const float* beta;
  int4* rec;
  int* roff;
  float* o;
  int* rent;  // optional: the block-local list entry (step * (W + R) + j) of each record
};
cudaError_t launch_plan(const Plan& p, const PlanIO& io, int t0, int tlen, DevStatus* st,
                        cudaStream_t s);

// snap == nullptr: the recurrence (writes into M, reads added into o).  snap
// given: the same walk, with no o, storing at every record the row it sees
// before the record's effect (snap[record] = d_v floats, record index as in rec)
// -- the values the backward pass needs; it starts from the table M0 without
// copying it: a row is read from M0 until the walk first stores it into M,
// which it records in touched (one byte per slot and head, zero at the start).
struct SaveIO {
  float* snap;
  const float* M0;
  uint8_t* touched;
};
cudaError_t launch_recur(const Plan& p, const void* v, float* M, float* o, const int4* rec,
                         const int* roff, int t0, int tlen, cudaStream_t s,
                         SaveIO sv = SaveIO{nullptr, nullptr, nullptr});

}  // namespace sdm
