// score_tc.cu -- sub-key scoring on the 5th-generation tensor cores (tcgen05)
// with a per-row threshold filter and an exact sorted top-k per half-row.
//
// SDM summaries (gist.science 2607.07386), "Mecanismo Central" item 2: each
// half of k'_t / q'_t is scored against its sub-key codebook (a dense
// contraction: tokens x d_h times d_h x n_sub) and keeps its top-k.
//
// One CTA = 128 tokens of one (b,h) head, one side (k' or q') and one half:
//   warp 0      TMA producer: the 128 x d_h token tile once, then the codebook
//               in 256-row tiles through a 2-stage shared-memory ring (128-byte
//               swizzle, bf16, K-major);
//   warp 1      allocates 512 TMEM columns; one lane issues
//               tcgen05.mma.kind::f16 (bf16 x bf16 -> fp32, M=128, N=256,
//               K=16 steps) into two 256-column TMEM buffers;
//   warps 2..17 epilogue, kQ = 4 threads per token row (the kQ warps whose
//               warp index is equal mod 4 share one 32-lane TMEM quarter; each
//               takes a quarter of every 256-column tile): tcgen05.ld the
//               row's scores and keep those above a threshold tau taken from
//               the row's own score mean and deviation (first 512 columns);
//               then, one warp per row, the exact top-k of the kept scores
//               (64 buckets of the key range, a warp scan of their counts,
//               ranks within the buckets down to the k-th), written sorted by
//               (score desc, row asc).
// A row whose kept count falls outside [k, capacity] (or whose scores do not
// spread) is queued for the exact CUDA-core path instead, so the result is
// exact for any input.  Every mbarrier wait is bounded: on a timeout the CTA
// records SDM_DEV_TIMEOUT, stops issuing work, drains what it issued (bounded),
// frees its TMEM and queues all of its rows for the exact path, so that the
// selection stays exact even then.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "select_dev.cuh"

namespace sdm {
namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kKAtom = 64;           // bf16 elements per 128-byte swizzle row
constexpr int kQ = 4;                // epilogue threads per token row
constexpr int kEpiThreads = kQ * kTileM;
constexpr int kThreads = 64 + kEpiThreads;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz
#ifndef SDM_POLL_SLEEP_NS
#define SDM_POLL_SLEEP_NS 32
#endif
constexpr unsigned kPollSleepNs = SDM_POLL_SLEEP_NS;  // pause between mbarrier polls
constexpr uint32_t kATileBytes = kTileM * 128;   // one 64-column chunk of the token tile
constexpr uint32_t kBTileBytes = kTileN * 128;   // one 64-column chunk of a codebook tile

struct TcArgs {
  Plan p;
  int t0, tlen;
  float z;          // threshold in deviations above the row mean (-inf: keep all)
  uint2* surv;
  int* cnt;
  int* redo;
  DevStatus* st;
};

// Per-row survivor lists are row-major with one element of padding (row
// stride C + 1 floats, C + 2 row numbers), so that the filter's appends (one
// lane per row) and the selection's reads (one warp per row) both spread over
// the banks.  The selection's per-warp scratch (bucket counters, then staged
// 64-bit keys) has its own area: the token tile and the codebook ring are
// already being refilled for the CTA's next work item while it runs.
struct TcLayout {
  uint32_t a, b, vals, idx, rows, sel, bars, total;
  int nkc, cap;
};

// Staged entries per warp: the k best plus 24 (the bucket holding the k-th),
// and at least the fallback's sort buffer (next_pow2(k) keys); at most C.
__host__ __device__ inline int sel_cap(int C, int k) {
  const int k2 = next_pow2(k < 2 ? 2 : k);
  int cap = k + 24 > k2 ? k + 24 : k2;
  cap = (cap + 7) & ~7;
  return cap < C ? cap : (C > k2 ? C : k2);
}

__host__ __device__ inline TcLayout tc_layout(const Plan& p) {
  TcLayout L;
  L.nkc = p.dh / kKAtom;
  L.cap = sel_cap(p.C, p.k);
  uint32_t o = 0;
  L.a = o; o += L.nkc * kATileBytes;
  L.b = o; o += 2 * L.nkc * kBTileBytes;
  L.vals = o; o += uint32_t(p.C + 1) * kTileM * 4;
  L.idx = o; o += uint32_t(p.C + 2) * kTileM * 2;
  o = (o + 15) & ~15u;
  L.rows = o; o += (2 + 2 * kQ) * kTileM * 4;  // per-row count, go flag, partial stats
  L.sel = o; o += uint32_t(kEpiThreads / 32) * uint32_t(kSelHeadBytes + 8 * L.cap);
  L.bars = o; o += 16 * 8;  // mbarriers, TMEM address, abort flags
  L.total = o + 1024;  // slack for 1024-byte alignment of the dynamic base
  return L;
}

// ---- PTX wrappers -------------------------------------------------------------
__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false when it timed out or another role already gave up.
// Between polls the warp sleeps briefly, so that waiting warps leave the issue
// slots to the epilogue warps that share their SM sub-partition.
__device__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag) {
  const long long t0 = clock64();
  while (!mbar_test(b, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      return false;
    }
    __nanosleep(kPollSleepNs);
  }
  return true;
}
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(su32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(su32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// K-major, 128-byte swizzle shared-memory matrix descriptor (8-row groups
// 1024 bytes apart).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
  uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t(1) << 16;          // leading byte offset (unused for swizzled K-major)
  d |= uint64_t(1024 >> 4) << 32;  // stride byte offset
  d |= uint64_t(1) << 46;          // descriptor version (sm_100)
  d |= uint64_t(2) << 61;          // 128-byte swizzle
  return d;
}
// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both K-major.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          su32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Predicated stores (no branch): write x at the address when `on` is nonzero.
__device__ __forceinline__ void sts_f32_if(uint32_t a, float x, uint32_t on) {
  asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %2, 0;\n @p st.shared.f32 [%0], %1;\n}\n"
               ::"r"(a), "f"(x), "r"(on));
}
__device__ __forceinline__ void sts_u16_if(uint32_t a, uint16_t x, uint32_t on) {
  asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %2, 0;\n @p st.shared.u16 [%0], %1;\n}\n"
               ::"r"(a), "h"(x), "r"(on));
}

// named barrier of the epilogue warps
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}


template <int PL>
__global__ void __launch_bounds__(kThreads, 1)
k_score_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
           const __grid_constant__ CUtensorMap mc1, const __grid_constant__ CUtensorMap mc2,
           TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the swizzled tiles, by offset arithmetic on the
  // shared array itself so that every access stays a shared-memory access
  unsigned char* smem = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
  const Plan& p = a.p;
  const TcLayout L = tc_layout(p);
  unsigned char* sA = smem + L.a;
  unsigned char* sB = smem + L.b;
  float* vals = reinterpret_cast<float*>(smem + L.vals);        // [128][C + 1]
  uint16_t* idxs = reinterpret_cast<uint16_t*>(smem + L.idx);   // [128][C + 2]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* full = bars;       // [2] TMA -> MMA (codebook ring)
  uint64_t* empty = bars + 2;  // [2] MMA -> TMA
  uint64_t* a_full = bars + 4; // token tile landed
  uint64_t* a_empty = bars + 5;// token tile consumed by every MMA of its item
  uint64_t* tfull = bars + 6;  // [2] MMA -> epilogue
  uint64_t* tempty = bars + 8; // [2] epilogue -> MMA
  uint64_t* drain = bars + 10;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 12);
  volatile int* epi_abort = reinterpret_cast<volatile int*>(bars + 13);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.n / kTileN;
  const int nk = p.dh / 16;
  // work items: (token tile, head, side, half), side/half fastest
  const int ntt = (a.tlen + kTileM - 1) / kTileM;
  const int nitems = ntt * p.BH * 4;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiThreads);
    }
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *epi_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     su32(const_cast<uint32_t*>(tmem_slot)))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer: each item's token tile, then its codebook
    // tiles through the ring (gb counts the ring's fills over all items)
    if (lane == 0) {
      tma_prefetch(&mq);
      tma_prefetch(&mk);
      tma_prefetch(&mc1);
      tma_prefetch(&mc2);
      int gb = 0, na = 0;
      bool live = true;
      for (int w = blockIdx.x, i = 0; w < nitems && live; w += gridDim.x, ++i) {
        const int z = w & 3, rest = w >> 2;
        const int tile = rest % ntt, bh = rest / ntt, side = z >> 1, half = z & 1;
        const CUtensorMap* mx = side ? &mq : &mk;
        const CUtensorMap* mc = half ? &mc2 : &mc1;
        if (i >= 1 && !mbar_wait(a_empty, (i - 1) & 1, abort_flag)) break;
        const int row0 = bh * p.T + a.t0 + tile * kTileM;
        mbar_expect_tx(a_full, L.nkc * kATileBytes);
        for (int kc = 0; kc < L.nkc; ++kc)
          tma_load_2d(mx, a_full, sA + kc * kATileBytes, half * p.dh + kc * kKAtom, row0);
        ++na;
        const int h = bh % p.H;
        for (int j = 0; j < ntiles; ++j, ++gb) {
          const int s = gb & 1;
          if (gb >= 2 && !mbar_wait(&empty[s], ((gb >> 1) & 1) ^ 1, abort_flag)) {
            live = false;
            break;
          }
          mbar_expect_tx(&full[s], L.nkc * kBTileBytes);
          for (int kc = 0; kc < L.nkc; ++kc)
            tma_load_2d(mc, &full[s], sB + (s * L.nkc + kc) * kBTileBytes, kc * kKAtom,
                        h * p.n + j * kTileN);
        }
      }
      // on abort: let the copies already issued land before the CTA leaves
      // (the last fill of each barrier: none of them has advanced past it)
      if (*abort_flag) {
        volatile int never = 0;
        if (na > 0) mbar_wait(a_full, (na - 1) & 1, &never);
        for (int g = (gb > 2 ? gb - 2 : 0); g < gb; ++g)
          mbar_wait(&full[g & 1], (g >> 1) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (gb: ring fills consumed, gt: TMEM buffers filled)
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kTileM, kTileN);
      // this CTA's items and ring fills: the producer waits for the release of
      // every fill but the last two, so only those releases are committed
      const int my_items = blockIdx.x < nitems ? (nitems - 1 - blockIdx.x) / gridDim.x + 1 : 0;
      const int nfill = my_items * ntiles;
      int gb = 0, gt = 0, issued = 0;
      bool live = true;
      for (int w = blockIdx.x, i = 0; w < nitems && live; w += gridDim.x, ++i) {
        if (!mbar_wait(a_full, i & 1, abort_flag)) break;
        for (int j = 0; j < ntiles; ++j, ++gb, ++gt) {
          const int s = gb & 1, buf = gt & 1;
          if (!mbar_wait(&full[s], (gb >> 1) & 1, abort_flag) ||
              (gt >= 2 && !mbar_wait(&tempty[buf], ((gt >> 1) & 1) ^ 1, abort_flag))) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + uint32_t(buf * kTileN);
          for (int kk = 0; kk < nk; ++kk) {
            const int kc = kk >> 2, ww = kk & 3;
            const uint64_t ad = sdesc(su32(sA + kc * kATileBytes + ww * 32));
            const uint64_t bd = sdesc(su32(sB + (s * L.nkc + kc) * kBTileBytes + ww * 32));
            umma_bf16(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          if (gb + 2 < nfill) umma_commit(&empty[s]);
          umma_commit(&tfull[buf]);
          ++issued;
        }
        if (live && i + 1 < my_items) umma_commit(a_empty);
      }
      if (*abort_flag && issued > 0) {
        // wait (bounded) for the MMAs already issued before TMEM is freed
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    // ---------------- epilogue: kQ threads per token row (= TMEM lane)
    const int q4 = warp & 3;
    const int sub = (warp - 2) >> 2;  // which kCols-column slice of every tile
    const int row = q4 * 32 + lane;
    const uint32_t tbase = tmem + (uint32_t(q4 * 32) << 16);
    const int C = p.C;
    const int k = p.k;
    constexpr int kCols = kTileN / kQ;
    int* rcnt = reinterpret_cast<int*>(smem + L.rows);      // [128] kept count
    int* rgo = rcnt + kTileM;                               // [128] row settled here
    float* rst = reinterpret_cast<float*>(rgo + kTileM);    // [2][kQ][128] sum, sq
    const int ew = warp - 2;
    const int K2 = next_pow2(k < 2 ? 2 : k);
    unsigned char* wscr = smem + L.sel + size_t(ew) * size_t(kSelHeadBytes + 8 * L.cap);
    uint32_t* scr = reinterpret_cast<uint32_t*>(wscr);
    uint64_t* stage = reinterpret_cast<uint64_t*>(wscr + kSelHeadBytes);
    const bool keep_all = !(a.z > -1e30f);
    const int nstat = ntiles < 2 ? ntiles : 2;
    bool ok = true;
    float v[32];
    for (int w = blockIdx.x, i = 0; w < nitems; w += gridDim.x, ++i) {
      const int z = w & 3, rest = w >> 2;
      const int tile = rest % ntt, bh = rest / ntt, side = z >> 1, half = z & 1;
      const int tl = tile * kTileM + row;
      const bool valid = tl < a.tlen;
      const int gt0 = i * ntiles;  // TMEM buffer fills before this item's
      if (sub == 0) rcnt[row] = 0;
      // statistics of the first (up to) two tiles
      float sum = 0.f, sq = 0.f;
      for (int j = 0; j < nstat && ok; ++j) {
        const int g = gt0 + j;
        ok = __all_sync(0xffffffffu, mbar_wait(&tfull[g & 1], (g >> 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kCols / 32; ++c) {
          tmem_ld32(tbase + uint32_t((g & 1) * kTileN + sub * kCols + c * 32), v);
#pragma unroll
          for (int ii = 0; ii < 32; ++ii) {
            sum += v[ii];
            sq = fmaf(v[ii], v[ii], sq);
          }
        }
      }
      if (!ok) *epi_abort = 1;
      rst[(0 * kQ + sub) * kTileM + row] = sum;
      rst[(1 * kQ + sub) * kTileM + row] = sq;
      epi_sync();
      ok = !*epi_abort;
      float tau = -INFINITY;
      bool redo = false;
      {
        float S = 0.f, S2 = 0.f;
#pragma unroll
        for (int j = 0; j < kQ; ++j) {
          S += rst[(0 * kQ + j) * kTileM + row];
          S2 += rst[(1 * kQ + j) * kTileM + row];
        }
        const float m = float(nstat * kTileN);
        const float mu = S / m;
        const float sd = sqrtf(fmaxf(S2 / m - mu * mu, 0.f));
        if (!keep_all) tau = mu + a.z * sd;
        redo = !keep_all && !(sd > 0.f);
        // rows past the end of the chunk keep nothing, so that a warp whose rows
        // are all past it skips the appends (single steps, ragged last tiles)
        if (!valid) tau = INFINITY;
      }
      // filter: append the kept scores of this thread's columns to the row's list
      float* vrow = vals + row * (C + 1);
      uint16_t* irow = idxs + row * (C + 2);
      for (int j = 0; j < ntiles && ok; ++j) {
        const int g = gt0 + j, buf = g & 1;
        if (j >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], (g >> 1) & 1, abort_flag));
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll 1
        for (int c = 0; c < kCols / 32; ++c) {
          tmem_ld32(tbase + uint32_t(buf * kTileN + sub * kCols + c * 32), v);
          const int col0 = j * kTileN + sub * kCols + c * 32;
          uint32_t mask = 0;
#pragma unroll
          for (int ii = 0; ii < 32; ++ii) mask |= (v[ii] >= tau ? 1u : 0u) << ii;
          // reserve the places (one shared atomic), then append with predicated
          // stores: no branch per score, so the warp does not diverge
          const int nk = __popc(mask);
          const int pos0 = atomicAdd(&rcnt[row], nk);
          if (pos0 + nk <= C) {
            uint32_t av = su32(vrow + pos0), ai = su32(irow + pos0);
#pragma unroll
            for (int ii = 0; ii < 32; ++ii) {
              const uint32_t on = mask & (1u << ii);
              sts_f32_if(av, v[ii], on);
              sts_u16_if(ai, uint16_t(col0 + ii), on);
              av += on ? 4u : 0u;
              ai += on ? 2u : 0u;
            }
          } else {
            int pos = pos0;  // the row overflows its list: it goes to the exact path
#pragma unroll
            for (int ii = 0; ii < 32; ++ii) {
              if ((mask >> ii) & 1u) {
                if (pos < C) {
                  vrow[pos] = v[ii];
                  irow[pos] = uint16_t(col0 + ii);
                }
                ++pos;
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
      }
      if (!ok) *epi_abort = 1;
      epi_sync();
      ok = !*epi_abort;
      if (!ok && threadIdx.x == 64) dev_flag(a.st, SDM_DEV_TIMEOUT, blockIdx.x);
      if (sub == 0) {
        const int cnt = rcnt[row];
        const bool go = ok && valid && !redo && cnt >= k && cnt <= C;
        rgo[row] = go ? 1 : 0;
        // every valid row this CTA does not settle -- including all of them
        // after a timed-out wait -- is re-scored exactly, so no later kernel
        // reads a list this call never wrote
        const size_t hr = (size_t(bh) * p.Tc + tl) * 4 + side * 2 + half;
        if (valid && !go) a.redo[atomicAdd(&a.st->redo, 1)] = int(hr);
      }
      epi_sync();
      // exact top-k of each settled row's kept scores, one warp per row, sorted
      // by (score desc, row asc) and written to the survivor list: by buckets
      // of the key range (warp_bucket_topk), or -- when the buckets down to the
      // k-th hold more entries than the staging area -- by a bitwise search for
      // the k-th largest, a gather of the k best and a warp sort.  Meanwhile the
      // producer and the MMA issuer already work on the CTA's next item.
      for (int r = ew; r < kTileM; r += kEpiThreads / 32) {
        if (!rgo[r]) continue;
        const int cnt = rcnt[r];
        const float* vr = vals + r * (C + 1);
        const uint16_t* ir = idxs + r * (C + 2);
        uint32_t key[PL], rw[PL];
#pragma unroll
        for (int ii = 0; ii < PL; ++ii) {
          const int jj = ii * 32 + lane;
          key[ii] = jj < cnt ? f2ord(vr[jj]) : 0u;
          rw[ii] = jj < cnt ? uint32_t(ir[jj]) : 0u;
        }
        const size_t hr = (size_t(bh) * p.Tc + tile * kTileM + r) * 4 + side * 2 + half;
        uint2* g = a.surv + hr * C;
        if (!warp_bucket_topk<PL>(key, rw, cnt, k, scr, stage, L.cap, g)) {
          const uint32_t thr = warp_kth_key<PL>(key, cnt, k);
          warp_gather_topk<PL>(key, rw, cnt, k, thr, stage);
          __syncwarp();
          for (int ii = k + lane; ii < K2; ii += 32) stage[ii] = 0;
          __syncwarp();
          warp_sort_desc(stage, K2);
          for (int ii = lane; ii < k; ii += 32)
            g[ii] = make_uint2(__float_as_uint(key_val(stage[ii])), key_idx(stage[ii]));
        }
        if (lane == 0) a.cnt[hr] = k;
        __syncwarp();
      }
      // the next item's counts, statistics and lists overwrite this one's
      epi_sync();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---- filter-only variant --------------------------------------------------
// k_score_tc_filter: the same TMA -> tcgen05 pipeline with 128-row codebook
// tiles (two 128-column TMEM buffers, 256 columns per CTA, so that two CTAs
// share an SM), and an epilogue of kQF = 2 threads per token row that only
// filters: every score at or above the row's threshold is appended, unsorted,
// to the half-row's survivor list in global memory (capacity C).  A row whose
// kept count falls outside [k, C], or whose scores do not spread, is queued
// for the exact CUDA-core path; the exact sorted top-k of the kept scores is
// taken afterwards by k_topk_surv.  This needs no shared memory for the
// survivors, so it serves every k (the in-kernel selection above needs about
// 6 * C bytes per token row).
constexpr int kTileNF = 128;
constexpr int kQF = 2;
constexpr int kEpiThreadsF = kQF * kTileM;
constexpr int kThreadsF = 64 + kEpiThreadsF;
constexpr int kStagesF = 2;
constexpr uint32_t kBTileBytesF = kTileNF * 128;  // one 64-column chunk of a codebook tile

struct TcLayoutF {
  uint32_t a, b, rows, bars, total;
  int nkc;
};

__host__ __device__ inline TcLayoutF tc_layout_f(const Plan& p) {
  TcLayoutF L;
  L.nkc = p.dh / kKAtom;
  uint32_t o = 0;
  L.a = o; o += L.nkc * kATileBytes;
  L.b = o; o += kStagesF * L.nkc * kBTileBytesF;
  L.rows = o; o += (1 + 2 * kQF) * kTileM * 4;  // per-row count, partial stats
  o = (o + 15) & ~15u;
  L.bars = o; o += 16 * 8;
  L.total = o + 1024;
  return L;
}

__device__ __forceinline__ void epi_sync_f() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreadsF) : "memory");
}

__global__ void __launch_bounds__(kThreadsF, 2)
k_score_tc_filter(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                  const __grid_constant__ CUtensorMap mc1, const __grid_constant__ CUtensorMap mc2,
                  TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
  const Plan& p = a.p;
  const TcLayoutF L = tc_layout_f(p);
  unsigned char* sA = smem + L.a;
  unsigned char* sB = smem + L.b;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* full = bars;        // [kStagesF] TMA -> MMA
  uint64_t* empty = bars + 2;   // [kStagesF] MMA -> TMA
  uint64_t* a_full = bars + 4;
  uint64_t* tfull = bars + 5;   // [2] MMA -> epilogue
  uint64_t* tempty = bars + 7;  // [2] epilogue -> MMA
  uint64_t* drain = bars + 9;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bars + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 11);
  volatile int* epi_abort = reinterpret_cast<volatile int*>(bars + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, bh = blockIdx.y, side = blockIdx.z >> 1, half = blockIdx.z & 1;
  const int h = bh % p.H;
  const int ntiles = p.n / kTileNF;
  const int nk = p.dh / 16;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiThreadsF);
    }
    mbar_init(a_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *epi_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
                     su32(const_cast<uint32_t*>(tmem_slot)))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      const CUtensorMap* mx = side ? &mq : &mk;
      const CUtensorMap* mc = half ? &mc2 : &mc1;
      tma_prefetch(mx);
      tma_prefetch(mc);
      const int row0 = bh * p.T + a.t0 + tile * kTileM;
      mbar_expect_tx(a_full, L.nkc * kATileBytes);
      for (int kc = 0; kc < L.nkc; ++kc)
        tma_load_2d(mx, a_full, sA + kc * kATileBytes, half * p.dh + kc * kKAtom, row0);
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&empty[s], ((j >> 1) & 1) ^ 1, abort_flag)) break;
        mbar_expect_tx(&full[s], L.nkc * kBTileBytesF);
        for (int kc = 0; kc < L.nkc; ++kc)
          tma_load_2d(mc, &full[s], sB + (s * L.nkc + kc) * kBTileBytesF, kc * kKAtom,
                      h * p.n + j * kTileNF);
        ++issued;
      }
      if (*abort_flag) {
        volatile int never = 0;
        mbar_wait(a_full, 0, &never);
        for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j)
          mbar_wait(&full[j & 1], (j >> 1) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kTileM, kTileNF);
      int issued = 0;
      if (mbar_wait(a_full, 0, abort_flag)) {
        for (int j = 0; j < ntiles; ++j) {
          const int s = j & 1;
          if (!mbar_wait(&full[s], (j >> 1) & 1, abort_flag)) break;
          if (j >= 2 && !mbar_wait(&tempty[s], ((j >> 1) & 1) ^ 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t d = tmem + uint32_t(s * kTileNF);
          for (int kk = 0; kk < nk; ++kk) {
            const int kc = kk >> 2, w = kk & 3;
            const uint64_t ad = sdesc(su32(sA + kc * kATileBytes + w * 32));
            const uint64_t bd = sdesc(su32(sB + (s * L.nkc + kc) * kBTileBytesF + w * 32));
            umma_bf16(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          umma_commit(&tfull[s]);
          ++issued;
        }
      }
      if (*abort_flag && issued > 0) {
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never);
      }
    }
  } else {
    // ---------------- epilogue: kQF threads per token row (= TMEM lane)
    const int q4 = warp & 3;
    const int sub = (warp - 2) >> 2;  // which half of every tile's columns
    const int row = q4 * 32 + lane;
    const int tl = tile * kTileM + row;
    const bool valid = tl < a.tlen;
    const uint32_t tbase = tmem + (uint32_t(q4 * 32) << 16);
    const int C = p.C;
    constexpr int kCols = kTileNF / kQF;  // 64
    int* rcnt = reinterpret_cast<int*>(smem + L.rows);       // [128] kept count
    float* rst = reinterpret_cast<float*>(rcnt + kTileM);    // [2][kQF][128] sum, sq
    const size_t hr = (size_t(bh) * p.Tc + tl) * 4 + side * 2 + half;
    uint2* g = a.surv + hr * C;
    float v[32];
    if (sub == 0) rcnt[row] = 0;
    // statistics of the first (up to) two tiles
    const int nstat = ntiles < 2 ? ntiles : 2;
    float sum = 0.f, sq = 0.f;
    bool ok = true;
    for (int j = 0; j < nstat && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&tfull[j], 0, abort_flag));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kCols / 32; ++c) {
        tmem_ld32(tbase + uint32_t(j * kTileNF + sub * kCols + c * 32), v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          sum += v[i];
          sq = fmaf(v[i], v[i], sq);
        }
      }
    }
    if (!ok) *epi_abort = 1;
    rst[(0 * kQF + sub) * kTileM + row] = sum;
    rst[(1 * kQF + sub) * kTileM + row] = sq;
    epi_sync_f();
    ok = !*epi_abort;
    const bool keep_all = !(a.z > -1e30f);
    float tau;
    bool redo;
    {
      float S = 0.f, S2 = 0.f;
#pragma unroll
      for (int j = 0; j < kQF; ++j) {
        S += rst[(0 * kQF + j) * kTileM + row];
        S2 += rst[(1 * kQF + j) * kTileM + row];
      }
      const float m = float(nstat * kTileNF);
      const float mu = S / m;
      const float sd = sqrtf(fmaxf(S2 / m - mu * mu, 0.f));
      tau = keep_all ? -INFINITY : mu + a.z * sd;
      redo = !keep_all && !(sd > 0.f);
      if (!valid) tau = INFINITY;  // rows past the chunk keep nothing
    }
    // filter: append the kept scores of this thread's columns to the row's
    // survivor list in global memory
    for (int j = 0; j < ntiles && ok; ++j) {
      const int s = j & 1;
      if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&tfull[s], (j >> 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
      }
#pragma unroll 1
      for (int c = 0; c < kCols / 32; ++c) {
        tmem_ld32(tbase + uint32_t(s * kTileNF + sub * kCols + c * 32), v);
        const int col0 = j * kTileNF + sub * kCols + c * 32;
        uint32_t mask = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) mask |= (v[i] >= tau ? 1u : 0u) << i;
        if (mask) {
          int pos = atomicAdd(&rcnt[row], __popc(mask));
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if ((mask >> i) & 1u) {
              if (pos < C) g[pos] = make_uint2(__float_as_uint(v[i]), uint32_t(col0 + i));
              ++pos;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[s]);
    }
    if (!ok) *epi_abort = 1;
    epi_sync_f();
    ok = !*epi_abort;
    if (!ok && threadIdx.x == 64) dev_flag(a.st, SDM_DEV_TIMEOUT, blockIdx.x);
    if (sub == 0 && valid) {
      const int cnt = rcnt[row];
      if (ok && !redo && cnt >= p.k && cnt <= C) a.cnt[hr] = cnt;
      else a.redo[atomicAdd(&a.st->redo, 1)] = int(hr);  // exact CUDA-core path
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem) : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {uint32_t(kKAtom), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// z with P(N(0,1) > z) = f (bisection on the normal tail)
double normal_upper_quantile(double f) {
  double lo = -10.0, hi = 10.0;
  for (int i = 0; i < 200; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * erfc(mid / sqrt(2.0)) > f) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

}  // namespace

// Survivor capacity of a half-row.  In-kernel selection: room for the expected
// kept count (1.5 k + 16) plus a margin of 48.  Filter only: the expected kept
// count is 1.7 k + 16 (its threshold comes from 256 scores, not 512) and the
// list lives in global memory, so the margin is wider: 2 k + 80.
int score_tc_capacity(const sdm_dims* d, int mode) {
  int c = mode == 2 ? 2 * d->k + 80 : (3 * d->k) / 2 + 16 + 48;
  c = (c + 15) & ~15;
  return c < d->n_sub ? c : d->n_sub;
}

static double kept_target(const Plan& p) {
  return p.tc == 2 ? 1.7 * p.k + 16.0 : 1.5 * p.k + 16.0;
}

size_t score_tc_smem(const Plan& p) {
  return p.tc == 2 ? tc_layout_f(p).total : tc_layout(p).total;
}

#ifndef SDM_TC_MODE
#define SDM_TC_MODE 0  // 0: chosen by shape; 1 or 2: that mode wherever it runs
#endif

// Which tensor-core scoring kernel serves d: 0 none (CUDA cores), 1 k_score_tc
// (in-kernel exact selection), 2 k_score_tc_filter + k_topk_surv.  Mode 1 is
// preferred where its per-row survivor lists fit shared memory.
int score_tc_mode(const sdm_dims* d) {
  if (d->in_dtype != SDM_DTYPE_BF16) return 0;
  const int dh = d->d_qk / 2;
  if (dh % kKAtom != 0 || dh > 256) return 0;
  if (d->n_sub % kTileNF != 0 || d->n_sub > 65535) return 0;
  if ((long long)d->B * d->H * d->T >= (1LL << 31)) return 0;
  if ((long long)d->H * d->n_sub >= (1LL << 31)) return 0;
  Plan tmp;
  tmp.dh = dh;
  tmp.C = score_tc_capacity(d, 1);
  tmp.k = d->k;
  tmp.tc = 1;
  const TcLayout L = tc_layout(tmp);
  // the selection holds a row's kept scores in registers, at most 8 per lane
  const bool m1 = d->n_sub % kTileN == 0 && tmp.C <= 8 * 32 && L.total <= 227 * 1024;
  tmp.tc = 2;
  tmp.C = score_tc_capacity(d, 2);
  const bool m2 = tc_layout_f(tmp).total <= 227 * 1024;
  if (SDM_TC_MODE == 1) return m1 ? 1 : 0;
  if (SDM_TC_MODE == 2) return m2 ? 2 : 0;
  return m1 ? 1 : (m2 ? 2 : 0);
}

cudaError_t launch_score_tc(const Plan& p, const void* q, const void* k, const void* C1,
                            const void* C2, int t0, int tlen, int* surv_cnt, uint2* surv,
                            int* redo_rows, DevStatus* st, cudaStream_t s) {
  CUtensorMap mq, mk, mc1, mc2;
  if (!encode_fn()) return cudaErrorNotSupported;
  const uint32_t box_n = p.tc == 2 ? kTileNF : kTileN;
  const uint64_t rows = uint64_t(p.BH) * p.T;
  if (!make_map(&mq, q, rows, p.dqk, kTileM) || !make_map(&mk, k, rows, p.dqk, kTileM) ||
      !make_map(&mc1, C1, uint64_t(p.H) * p.n, p.dh, box_n) ||
      !make_map(&mc2, C2, uint64_t(p.H) * p.n, p.dh, box_n))
    return cudaErrorInvalidValue;
  TcArgs a;
  a.p = p;
  a.t0 = t0;
  a.tlen = tlen;
  const double f = kept_target(p) / double(p.n);
  a.z = (f >= 1.0 || p.C >= p.n) ? -INFINITY : float(normal_upper_quantile(f));
  a.surv = surv;
  a.cnt = surv_cnt;
  a.redo = redo_rows;
  a.st = st;
  const size_t smem = score_tc_smem(p);
  dim3 grid((tlen + kTileM - 1) / kTileM, p.BH, 4);
  cudaError_t e;
  if (p.tc == 2) {
    e = cudaFuncSetAttribute(k_score_tc_filter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    k_score_tc_filter<<<grid, kThreadsF, smem, s>>>(mq, mk, mc1, mc2, a);
  } else {
    // persistent: one CTA per SM (its shared memory), each walking the work
    // items (token tile, head, side, half) with a stride of the grid
    int dev = 0, nsm = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long nitems = (long long)grid.x * p.BH * 4;
    const int pgrid = int(nitems < nsm ? nitems : nsm);
    if (p.C <= 4 * 32) {
      e = cudaFuncSetAttribute(k_score_tc<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem));
      if (e != cudaSuccess) return e;
      k_score_tc<4><<<pgrid, kThreads, smem, s>>>(mq, mk, mc1, mc2, a);
    } else if (p.C <= 5 * 32) {
      e = cudaFuncSetAttribute(k_score_tc<5>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem));
      if (e != cudaSuccess) return e;
      k_score_tc<5><<<pgrid, kThreads, smem, s>>>(mq, mk, mc1, mc2, a);
    } else {
      e = cudaFuncSetAttribute(k_score_tc<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem));
      if (e != cudaSuccess) return e;
      k_score_tc<8><<<pgrid, kThreads, smem, s>>>(mq, mk, mc1, mc2, a);
    }
  }
  return cudaGetLastError();
}

}  // namespace sdm
