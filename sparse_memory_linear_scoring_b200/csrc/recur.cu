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
// Work split.  A head's slots are hashed into NB buckets, and each of the
// head's S streams owns a fixed range of buckets: every record of a slot, in
// every time block, belongs to one stream, so no two streams ever touch the
// same row and a stream needs no barrier and no shared memory.  A stream is
// one warp (LPR = 32 lanes, F = d_v / 32 floats of a row each) or, for
// d_v < 32, a group of LPR = d_v lanes.  It walks the time blocks in order;
// in each block its records are sorted by (bucket, slot, step, write before
// read), so a slot's records are adjacent and in time order.  Records are
// taken U at a time: every lane loads its share of the rows of the U records
// at once (the first record of each slot run only), then the records are
// applied in order -- a write is M = f1 * M + f2 * v_t (f1 = alpha (1 - c),
// f2 = c, folded by the plan kernel), a read adds u * M to o_t with a vector
// reduction (o was zeroed by the plan kernel) -- and each run's row is stored
// once after its last write.  The next chunk's records and the next blocks'
// segment bounds are loaded one step ahead.
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

template <int F>
__device__ __forceinline__ void ld_row(const float* ptr, float* m) {
  if constexpr (F == 8) {
    const float4 x = ld_cg4(ptr), y = ld_cg4(ptr + 4);
    m[0] = x.x; m[1] = x.y; m[2] = x.z; m[3] = x.w;
    m[4] = y.x; m[5] = y.y; m[6] = y.z; m[7] = y.w;
  } else if constexpr (F == 4) {
    const float4 x = ld_cg4(ptr);
    m[0] = x.x; m[1] = x.y; m[2] = x.z; m[3] = x.w;
  } else if constexpr (F == 2) {
    float2 x;
    asm volatile("ld.global.cg.v2.f32 {%0,%1}, [%2];" : "=f"(x.x), "=f"(x.y) : "l"(ptr));
    m[0] = x.x; m[1] = x.y;
  } else {
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(m[0]) : "l"(ptr));
  }
}
template <int F>
__device__ __forceinline__ void st_row(float* ptr, const float* m) {
  if constexpr (F == 8) {
    st4(ptr, make_float4(m[0], m[1], m[2], m[3]));
    st4(ptr + 4, make_float4(m[4], m[5], m[6], m[7]));
  } else if constexpr (F == 4) {
    st4(ptr, make_float4(m[0], m[1], m[2], m[3]));
  } else if constexpr (F == 2) {
    asm volatile("st.global.v2.f32 [%0], {%1,%2};" ::"l"(ptr), "f"(m[0]), "f"(m[1]) : "memory");
  } else {
    asm volatile("st.global.f32 [%0], %1;" ::"l"(ptr), "f"(m[0]) : "memory");
  }
}
template <int F>
__device__ __forceinline__ void red_row(float* ptr, const float* m, float u) {
  if constexpr (F == 8) {
    red_add4(ptr, make_float4(u * m[0], u * m[1], u * m[2], u * m[3]));
    red_add4(ptr + 4, make_float4(u * m[4], u * m[5], u * m[6], u * m[7]));
  } else if constexpr (F == 4) {
    red_add4(ptr, make_float4(u * m[0], u * m[1], u * m[2], u * m[3]));
  } else if constexpr (F == 2) {
    asm volatile("red.global.add.v2.f32 [%0], {%1,%2};" ::"l"(ptr), "f"(u * m[0]), "f"(u * m[1])
                 : "memory");
  } else {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(ptr), "f"(u * m[0]) : "memory");
  }
}

// F consecutive elements of a v row, raw (Vw 32-bit words), and as fp32
template <typename Tv, int F>
struct VRaw {
  static constexpr int n = (sizeof(Tv) * F + 3) / 4;
  uint32_t w[n];
};
template <typename Tv, int F>
__device__ __forceinline__ void ld_v(const Tv* ptr, VRaw<Tv, F>& r) {
  if constexpr (VRaw<Tv, F>::n == 8) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(ptr));
    const uint4 y = __ldg(reinterpret_cast<const uint4*>(ptr) + 1);
    r.w[0] = x.x; r.w[1] = x.y; r.w[2] = x.z; r.w[3] = x.w;
    r.w[4] = y.x; r.w[5] = y.y; r.w[6] = y.z; r.w[7] = y.w;
  } else if constexpr (VRaw<Tv, F>::n == 4) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(ptr));
    r.w[0] = x.x; r.w[1] = x.y; r.w[2] = x.z; r.w[3] = x.w;
  } else if constexpr (VRaw<Tv, F>::n == 2) {
    const uint2 x = __ldg(reinterpret_cast<const uint2*>(ptr));
    r.w[0] = x.x; r.w[1] = x.y;
  } else if constexpr (sizeof(Tv) * F == 2) {
    r.w[0] = __ldg(reinterpret_cast<const unsigned short*>(ptr));
  } else {
    r.w[0] = __ldg(reinterpret_cast<const unsigned int*>(ptr));
  }
}
template <typename Tv, int F>
__device__ __forceinline__ float v_at(const VRaw<Tv, F>& r, int j) {
  if constexpr (sizeof(Tv) == 4) {
    return __uint_as_float(r.w[j]);
  } else {
    const uint32_t u = r.w[j >> 1];
    return (j & 1) ? __uint_as_float(u & 0xffff0000u) : __uint_as_float(u << 16);
  }
}

// shared-memory record reads that the compiler neither merges nor hoists, so
// that a record's fields are live only where they are used
__device__ __forceinline__ int2 lds2(const int4* ptr) {
  int2 r;
  asm volatile("ld.shared.v2.s32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(ptr))));
  return r;
}
__device__ __forceinline__ int4 lds4(const int4* ptr) {
  int4 r;
  asm volatile("ld.shared.v4.s32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(ptr))));
  return r;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// cp.async of NB bytes (4, 8, 16 or a multiple of 16) from global to shared
template <int NB>
__device__ __forceinline__ void cp_bytes(void* dst, const void* src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  if constexpr (NB >= 16) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + 16 * i),
                   "l"(static_cast<const char*>(src) + 16 * i)
                   : "memory");
  } else {
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(d), "l"(src), "n"(NB)
                 : "memory");
  }
}

#ifndef SDM_RECUR_VREG
#define SDM_RECUR_VREG 1
#endif

template <typename Tv, int LPR, int F>
struct RecurSmem {
  static constexpr int dv = LPR * F;
  static constexpr int U = kRecurChunk;
  static constexpr int kStreams = kRecurThreads / LPR;
  // bf16 v rows are held in registers (F / 2 words a record), float32 ones
  // are staged in shared memory
  static constexpr bool kVReg = SDM_RECUR_VREG && sizeof(Tv) == 2;
  // per stream: two chunks of records (the one applied, the one arriving),
  // then the chunk's rows of M (and of v)
  static constexpr size_t ring = size_t(2) * U * 16;
  static constexpr size_t mrow = size_t(U) * dv * 4;
  static constexpr size_t vrow = kVReg ? 0 : (size_t(U) * dv * sizeof(Tv) + 15) & ~size_t(15);
  static constexpr size_t per_stream = ring + mrow + vrow;
  static constexpr size_t total = per_stream * kStreams;
};

template <typename Tv, int LPR, int F, bool SAVE>
__global__ void __launch_bounds__(kRecurThreads, kRecurWarps / 148 / (kRecurThreads / 32))
k_recur(Plan p, const Tv* __restrict__ v, float* __restrict__ M, float* __restrict__ o,
        const int4* __restrict__ rec, const int* __restrict__ roff, int t0, int tlen, int bh0,
        int nbh, SaveIO sv) {
  using SM = RecurSmem<Tv, LPR, F>;
  constexpr int dv = LPR * F;
  constexpr int U = SM::U;
  extern __shared__ __align__(16) unsigned char smem[];
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int stream = tid / LPR;
  const int ls = threadIdx.x / LPR;  // stream within the CTA
  const int sl = threadIdx.x % LPR;
  unsigned char* mine = smem + size_t(ls) * SM::per_stream;
  int4* ring = reinterpret_cast<int4*>(mine);                           // [2][U]
  float* mrow = reinterpret_cast<float*>(mine + SM::ring) + sl * F;     // [U][dv], own part
  Tv* vrow = reinterpret_cast<Tv*>(mine + SM::ring + SM::mrow) + sl * F;  // [U][dv], own part
  const unsigned gmask =
      LPR == 32 ? 0xffffffffu : (((1u << LPR) - 1u) << ((threadIdx.x & 31) / LPR * LPR));
  const int bh = bh0 + stream / p.S, s = stream % p.S;
  if (bh >= bh0 + nbh) return;  // whole lane groups leave together
  const int nb = (tlen + p.P - 1) / p.P;
  const int g0 = s * p.mb, g1 = g0 + p.mb;
  float* Mh = M + size_t(bh) * size_t(p.N) * dv + sl * F;
  // snapshot mode: rows not yet stored by this walk come from M0
  const float* M0h = SAVE ? sv.M0 + size_t(bh) * size_t(p.N) * dv + sl * F : nullptr;
  uint8_t* toh = SAVE ? sv.touched + size_t(bh) * size_t(p.N) : nullptr;
  const size_t trow = size_t(bh) * p.T + t0;
  const Tv* vh = v + trow * dv + sl * F;
  float* oh = o + trow * dv + sl * F;
  const int* rofh = roff + size_t(bh) * p.nblk * (p.NB + 1);
  const int4* rech = rec + size_t(bh) * p.nblk * p.E;

  // Segment bounds of blocks [wb, wb + LPR) (lane j: block wb + j) and of the
  // window after it.
  int wb = 0, wlo, whi, nlo, nhi;
  auto load_win = [&](int base, int& lo, int& hi) {
    const int blk = base + sl;
    lo = hi = 0;
    if (blk < nb) {
      const int* rr = rofh + size_t(blk) * (p.NB + 1);
      lo = __ldg(rr + g0);
      hi = __ldg(rr + g1);
    }
  };
  // bounds of block x, wb <= x < wb + 2 LPR (empty past the last block)
  auto bounds = [&](int x, int& lo, int& hi) {
    const int j = x - wb;
    const int l0 = __shfl_sync(gmask, wlo, j & (LPR - 1), LPR);
    const int h0 = __shfl_sync(gmask, whi, j & (LPR - 1), LPR);
    const int l1 = __shfl_sync(gmask, nlo, j & (LPR - 1), LPR);
    const int h1 = __shfl_sync(gmask, nhi, j & (LPR - 1), LPR);
    lo = j < LPR ? l0 : l1;
    hi = j < LPR ? h0 : h1;
  };
  // A chunk is up to U records: the rest of block blk's segment from pos, then
  // the start of block blk+1's.  Lanes copy the records into the ring.
  auto fetch_chunk = [&](int buf, int blk, int pos, int end, int npos, int nend) {
    const int t1 = min(U, end - pos);
    const int t2 = blk + 1 < nb ? min(U - t1, nend - npos) : 0;
    for (int i = sl; i < t1 + t2; i += LPR) {
      const int4* src = i < t1 ? rech + size_t(blk) * p.E + pos + i
                               : rech + size_t(blk + 1) * p.E + npos + (i - t1);
      cp_bytes<16>(&ring[buf * U + i], src);
    }
    cp_async_commit();
  };
  load_win(0, wlo, whi);
  load_win(LPR, nlo, nhi);
  int b = 0, pos, end, npos, nend;
  bounds(0, pos, end);
  bounds(1, npos, nend);
  int buf = 0;
  fetch_chunk(0, 0, pos, end, npos, nend);
  int pre_b = 0, pre_pos = pos;

  while (b < nb) {
    if (pos >= end) {
      // next block; keep the bounds window two blocks ahead
      ++b;
      pos = npos;
      end = nend;
      if (b >= wb + LPR) {
        wb += LPR;
        wlo = nlo;
        whi = nhi;
        load_win(wb + LPR, nlo, nhi);
      }
      bounds(b + 1, npos, nend);
      continue;
    }
    if (pre_b != b || pre_pos != pos) {
      cp_async_wait_all();
      __syncwarp(gmask);
      fetch_chunk(buf, b, pos, end, npos, nend);
    }
    cp_async_wait_all();
    __syncwarp(gmask);
    const int4* rs = ring + buf * U;
    const int t1 = min(U, end - pos);
    int t2 = b + 1 < nb ? min(U - t1, nend - npos) : 0;
    if (t2 > 0) {
      // a slot of block b+1 that block b's part of the chunk also holds would
      // be loaded before that part stores it: end the chunk at the block edge
      bool clash = false;
      for (int i = t1 + sl; i < t1 + t2; i += LPR) {
        const int si = lds2(&rs[i]).x;
        for (int j = 0; j < t1; ++j) clash |= lds2(&rs[j]).x == si;
      }
      if (__any_sync(gmask, clash)) t2 = 0;
    }
    const int n = t1 + t2;
    // the next chunk's position, and the prefetch of its records
    int qb = b, qpos = pos + t1, qend = end, qnpos = npos, qnend = nend;
    if (t2 > 0 || pos + t1 >= end) {
      qb = b + 1;
      qpos = npos + t2;
      qend = nend;
      bounds(b + 2, qnpos, qnend);
    }
    if (qb < nb && qpos < qend) {
      fetch_chunk(buf ^ 1, qb, qpos, qend, qnpos, qnend);
      pre_b = qb;
      pre_pos = qpos;
    } else {
      pre_b = -1;
    }
    // gather into shared memory: the first record of every slot run copies
    // the row; writes copy v_t (or load it into registers).  Each lane copies
    // and later reads only its own F columns, so its own wait makes them
    // visible.
    uint32_t head = 0, last = 0;  // per record: first / last of its slot run
    VRaw<Tv, F> vr[SM::kVReg ? U : 1];
    // snapshot mode: which records' rows the walk has already written (bit u),
    // all flags loaded before the copies that depend on them
    uint32_t written = 0;
    if constexpr (SAVE) {
      uint8_t fl[U];
#pragma unroll
      for (int u = 0; u < U; ++u) fl[u] = u < n ? toh[unsigned(lds2(&rs[u]).x)] : uint8_t(0);
#pragma unroll
      for (int u = 0; u < U; ++u) written |= uint32_t(fl[u] != 0) << u;
    }
    {
      int prev = -1;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (u >= n) break;
        const int2 sm = lds2(&rs[u]);  // slot, meta
        if (u == 0 || u == t1 || sm.x != prev) {
          head |= 1u << u;
          if (u > 0) last |= 1u << (u - 1);
          const float* src = Mh + size_t(unsigned(sm.x)) * dv;
          if constexpr (SAVE) {
            if (!((written >> u) & 1u)) src = M0h + size_t(unsigned(sm.x)) * dv;
          }
          cp_bytes<F * 4>(mrow + u * dv, src);
        }
        if (!(sm.y & 1)) {
          if constexpr (SM::kVReg)
            ld_v<Tv, F>(vh + size_t(sm.y >> 1) * dv, vr[SM::kVReg ? u : 0]);
          else if constexpr (F * sizeof(Tv) >= 4)
            cp_bytes<F * sizeof(Tv)>(vrow + u * dv, vh + size_t(sm.y >> 1) * dv);
          else
            vrow[u * dv] = vh[size_t(sm.y >> 1) * dv];
        }
        prev = sm.x;
      }
      last |= 1u << (n - 1);
      cp_async_commit();
      cp_async_wait_all();
    }
    // apply in order; store each run's row after its last record
    {
      float cur[F];
      bool dirty = false;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (u >= n) break;
        const int4 r = lds4(&rs[u]);
        const float f1 = __int_as_float(r.z), f2 = __int_as_float(r.w);
        if ((head >> u) & 1u) {
#pragma unroll
          for (int j = 0; j < F; ++j) cur[j] = mrow[u * dv + j];
        }
        if constexpr (SAVE) {
          // the row as this record finds it (record index as in rec)
          const size_t ri = u < t1 ? (size_t(bh) * p.nblk + b) * p.E + pos + u
                                   : (size_t(bh) * p.nblk + b + 1) * p.E + npos + (u - t1);
          st_row<F>(sv.snap + ri * dv + sl * F, cur);
        }
        if (!(r.y & 1)) {
#pragma unroll
          for (int j = 0; j < F; ++j) {
            float vj;
            if constexpr (SM::kVReg) vj = v_at<Tv, F>(vr[SM::kVReg ? u : 0], j);
            else vj = to_f32(vrow[u * dv + j]);
            cur[j] = fmaf(f1, cur[j], f2 * vj);
          }
          dirty = true;
        } else if constexpr (!SAVE) {
          red_row<F>(oh + size_t(r.y >> 1) * dv, cur, f1);
        }
        if ((last >> u) & 1u) {
          if (dirty) {
            st_row<F>(Mh + size_t(unsigned(r.x)) * dv, cur);
            if constexpr (SAVE) toh[unsigned(r.x)] = 1;  // every lane: its own later loads see it
          }
          dirty = false;
        }
      }
    }
    // every lane has read this chunk's records before the ring slot is reused
    __syncwarp(gmask);
    buf ^= (pre_b >= 0) ? 1 : 0;
    // advance
    if (qb != b) {
      b = qb;
      pos = qpos;
      end = qend;
      npos = qnpos;
      nend = qnend;
      if (b >= wb + LPR) {
        wb += LPR;
        wlo = nlo;
        whi = nhi;
        load_win(wb + LPR, nlo, nhi);
      }
    } else {
      pos = qpos;
    }
  }
  cp_async_wait_all();
}

template <typename Tv, int LPR, int F, bool SAVE>
static cudaError_t launch_recur_t(const Plan& p, const void* v, float* M, float* o,
                                  const int4* rec, const int* roff, int t0, int tlen,
                                  cudaStream_t s, SaveIO sv) {
  const size_t smem = RecurSmem<Tv, LPR, F>::total;
  cudaError_t e = cudaFuncSetAttribute(k_recur<Tv, LPR, F, SAVE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  // heads in groups of p.HG per launch, so that the rows in use at a time
  // span a bounded range of the table (address translation reach)
  for (int bh0 = 0; bh0 < p.BH; bh0 += p.HG) {
    const int nbh = min(p.HG, p.BH - bh0);
    const long long threads = (long long)nbh * p.S * LPR;
    const int grid = int((threads + kRecurThreads - 1) / kRecurThreads);
    k_recur<Tv, LPR, F, SAVE><<<grid, kRecurThreads, smem, s>>>(
        p, (const Tv*)v, M, o, rec, roff, t0, tlen, bh0, nbh, sv);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Floats per lane F for a row width: kRecurMaxF, kept within [d_v / 32, d_v / 4]
// so that a row takes 4..32 lanes.
constexpr int recur_floats_per_lane(int dv) {
  return (kRecurMaxF < dv / 4 ? (kRecurMaxF > dv / 32 ? kRecurMaxF : dv / 32) : dv / 4) < 1
             ? 1
             : (kRecurMaxF < dv / 4 ? (kRecurMaxF > dv / 32 ? kRecurMaxF : dv / 32) : dv / 4);
}

int recur_lanes_per_row(int dv) { return dv / recur_floats_per_lane(dv); }

template <typename Tv, int DV>
static cudaError_t launch_recur_w(const Plan& p, const void* v, float* M, float* o,
                                  const int4* rec, const int* roff, int t0, int tlen,
                                  cudaStream_t s, SaveIO sv) {
  constexpr int F = recur_floats_per_lane(DV);
  if (sv.snap) return launch_recur_t<Tv, DV / F, F, true>(p, v, M, o, rec, roff, t0, tlen, s, sv);
  return launch_recur_t<Tv, DV / F, F, false>(p, v, M, o, rec, roff, t0, tlen, s,
                                               SaveIO{nullptr, nullptr, nullptr});
}

template <typename Tv>
static cudaError_t launch_recur_dt(const Plan& p, const void* v, float* M, float* o,
                                   const int4* rec, const int* roff, int t0, int tlen,
                                   cudaStream_t s, SaveIO sv) {
  switch (p.dv) {
    case 4: return launch_recur_w<Tv, 4>(p, v, M, o, rec, roff, t0, tlen, s, sv);
    case 8: return launch_recur_w<Tv, 8>(p, v, M, o, rec, roff, t0, tlen, s, sv);
    case 16: return launch_recur_w<Tv, 16>(p, v, M, o, rec, roff, t0, tlen, s, sv);
    case 32: return launch_recur_w<Tv, 32>(p, v, M, o, rec, roff, t0, tlen, s, sv);
    case 64: return launch_recur_w<Tv, 64>(p, v, M, o, rec, roff, t0, tlen, s, sv);
    case 128: return launch_recur_w<Tv, 128>(p, v, M, o, rec, roff, t0, tlen, s, sv);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_recur(const Plan& p, const void* v, float* M, float* o, const int4* rec,
                         const int* roff, int t0, int tlen, cudaStream_t s, SaveIO sv) {
  if (p.dtype == SDM_DTYPE_F32)
    return launch_recur_dt<float>(p, v, M, o, rec, roff, t0, tlen, s, sv);
  return launch_recur_dt<__nv_bfloat16>(p, v, M, o, rec, roff, t0, tlen, s, sv);
}

}  // namespace sdm
