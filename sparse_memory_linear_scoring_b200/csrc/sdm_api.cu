// sdm_api.cu -- the C ABI (include/sdm.h): argument checks, workspace layout,
// and the per-chunk launch sequence on the caller's stream.
//
// Per time chunk [t0, t0+Tc):
//   1. scoring: half scores of k' and q' against C1 / C2 and per-half
//      candidate lists (tensor cores for bf16 shapes they cover, else CUDA
//      cores; rows the tensor-core filter could not settle are redone exactly
//      on CUDA cores);
//   2. merge: top-W / top-R lists with softmax weights (into the workspace, or
//      the caller's lists for sdm_select);
//   3. plan: the lists sorted into the recurrence's per-stream records;
//   4. recur: the gated delta writes and the reads, in time order.
#include <limits.h>
#include <stdint.h>
#include <string.h>

#include "sdm_internal.cuh"

namespace sdm {

size_t score_simt_smem(const Plan& p);
size_t merge_smem_bytes(const Plan& p, int warps);
size_t plan_smem_bytes(const Plan& p);
int recur_lanes_per_row(int dv);

constexpr size_t kMaxSmem = 227 * 1024;

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Staircase of the merge: rows a < k with min(k, n_sel / (a+1)) columns; the
// frontier has one cell per row that stops short of k (rows past the last
// non-empty one contribute only their first empty cell).
static void staircase(int k, int n_sel, int* nc, int* nf) {
  int c = 0, f = 0, prev = -1;
  for (int a = 0; a < k; ++a) {
    int bm = n_sel / (a + 1);
    if (bm > k) bm = k;
    c += bm;
    if (bm < k && !(bm == 0 && prev == 0)) ++f;
    prev = bm;
  }
  *nc = c;
  *nf = f;
}

static bool dv_supported(int dv) {
  return dv == 4 || dv == 8 || dv == 16 || dv == 32 || dv == 64 || dv == 128;
}

int make_plan(const sdm_dims* d, Plan* p, size_t chunk_budget) {
  if (!d) return SDM_ERR_NULL;
  memset(p, 0, sizeof(*p));
  const long long kk = (long long)d->k * d->k;
  if (d->B < 1 || d->H < 1 || d->T < 0 || d->d_qk < 2 || (d->d_qk & 1) || d->n_sub < 1 ||
      d->d_v < 1 || d->k < 1 || d->k > d->n_sub || d->W < 1 || d->R < 1 || d->W > kk ||
      d->R > kk || (d->in_dtype != SDM_DTYPE_F32 && d->in_dtype != SDM_DTYPE_BF16))
    return SDM_ERR_DIMS;
  if ((long long)d->n_sub * d->n_sub >= (1LL << 31)) return SDM_ERR_DIMS;
  if ((long long)d->B * d->H > (1 << 24) || (long long)d->B * d->H * (long long)d->T > (1LL << 40))
    return SDM_ERR_DIMS;
  if (!dv_supported(d->d_v)) return SDM_ERR_UNSUPPORTED;
  if (d->W + d->R > kMaxBlockEntries || d->k > 4096 || d->d_qk > 4096) return SDM_ERR_UNSUPPORTED;
  p->B = d->B; p->H = d->H; p->T = d->T; p->dqk = d->d_qk; p->dh = d->d_qk / 2;
  p->dv = d->d_v; p->n = d->n_sub; p->k = d->k; p->W = d->W; p->R = d->R;
  p->dtype = d->in_dtype;
  p->BH = d->B * d->H;
  p->N = (long long)d->n_sub * d->n_sub;
  p->tc = score_tc_mode(d);
  if (p->tc == 2 && !topk_surv_supported(score_tc_capacity(d, 2))) p->tc = 0;
  if (!p->tc && d->n_sub > 4096) return SDM_ERR_UNSUPPORTED;
  p->C = p->tc ? score_tc_capacity(d, p->tc) : d->k;
  staircase(p->k, p->W, &p->ncW, &p->nfW);
  staircase(p->k, p->R, &p->ncR, &p->nfR);
  if (p->ncW < p->W || p->ncR < p->R) return SDM_ERR_UNSUPPORTED;
  int P = kMaxBlockEntries / (p->W + p->R);
  if (P > 1024) P = 1024;
  if (p->T > 0 && P > p->T) P = p->T;
  if (P < 1) P = 1;
  p->P = P;
  p->E = P * (p->W + p->R);
  // recurrence streams per head: fill the target warp count (a warp holds
  // 32 / LPR streams), keeping at least kStreamMin records per stream and block
  {
    // heads per recurrence launch: their tables span at most kRecurGroupBytes
    const size_t table = size_t(p->N) * p->dv * 4;
    long long HG = (long long)(kRecurGroupBytes / (table > 0 ? table : 1));
    if (HG < 1) HG = 1;
    if (HG > p->BH) HG = p->BH;
    p->HG = int(HG);
    const long long per_warp = 32 / recur_lanes_per_row(p->dv);
    long long S = (kRecurWarps * per_warp + HG - 1) / HG;
    const long long smax = p->E / kStreamMin > 1 ? p->E / kStreamMin : 1;
    if (S > smax) S = smax;
    if (S < 1) S = 1;
    p->S = int(S);
    long long mb = (p->E / kBucketTarget + S - 1) / S;
    if (mb < 1) mb = 1;
    p->mb = int(mb);
    p->NB = int(S * mb);
  }
  // time chunk: bounded workspace
  const size_t per_step = size_t(p->BH) * (4 * 4 + size_t(4) * p->C * 8 + 4 * 4 +
                                           size_t(p->W + p->R) * (16 + 8)) +
                          (size_t(p->BH) * (p->NB + 1) * 4 + size_t(P) - 1) / size_t(P);
  const long long Tround = ((long long)(p->T > 0 ? p->T : 1) + P - 1) / P * P;
  long long Tc = (long long)(chunk_budget / per_step) / P * P;
  if (Tc < P) Tc = P;
  if (Tc > Tround) Tc = Tround;
  p->Tc = int(Tc);
  p->nchunks = p->T == 0 ? 0 : int((p->T + Tc - 1) / Tc);
  p->nblk = int((Tc + P - 1) / P);
  p->merge_smem = merge_smem_bytes(*p, kMergeWarps);
  p->plan_smem = plan_smem_bytes(*p);
  p->recur_smem = 0;
  p->score_smem = p->tc ? score_tc_smem(*p) : score_simt_smem(*p);
  if (p->merge_smem > kMaxSmem || p->plan_smem > kMaxSmem || p->recur_smem > kMaxSmem ||
      p->score_smem > kMaxSmem || (p->tc == 2 && topk_surv_smem(*p) > kMaxSmem))
    return SDM_ERR_UNSUPPORTED;
  const size_t nhr = size_t(p->BH) * p->Tc * 4;
  size_t o = 0;
  p->off_status = o; o = align256(o + sizeof(DevStatus));
  p->off_cnt = o; o = align256(o + nhr * 4);
  p->off_surv = o; o = align256(o + nhr * p->C * 8);
  p->off_redo = o; o = align256(o + nhr * 4);
  p->off_lists = o; o = align256(o + size_t(p->BH) * p->Tc * (p->W + p->R) * 8);
  p->off_rec = o; o = align256(o + size_t(p->BH) * p->nblk * p->E * 16);
  p->off_roff = o; o = align256(o + size_t(p->BH) * p->nblk * (p->NB + 1) * 4);
  p->total = o;
  return SDM_OK;
}

__global__ void k_init(DevStatus* st, int all) {
  if (threadIdx.x == 0) {
    if (all) {
      st->flags = 0;
      st->info = -1;
    }
    st->redo = 0;
  }
}

cudaError_t launch_init(const Plan& p, DevStatus* st, cudaStream_t s) {
  (void)p;
  k_init<<<1, 32, 0, s>>>(st, 1);
  return cudaGetLastError();
}

static cudaError_t launch_reset_redo(DevStatus* st, cudaStream_t s) {
  k_init<<<1, 32, 0, s>>>(st, 0);
  return cudaGetLastError();
}

struct Carve {
  DevStatus* st;
  int* cnt;
  uint2* surv;
  int* redo;
  int32_t* iw; float* ww; int32_t* ir; float* wr;  // this chunk's lists
  int4* rec;
  int* roff;
};

static Carve carve(const Plan& p, void* ws) {
  char* b = static_cast<char*>(ws);
  Carve c;
  c.st = reinterpret_cast<DevStatus*>(b + p.off_status);
  c.cnt = reinterpret_cast<int*>(b + p.off_cnt);
  c.surv = reinterpret_cast<uint2*>(b + p.off_surv);
  c.redo = reinterpret_cast<int*>(b + p.off_redo);
  {
    const size_t rows = size_t(p.BH) * p.Tc;
    char* l = b + p.off_lists;
    c.iw = reinterpret_cast<int32_t*>(l);
    c.ww = reinterpret_cast<float*>(l + rows * p.W * 4);
    c.ir = reinterpret_cast<int32_t*>(l + rows * p.W * 8);
    c.wr = reinterpret_cast<float*>(l + rows * p.W * 8 + rows * p.R * 4);
  }
  c.rec = reinterpret_cast<int4*>(b + p.off_rec);
  c.roff = reinterpret_cast<int*>(b + p.off_roff);
  return c;
}

static int ptr_ok(const void* ptr) {
  if (!ptr) return SDM_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(ptr) & 15) return SDM_ERR_ALIGN;
  return SDM_OK;
}

static int check_ptrs(std::initializer_list<const void*> ps) {
  int worst = SDM_OK;
  for (const void* q : ps) {
    const int rc = ptr_ok(q);
    if (rc == SDM_ERR_NULL) return rc;
    if (rc != SDM_OK) worst = rc;
  }
  return worst;
}

// Per-step scalars (alpha, beta, a) are read one float at a time: 4-byte
// alignment is enough, so a time slice of a caller's gate tensor can be passed
// as it is.
static int check_gates(std::initializer_list<const void*> ps) {
  for (const void* q : ps) {
    if (!q) return SDM_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(q) & 3) return SDM_ERR_ALIGN;
  }
  return SDM_OK;
}

static cudaError_t score_chunk(const Plan& p, const Carve& c, const void* q, const void* k,
                               const void* C1, const void* C2, int t0, int tlen, cudaStream_t s) {
  cudaError_t e;
  if (p.tc) {
    // the redo list of the tensor-core filter starts empty in every chunk (the
    // first chunk's was emptied with the status word)
    if (t0 > 0 && (e = launch_reset_redo(c.st, s)) != cudaSuccess) return e;
    if ((e = launch_score_tc(p, q, k, C1, C2, t0, tlen, c.cnt, c.surv, c.redo, c.st, s)) !=
        cudaSuccess)
      return e;
    if ((e = launch_score_simt(p, q, k, C1, C2, t0, tlen, c.redo, c.st, c.cnt, c.surv, c.st,
                               s)) != cudaSuccess)
      return e;
    // filter mode: the survivor lists are unsorted supersets; keep their exact top-k
    return p.tc == 2 ? launch_topk_surv(p, tlen, c.cnt, c.surv, c.st, s) : cudaSuccess;
  }
  return launch_score_simt(p, q, k, C1, C2, t0, tlen, nullptr, nullptr, c.cnt, c.surv, c.st, s);
}

}  // namespace sdm

using namespace sdm;

extern "C" size_t sdm_workspace_bytes(const sdm_dims* dims) {
  Plan p;
  if (make_plan(dims, &p) != SDM_OK) return 0;
  return p.total;
}

int sdm::forward_with_budget(const void* q, const void* k, const void* v, const float* alpha,
                             const float* beta, const void* C1, const void* C2, float* M_inout,
                             float* o_out, const sdm_dims* dims, void* workspace,
                             size_t ws_bytes, void* stream, void* const* events, int n_events,
                             size_t chunk_budget, int rule) {
  Plan p;
  int rc = make_plan(dims, &p, chunk_budget);
  if (rc != SDM_OK) return rc;
  p.rule = rule;
  if (p.T == 0) return SDM_OK;  // nothing to do; no pointer is read
  rc = check_ptrs({q, k, v, C1, C2, M_inout, o_out, workspace});
  if (rc != SDM_OK) return rc == SDM_ERR_NULL && !workspace ? SDM_ERR_WORKSPACE : rc;
  // the selective-decay rule has no beta
  if ((rc = check_gates({alpha, rule == 1 ? alpha : beta})) != SDM_OK) return rc;
  if (ws_bytes < p.total) return SDM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Carve c = carve(p, workspace);
  auto mark = [&](int j) -> bool {
    if (!events || j >= n_events || !events[j]) return true;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[j]), s) == cudaSuccess;
  };
  if (launch_init(p, c.st, s) != cudaSuccess) return SDM_ERR_CUDA;
  MergeIO mio;
  memset(&mio, 0, sizeof(mio));
  mio.surv_cnt = c.cnt;
  mio.surv = c.surv;
  mio.out_iw = c.iw; mio.out_ww = c.ww; mio.out_ir = c.ir; mio.out_wr = c.wr;
  mio.list_T = p.Tc;
  mio.list_t0 = 0;
  mio.sorted = 0;
  PlanIO pio;
  memset(&pio, 0, sizeof(pio));
  pio.iw = c.iw; pio.ww = c.ww; pio.ir = c.ir; pio.wr = c.wr;
  pio.list_T = p.Tc;
  pio.list_t0 = 0;
  pio.validate = 0;
  pio.alpha = alpha;
  pio.beta = beta;
  pio.rec = c.rec;
  pio.roff = c.roff;
  pio.o = o_out;
  for (int ch = 0; ch < p.nchunks; ++ch) {
    const int t0 = ch * p.Tc;
    const int tlen = (p.T - t0 < p.Tc) ? p.T - t0 : p.Tc;
    if (!mark(5 * ch)) return SDM_ERR_CUDA;
    if (score_chunk(p, c, q, k, C1, C2, t0, tlen, s) != cudaSuccess) return SDM_ERR_CUDA;
    if (!mark(5 * ch + 1)) return SDM_ERR_CUDA;
    if (launch_merge(p, mio, t0, tlen, c.st, s) != cudaSuccess) return SDM_ERR_CUDA;
    if (!mark(5 * ch + 2)) return SDM_ERR_CUDA;
    if (launch_plan(p, pio, t0, tlen, c.st, s) != cudaSuccess) return SDM_ERR_CUDA;
    if (!mark(5 * ch + 3)) return SDM_ERR_CUDA;
    if (launch_recur(p, v, M_inout, o_out, c.rec, c.roff, t0, tlen, s) != cudaSuccess)
      return SDM_ERR_CUDA;
    if (!mark(5 * ch + 4)) return SDM_ERR_CUDA;
  }
  return SDM_OK;
}

extern "C" int sdm_forward(const void* q, const void* k, const void* v, const float* alpha,
                           const float* beta, const void* C1, const void* C2, float* M_inout,
                           float* o_out, const sdm_dims* dims, void* workspace, size_t ws_bytes,
                           void* stream) {
  return forward_with_budget(q, k, v, alpha, beta, C1, C2, M_inout, o_out, dims, workspace,
                             ws_bytes, stream, nullptr, 0, kChunkBudget);
}

extern "C" int sdm_forward_timed(const void* q, const void* k, const void* v, const float* alpha,
                                 const float* beta, const void* C1, const void* C2,
                                 float* M_inout, float* o_out, const sdm_dims* dims,
                                 void* workspace, size_t ws_bytes, void* stream,
                                 void* const* events, int n_events) {
  return forward_with_budget(q, k, v, alpha, beta, C1, C2, M_inout, o_out, dims, workspace,
                             ws_bytes, stream, events, n_events, kChunkBudget);
}

extern "C" int sdm_forward_decay(const void* q, const void* k, const void* v, const float* a,
                                 const void* C1, const void* C2, float* M_inout, float* o_out,
                                 const sdm_dims* dims, void* workspace, size_t ws_bytes,
                                 void* stream) {
  return forward_with_budget(q, k, v, a, nullptr, C1, C2, M_inout, o_out, dims, workspace,
                             ws_bytes, stream, nullptr, 0, kChunkBudget, 1);
}

extern "C" int sdm_query_plan(const sdm_dims* dims, int64_t* out, int n) {
  Plan p;
  const int rc = make_plan(dims, &p);
  if (rc != SDM_OK) return rc;
  const int64_t per_chunk = (p.tc == 2 ? 4 : p.tc ? 3 : 1) + 2 + (p.BH + p.HG - 1) / p.HG;
  const int64_t launches = 1 + per_chunk * p.nchunks - (p.tc && p.nchunks > 0 ? 1 : 0);
  const int64_t vals[9] = {p.tc ? 1 : 0, p.C, p.P, p.S, p.Tc, p.nchunks, launches, p.NB, p.tc};
  for (int i = 0; i < n && i < 9; ++i) out[i] = vals[i];
  return SDM_OK;
}

extern "C" int sdm_select(const void* q, const void* k, const void* C1, const void* C2,
                          int32_t* idx_w, float* w_w, int32_t* idx_r, float* w_r,
                          const sdm_dims* dims, void* workspace, size_t ws_bytes, void* stream) {
  Plan p;
  int rc = make_plan(dims, &p);
  if (rc != SDM_OK) return rc;
  if (p.T == 0) return SDM_OK;  // nothing to do; no pointer is read
  rc = check_ptrs({q, k, C1, C2, idx_w, w_w, idx_r, w_r, workspace});
  if (rc != SDM_OK) return rc == SDM_ERR_NULL && !workspace ? SDM_ERR_WORKSPACE : rc;
  if (ws_bytes < p.total) return SDM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Carve c = carve(p, workspace);
  if (launch_init(p, c.st, s) != cudaSuccess) return SDM_ERR_CUDA;
  MergeIO mio;
  memset(&mio, 0, sizeof(mio));
  mio.surv_cnt = c.cnt;
  mio.surv = c.surv;
  mio.out_iw = idx_w; mio.out_ww = w_w; mio.out_ir = idx_r; mio.out_wr = w_r;
  mio.list_T = p.T;
  mio.sorted = 1;
  for (int ch = 0; ch < p.nchunks; ++ch) {
    const int t0 = ch * p.Tc;
    const int tlen = (p.T - t0 < p.Tc) ? p.T - t0 : p.Tc;
    mio.list_t0 = t0;
    if (score_chunk(p, c, q, k, C1, C2, t0, tlen, s) != cudaSuccess) return SDM_ERR_CUDA;
    if (launch_merge(p, mio, t0, tlen, c.st, s) != cudaSuccess) return SDM_ERR_CUDA;
  }
  return SDM_OK;
}

extern "C" int sdm_recur(const void* v, const float* alpha, const float* beta,
                         const int32_t* idx_w, const float* w_w, const int32_t* idx_r,
                         const float* w_r, float* M_inout, float* o_out, const sdm_dims* dims,
                         void* workspace, size_t ws_bytes, void* stream) {
  Plan p;
  int rc = make_plan(dims, &p);
  if (rc != SDM_OK) return rc;
  if (p.T == 0) return SDM_OK;  // nothing to do; no pointer is read
  rc = check_ptrs({v, idx_w, w_w, idx_r, w_r, M_inout, o_out, workspace});
  if (rc != SDM_OK) return rc == SDM_ERR_NULL && !workspace ? SDM_ERR_WORKSPACE : rc;
  if ((rc = check_gates({alpha, beta})) != SDM_OK) return rc;
  if (ws_bytes < p.total) return SDM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Carve c = carve(p, workspace);
  if (launch_init(p, c.st, s) != cudaSuccess) return SDM_ERR_CUDA;
  PlanIO pio;
  memset(&pio, 0, sizeof(pio));
  pio.iw = idx_w; pio.ww = w_w; pio.ir = idx_r; pio.wr = w_r;
  pio.list_T = p.T;
  pio.validate = 1;
  pio.alpha = alpha;
  pio.beta = beta;
  pio.rec = c.rec;
  pio.roff = c.roff;
  pio.o = o_out;
  for (int ch = 0; ch < p.nchunks; ++ch) {
    const int t0 = ch * p.Tc;
    const int tlen = (p.T - t0 < p.Tc) ? p.T - t0 : p.Tc;
    pio.list_t0 = t0;
    if (launch_plan(p, pio, t0, tlen, c.st, s) != cudaSuccess) return SDM_ERR_CUDA;
    if (launch_recur(p, v, M_inout, o_out, c.rec, c.roff, t0, tlen, s) != cudaSuccess)
      return SDM_ERR_CUDA;
  }
  return SDM_OK;
}

extern "C" int sdm_get_device_status(const void* workspace, size_t ws_bytes, int32_t* status,
                                     int32_t* info, void* stream) {
  if (!workspace || !status) return SDM_ERR_NULL;
  if (ws_bytes < sizeof(DevStatus)) return SDM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DevStatus h;
  if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SDM_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SDM_ERR_CUDA;
  *status = h.flags;
  if (info) *info = h.info;
  return SDM_OK;
}

extern "C" const char* sdm_status_string(int status) {
  switch (status) {
    case SDM_OK: return "ok";
    case SDM_ERR_NULL: return "a required pointer is NULL";
    case SDM_ERR_DIMS: return "sizes out of range or inconsistent";
    case SDM_ERR_ALIGN: return "a device pointer is misaligned (16 bytes; 4 for gate arrays)";
    case SDM_ERR_WORKSPACE: return "workspace missing or too small";
    case SDM_ERR_UNSUPPORTED: return "valid sizes without a kernel in this build";
    case SDM_ERR_CUDA: return "a CUDA call failed while enqueueing";
    case SDM_ERR_DEVICE: return "a kernel's own check fired";
    case SDM_ERR_SCRATCH_LIMIT: return "problem does not fit the 64 MiB static scratch";
    default: return "unknown status";
  }
}

extern "C" int sdm_version(void) { return 100; }
