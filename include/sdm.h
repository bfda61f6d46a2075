/*
 * sdm.h -- C ABI of the Sparse Delta Memory (SDM) forward pass on NVIDIA B200 (sm_100a).
 *
 * The operation (SDM technical summaries of arXiv 2607.07386, gist.science,
 * es "Resumen Tecnico: Memoria Delta Dispersa (SDM)" / fr "Resume Technique :
 * Memoire Delta Creuse (SDM)", section "Mecanismo Central" items 1-4): each
 * (b,h) head keeps a slot table M in R^{N x d_v}, N = n_sub^2.  At step t the
 * projected key k'_t and query q'_t are each cut into two contiguous halves;
 * half 1 is scored against codebook C1, half 2 against C2 (n_sub rows of
 * d_qk/2 each); each half keeps its top-k; the k x k outer-sum candidates give
 * slot i = i1 * n_sub + i2 with score s1[i1] + s2[i2] (float32); k' selects the
 * top-W write slots, q' the top-R read slots (lower index wins ties).  Each
 * write slot is gated then delta-updated,
 *     M~[i] = alpha_t * M[i];  M[i] = M~[i] + beta_t * w_i * (v_t - M~[i]),
 * with w = softmax over the W selected write scores; other slots are left
 * bit-identical.  o_t = sum_r u_r * M_t[r] over the R read slots, u = softmax
 * over the R read scores, taken after step t's write.
 *
 * Conventions for every entry point:
 *  - Pointers are CUDA device pointers unless stated otherwise; the caller
 *    allocates and owns every buffer, including the workspace.  The library
 *    allocates no device memory and keeps no state between calls.
 *  - Layouts are dense row-major, no padding:
 *      q, k   [B][H][T][d_qk]   (in_dtype)
 *      v      [B][H][T][d_v]    (in_dtype)
 *      alpha, beta [B][H][T]    float32
 *      C1, C2 [H][n_sub][d_qk/2] (in_dtype)
 *      M      [B][H][N][d_v]    float32, N = n_sub^2
 *      o      [B][H][T][d_v]    float32
 *      idx_w / w_w [B][H][T][W] int32 / float32 (idx_r / w_r likewise with R)
 *  - Every device pointer must be 16-byte aligned, except the per-step gate
 *    arrays (alpha, beta, a), which need 4 bytes; outputs must not alias
 *    inputs or each other.  With T == 0 nothing is enqueued and no pointer is
 *    read (empty tensors may pass NULL).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  All work
 *    is enqueued on it and the call returns without waiting; results are
 *    valid after the stream is synchronised.
 *  - Return value: SDM_OK, or an sdm_status code.  Argument errors are found
 *    on the host before anything is enqueued.  A failure to enqueue returns
 *    SDM_ERR_CUDA.  A check made by the kernels themselves (an index out of
 *    range, a bounded wait that ran out) is recorded in the workspace's status
 *    word; read it with sdm_get_device_status after synchronising.
 *  - No C++ exception crosses this boundary.
 */
#ifndef SDM_H_
#define SDM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SDM_API __attribute__((visibility("default")))
#else
#define SDM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Problem sizes.  in_dtype applies to q', k', v, C1 and C2. */
typedef struct sdm_dims {
  int32_t B;        /* batch */
  int32_t H;        /* heads */
  int32_t T;        /* steps */
  int32_t d_qk;     /* projected key/query width (even); halves of d_qk/2 */
  int32_t d_v;      /* slot row width: 4, 8, 16, 32, 64 or 128 */
  int32_t n_sub;    /* rows per sub-key codebook; N = n_sub^2 < 2^31 */
  int32_t k;        /* per-half top-k, 1 <= k <= n_sub */
  int32_t W;        /* write slots per step, 1 <= W <= k^2 */
  int32_t R;        /* read slots per step, 1 <= R <= k^2 */
  int32_t in_dtype; /* SDM_DTYPE_F32 or SDM_DTYPE_BF16 */
} sdm_dims;

enum { SDM_DTYPE_F32 = 0, SDM_DTYPE_BF16 = 1 };

enum {
  SDM_OK = 0,
  SDM_ERR_NULL = 1,        /* a required pointer is NULL */
  SDM_ERR_DIMS = 2,        /* sizes out of range or inconsistent */
  SDM_ERR_ALIGN = 3,       /* a pointer is misaligned (16 bytes; 4 for gate arrays) */
  SDM_ERR_WORKSPACE = 4,   /* workspace missing or smaller than sdm_workspace_bytes */
  SDM_ERR_UNSUPPORTED = 5, /* valid sizes this build has no kernel for */
  SDM_ERR_CUDA = 6,        /* a CUDA call failed while enqueueing */
  SDM_ERR_DEVICE = 7,      /* a kernel's own check fired (see sdm_get_device_status) */
  SDM_ERR_SCRATCH_LIMIT = 8 /* sdm_forward_noalloc: problem does not fit its 64 MiB scratch */
};

/* Device status bits recorded by the kernels (sdm_get_device_status). */
enum {
  SDM_DEV_BAD_INDEX = 1,    /* a slot or list index outside its range (access skipped) */
  SDM_DEV_CAPACITY = 2,     /* a per-row survivor list overflowed its capacity */
  SDM_DEV_TIMEOUT = 4,      /* a bounded wait ran out (work skipped) */
  SDM_DEV_BAD_LIST = 8      /* a given selection list repeats a slot within one step (applied in order) */
};

/*
 * Bytes of device workspace sdm_forward / sdm_select / sdm_recur need for
 * `dims` (0 if dims are invalid).  Depends on dims only.  The workspace
 * holds per-call scratch (per-half survivor lists, the write/read plans of
 * the recurrence, a status word); its contents need not be initialised and
 * are overwritten by each call.  Long sequences run as several time chunks,
 * so that it stays near 4 GiB at most.
 */
SDM_API size_t sdm_workspace_bytes(const sdm_dims* dims);

/*
 * Full forward pass ("Mecanismo Central" items 1-4).
 *   q, k, v, alpha, beta, C1, C2: inputs (read only), layouts above.
 *   M_inout: read as M_0 and overwritten with M_T.
 *   o_out:   written with o_0 .. o_{T-1}.
 *   workspace: ws_bytes >= sdm_workspace_bytes(dims) device bytes.
 * Calls on the same workspace must be serialised (same stream or an event).
 */
SDM_API int sdm_forward(const void* q, const void* k, const void* v, const float* alpha,
                const float* beta, const void* C1, const void* C2, float* M_inout,
                float* o_out, const sdm_dims* dims, void* workspace, size_t ws_bytes,
                void* stream);

/*
 * Selection only (item 2): the write list from k' and the read list from q',
 * each in rank order (score descending, slot ascending), with their softmax
 * weights.  idx_w / w_w: [B][H][T][W]; idx_r / w_r: [B][H][T][R].
 * v, alpha, beta, M are not needed.
 */
SDM_API int sdm_select(const void* q, const void* k, const void* C1, const void* C2, int32_t* idx_w,
               float* w_w, int32_t* idx_r, float* w_r, const sdm_dims* dims, void* workspace,
               size_t ws_bytes, void* stream);

/*
 * Recurrence only (items 3-4) from given selection lists: the write slots
 * idx_w with weights w_w and the read slots idx_r with weights u = w_r, as
 * sdm_select produces them (any order within a step).  The W slots of one
 * step should be distinct, as should the R slots: a repeat is applied in list
 * order and flagged (SDM_DEV_BAD_LIST); a slot outside [0, N) is skipped and
 * flagged (SDM_DEV_BAD_INDEX).  q, k, C1, C2 are not needed; in_dtype applies
 * to v; d_qk and n_sub still give N and must be valid.
 */
SDM_API int sdm_recur(const void* v, const float* alpha, const float* beta, const int32_t* idx_w,
              const float* w_w, const int32_t* idx_r, const float* w_r, float* M_inout,
              float* o_out, const sdm_dims* dims, void* workspace, size_t ws_bytes,
              void* stream);

/*
 * The forward pass for short calls -- decoding one step (T = 1) or a few at a
 * time with M carried from call to call -- fused into one kernel that needs no
 * workspace ("Mecanismo Central" items 1-4; the inference use of the method
 * in "Resultados").  One CTA per (b,h) head runs the call's T steps in order,
 * each on chip: scoring on CUDA cores (float32 FMA), the exact per-half top-k,
 * the same staircase merge and softmax weights as sdm_forward, the gated delta
 * writes, then the reads.  Same inputs, outputs and layouts as sdm_forward; o
 * is reduced in a fixed order (identical calls give identical bits).  Its
 * float32 scores can round differently from sdm_forward's (tensor cores) in the
 * last bits, so the two may choose differently at exact near-ties only.
 *   idx_w, w_w, idx_r, w_r: optional (all four NULL, or all four given): the
 *     selections of every step in rank order, as sdm_select writes them.
 * Sizes this kernel serves: n_sub <= 1024, k <= 256, d_v <= 128, d_qk/2 a
 * power-of-two multiple of 8 (bf16) or 4 (float32) up to 32 times that, and
 * its shared memory (staircase tables grow with W and R) within 227 KB;
 * others return SDM_ERR_UNSUPPORTED before anything is enqueued.  Longer
 * sequences are better served by sdm_forward.  Asynchronous on `stream`.
 */
SDM_API int sdm_step(const void* q, const void* k, const void* v, const float* alpha,
                     const float* beta, const void* C1, const void* C2, float* M_inout,
                     float* o_out, int32_t* idx_w, float* w_w, int32_t* idx_r, float* w_r,
                     const sdm_dims* dims, void* stream);

/*
 * The forward pass with the Raven page's selective-decay write rule ("Raven -
 * Modelado de Secuencias de Alta Recuperacion con Enrutamiento de Memoria
 * Dispersa", section 2.2) in place of the gated delta write, on SDM's
 * product-key selection: the router weight of write slot i is the sigmoid of
 * its selected score normalised over the W selected slots, r_i = s(x_i) /
 * sum_j s(x_j), and each selected row decays toward v_t,
 *     M[i] = exp(a_t r_i) M[i] + (1 - exp(a_t r_i)) v_t,
 * unselected rows staying frozen; the read is SDM's (softmax over the R read
 * scores, after the write).  a [B][H][T] float32 holds the decay rate a_t
 * (<= 0; 0 freezes).  Everything else, including the workspace
 * (sdm_workspace_bytes), as sdm_forward.
 */
SDM_API int sdm_forward_decay(const void* q, const void* k, const void* v, const float* a,
                              const void* C1, const void* C2, float* M_inout, float* o_out,
                              const sdm_dims* dims, void* workspace, size_t ws_bytes,
                              void* stream);

/*
 * sdm_forward that also records caller-created CUDA events (cudaEvent_t) on
 * `stream` at the boundaries of its kernel phases, for timing: for time chunk c
 * (see sdm_query_plan) events[5c+0] before scoring, [5c+1] after scoring,
 * [5c+2] after the merge kernel, [5c+3] after the plan kernel, [5c+4] after
 * the recurrence kernel.
 * Boundaries past n_events are not recorded.  Same results as sdm_forward.
 */
SDM_API int sdm_forward_timed(const void* q, const void* k, const void* v, const float* alpha,
                              const float* beta, const void* C1, const void* C2, float* M_inout,
                              float* o_out, const sdm_dims* dims, void* workspace,
                              size_t ws_bytes, void* stream, void* const* events, int n_events);

/*
 * sdm_forward without a workspace argument, for callers that cannot allocate
 * device memory: a plugin whose host framework owns the whole device-memory
 * budget and forbids allocations on the execution path, or a latency-critical
 * loop that cannot pay for the device synchronisation cudaMalloc / cudaFree
 * imply.  The pages have no counterpart; this is an interface convenience.
 *
 * Its scratch is one file-scope device array of 64 MiB that every GPU loading
 * this library holds until the process exits.  The call runs in time chunks
 * short enough for its scratch to fit there (the results do not depend on the
 * chunk length); a problem that does not fit even with the shortest chunk (one
 * plan block of steps, see sdm_query_plan) is rejected with
 * SDM_ERR_SCRATCH_LIMIT before anything is enqueued.  Runs on the current
 * device; `stream` must belong to it.  Every call looks up the array's device
 * address (cudaGetSymbolAddress, which allocates nothing) with that device
 * current; the first call on a device may also load the library's device
 * code, so make it before any stream capture.  Every call shares the one array
 * and it keeps the last call's contents (nothing in it needs to start at
 * zero), so calls that overlap on the GPU race: serialise them (one stream, or
 * events).  The kernels' status word is not readable through this entry point.
 * Allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 * Results and other return codes as sdm_forward.
 */
SDM_API int sdm_forward_noalloc(const void* q, const void* k, const void* v, const float* alpha,
                                const float* beta, const void* C1, const void* C2,
                                float* M_inout, float* o_out, const sdm_dims* dims,
                                void* stream);

/*
 * How the library will run `dims` (host only, no GPU work).  Writes up to n
 * values into out: [0] tensor-core scoring (1) or CUDA-core scoring (0),
 * [1] survivor capacity per half-row, [2] steps per plan block P,
 * [3] recurrence streams per head S, [4] steps per time chunk, [5] number of
 * chunks, [6] kernel launches per sdm_forward call, [7] slot buckets per head,
 * [8] scoring mode: 0 CUDA cores, 1 tensor cores with the exact top-k taken in
 * the same kernel, 2 tensor-core threshold filter then a separate exact top-k.
 * Returns SDM_OK or a dims error.
 */
SDM_API int sdm_query_plan(const sdm_dims* dims, int64_t* out, int n);

/*
 * Copy the device status word of the last call made with `workspace` into
 * *status (SDM_DEV_* bits, 0 = clean) and *info (the first offending index, or
 * -1).  Synchronises `stream`.  Returns SDM_OK, SDM_ERR_NULL,
 * SDM_ERR_WORKSPACE or SDM_ERR_CUDA.
 */
SDM_API int sdm_get_device_status(const void* workspace, size_t ws_bytes, int32_t* status,
                          int32_t* info, void* stream);

/* Static text for a return code (never NULL). */
SDM_API const char* sdm_status_string(int status);

/*
 * Gradients of the forward pass, for training (the pages make the initial
 * table M_0 a learned parameter, "Estado Inicial Aprendido"; they give no
 * backward pass).  The gradient is that of "Mecanismo Central" items 2-4 with
 * the discrete choices (each half's top-k, the top-W / top-R candidates) held
 * at the ones the forward made -- they are piecewise constant in the inputs.
 * Given the forward's inputs, the table it started from (M0, read only: keep a
 * copy, since sdm_forward overwrites M_inout), its selections as sdm_select
 * writes them (idx_w, w_w, idx_r, w_r; any order within a step), d_o = dL/do
 * [B][H][T][d_v] float32 and dM_T = dL/dM_T [B][H][N][d_v] float32 (NULL for
 * 0), it writes float32 dq, dk [B][H][T][d_qk], dv [B][H][T][d_v], dalpha,
 * dbeta [B][H][T], dC1, dC2 [H][n_sub][d_qk/2] and dM0 [B][H][N][d_v].
 * The whole sequence is one call (a long sequence is split by the caller:
 * segments backward in reverse order, each given the table at its start and
 * the dM0 of the segment after it as its dM_T); the workspace
 * (sdm_backward_workspace_bytes) holds the plan and the row each access of the
 * forward saw, (2W + R) d_v floats per token-head, plus a working table the
 * size of M0 (rows are read from M0 until first written there; M0 is not
 * copied) and one byte per slot marking the rows written.
 * The codebook gradients are accumulated with float atomics, so their last
 * bits vary from call to call.  Same pointer, stream and error conventions as
 * sdm_forward (dalpha, dbeta: 4-byte alignment), with one exception to the
 * no-alias rule: dM0 may be dM_T itself, and dL/dM_0 then accumulates in
 * place (dM_T is overwritten), which saves copying it.
 */
SDM_API size_t sdm_backward_workspace_bytes(const sdm_dims* dims);

SDM_API int sdm_backward(const void* q, const void* k, const void* v, const float* alpha,
                         const float* beta, const void* C1, const void* C2, const float* M0,
                         const int32_t* idx_w, const float* w_w, const int32_t* idx_r,
                         const float* w_r, const float* d_o, const float* dM_T, float* dq,
                         float* dk, float* dv, float* dalpha, float* dbeta, float* dC1,
                         float* dC2, float* dM0, const sdm_dims* dims, void* workspace,
                         size_t ws_bytes, void* stream);

/*
 * Dense Gated DeltaNet (GDN) baseline, for comparison at matched sizes (the
 * SDM summaries' "Resultados": SDM trains 1.49x slower than the dense GDN, an
 * HBM-against-SRAM difference).  Per (b,h) head a dense state S in
 * R^{d_v x d_k} follows the gated delta rule in the SDM pages' gate order
 * ("Mecanismo Central" item 3 applied densely; the delta-mem page's section
 * 2.A writes the dense rule):
 *     S~ = alpha_t S_{t-1};  S_t = S~ + beta_t (v_t - S~ k_t) k_t^T;  o_t = S_t q_t.
 * Evaluated in chunks of 64 steps in float32 on CUDA cores: a parallel pass
 * over all (head, chunk) pairs solves each chunk's unit-lower-triangular
 * system, then a pass per head and block of 8 rows of S walks the chunks in
 * order.  Layouts: q, k [B][H][T][d_k] and v [B][H][T][d_v] (in_dtype);
 * alpha, beta [B][H][T] float32 (alpha > 0); S_inout [B][H][d_v][d_k] float32,
 * read as S_0 and overwritten with S_T; o_out [B][H][T][d_v] float32.  d_k, d_v
 * in {16, 32, 64, 128}.  Keys are expected L2-normalised, as GDN uses them
 * (the delta-mem page normalises q and k for stability).  The workspace holds
 * the per-chunk quantities (sdm_gdn_workspace_bytes, which grows with T).
 * Same pointer, stream and error conventions as sdm_forward.
 */
typedef struct sdm_gdn_dims {
  int32_t B, H, T;
  int32_t d_k;      /* key / query width */
  int32_t d_v;      /* value width (rows of S) */
  int32_t in_dtype; /* SDM_DTYPE_F32 or SDM_DTYPE_BF16, for q, k, v */
} sdm_gdn_dims;

SDM_API size_t sdm_gdn_workspace_bytes(const sdm_gdn_dims* dims);

SDM_API int sdm_gdn_forward(const void* q, const void* k, const void* v, const float* alpha,
                            const float* beta, float* S_inout, float* o_out,
                            const sdm_gdn_dims* dims, void* workspace, size_t ws_bytes,
                            void* stream);

/* Library version, major*10000 + minor*100 + patch. */
SDM_API int sdm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDM_H_ */
