// sdm_noalloc.cu -- sdm_forward for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: a plugin whose host
// framework owns the whole device-memory budget and forbids allocations on the
// execution path, or a latency-critical loop that must not pay for the device
// synchronisation that cudaMalloc / cudaFree imply.  sdm_forward_noalloc runs
// the same kernels as sdm_forward with its scratch in a fixed, file-scope device
// array instead of a caller-provided workspace, so it allocates nothing.
//
// The array is sized once, at kStaticScratchBytes; every GPU that loads this
// library holds that much memory until the process exits.  The call is planned
// with time chunks short enough for its scratch to fit the array (the results
// do not depend on the chunk length).  A problem whose scratch does not fit
// even with the shortest chunk is rejected with SDM_ERR_SCRATCH_LIMIT before
// anything is enqueued.
#include "sdm_internal.cuh"

namespace sdm {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per device
// Chunk budget handed to the planner: the array less room for the status word
// and the 256-byte alignment of each workspace region.
constexpr size_t kStaticChunkBudget = kStaticScratchBytes - (size_t(64) << 10);

// The scratch itself.  Host code must not use this name as an address: in host
// code it is only a stand-in for the device symbol; its device address comes
// from cudaGetSymbolAddress with the device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

// Device address of the scratch on the current device.  Looked up on every
// call (it allocates nothing), so that no address outlives the context it was
// taken in.
static int scratch_address(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SDM_ERR_CUDA;
  *out = ptr;
  return SDM_OK;
}

}  // namespace sdm

extern "C" int sdm_forward_noalloc(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta, const void* C1,
                                   const void* C2, float* M_inout, float* o_out,
                                   const sdm_dims* dims, void* stream) {
  sdm::Plan p;
  const int rc = sdm::make_plan(dims, &p, sdm::kStaticChunkBudget);
  if (rc != SDM_OK) return rc;
  if (p.total > sdm::kStaticScratchBytes) return SDM_ERR_SCRATCH_LIMIT;
  if (p.T == 0) return SDM_OK;
  void* scratch = nullptr;
  const int rs = sdm::scratch_address(&scratch);
  if (rs != SDM_OK) return rs;
  // Nothing in the scratch has to start at zero: the first kernel of the call
  // resets the status word, and every other region is written before it is read.
  return sdm::forward_with_budget(q, k, v, alpha, beta, C1, C2, M_inout, o_out, dims, scratch,
                                  sdm::kStaticScratchBytes, stream, nullptr, 0,
                                  sdm::kStaticChunkBudget);
}
