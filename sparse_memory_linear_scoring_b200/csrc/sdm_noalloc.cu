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
// library holds that much memory until the process exits.  Problems whose
// workspace (sdm_workspace_bytes) exceeds it are rejected with
// SDM_ERR_SCRATCH_LIMIT before anything is enqueued.
#include <mutex>

#include "sdm_internal.cuh"

namespace sdm {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per device
constexpr int kMaxDevices = 128;

// The scratch itself.  Host code must not use this name as an address: in host
// code it is only a stand-in for the device symbol; its device address comes
// from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

static void* g_scratch_addr[kMaxDevices];
static std::mutex g_scratch_mu;

// Device address of the scratch on the current device (looked up on the first
// call made with that device current).
static int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SDM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SDM_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return SDM_OK;
}

}  // namespace sdm

extern "C" int sdm_forward_noalloc(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta, const void* C1,
                                   const void* C2, float* M_inout, float* o_out,
                                   const sdm_dims* dims, void* stream) {
  sdm::Plan p;
  const int rc = sdm::make_plan(dims, &p);
  if (rc != SDM_OK) return rc;
  if (p.total > sdm::kStaticScratchBytes) return SDM_ERR_SCRATCH_LIMIT;
  if (p.T == 0) return SDM_OK;
  void* scratch = nullptr;
  const int rs = sdm::scratch_address(&scratch);
  if (rs != SDM_OK) return rs;
  // Nothing in the scratch has to start at zero: the first kernel of the call
  // resets the status word, and every other region is written before it is read.
  return sdm_forward(q, k, v, alpha, beta, C1, C2, M_inout, o_out, dims, scratch,
                     sdm::kStaticScratchBytes, stream);
}
