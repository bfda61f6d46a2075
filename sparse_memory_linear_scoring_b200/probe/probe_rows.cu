// probe_rows.cu -- measurement helper, built into its own library
// (libsdm_probe.so) and not part of the SDM C ABI: the HBM bandwidth of the
// recurrence's access pattern on its own, i.e. random whole-row (256-byte)
// gathers and read-modify-writes of a float32 table, with many rows in flight.
// It gives the pattern's practical ceiling beside the streaming-copy peak.
#include <cuda_runtime.h>
#include <stdint.h>

#include "probe_rows.h"

namespace sdm_probe {
namespace {

__device__ __forceinline__ uint32_t hash32(uint32_t x) {
  x ^= x >> 16; x *= 0x7feb352du;
  x ^= x >> 15; x *= 0x846ca68bu;
  x ^= x >> 16;
  return x;
}

// 8 lanes per 64-float row, 32 bytes per lane; U rows in flight per lane group
template <int U, bool RMW>
__global__ void __launch_bounds__(256) k_probe_rows(float* __restrict__ M, long long nrows,
                                                     int iters, uint32_t seed) {
  const int g = (blockIdx.x * blockDim.x + threadIdx.x) / 8, l = threadIdx.x & 7;
  for (int it = 0; it < iters; ++it) {
    long long r[U];
    float4 a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      r[u] = (long long)(hash32(uint32_t(g) * 7919u + uint32_t(it * U + u) ^ seed) %
                         uint32_t(nrows));
      const float* ptr = M + r[u] * 64 + l * 8;
      asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
                   : "=f"(a[u].x), "=f"(a[u].y), "=f"(a[u].z), "=f"(a[u].w)
                   : "l"(ptr));
      asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
                   : "=f"(b[u].x), "=f"(b[u].y), "=f"(b[u].z), "=f"(b[u].w)
                   : "l"(ptr + 4));
    }
    if (RMW) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float4* ptr = reinterpret_cast<float4*>(M + r[u] * 64 + l * 8);
        a[u].x += 1.f;
        b[u].w += 1.f;
        ptr[0] = a[u];
        ptr[1] = b[u];
      }
    } else {
      float acc = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) acc += a[u].x + b[u].w;
      if (acc == 1.2345e-30f) M[0] = acc;  // keeps the loads; never true for this table
    }
  }
}

}  // namespace
}  // namespace sdm_probe

using namespace sdm_probe;

extern "C" SDM_PROBE_API int sdm_probe_random_rows(float* table, long long nrows, int rmw, int rows_in_flight,
                                     int ctas, int iters, void* stream) {
  if (!table) return SDM_PROBE_ERR_NULL;
  if (nrows < 1 || nrows > 0xffffffffLL || ctas < 1 || iters < 1) return SDM_PROBE_ERR_DIMS;
  if (reinterpret_cast<uintptr_t>(table) & 15) return SDM_PROBE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint32_t seed = 0x5bd1e995u;
  if (rows_in_flight == 4) {
    if (rmw) k_probe_rows<4, true><<<ctas, 256, 0, s>>>(table, nrows, iters, seed);
    else k_probe_rows<4, false><<<ctas, 256, 0, s>>>(table, nrows, iters, seed);
  } else if (rows_in_flight == 8) {
    if (rmw) k_probe_rows<8, true><<<ctas, 256, 0, s>>>(table, nrows, iters, seed);
    else k_probe_rows<8, false><<<ctas, 256, 0, s>>>(table, nrows, iters, seed);
  } else {
    return SDM_PROBE_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? SDM_PROBE_OK : SDM_PROBE_ERR_CUDA;
}
