// mlstm_fw_static_scratch: the forward pass without a caller-provided
// workspace.  The scratch lives in a fixed-size array that is part of this
// library's device image, so the call itself never allocates device memory.
//
// Who needs it: callers that hand the library their input and output buffers
// but cannot allocate anything themselves -- a plugin hook in a host
// framework that exposes tensors but no allocator, or a latency-critical loop
// that forbids cudaMalloc after start-up because it can synchronise the whole
// device.
//
// Costs and limits:
//  * every GPU that loads this library holds kStaticScratchBytes (16 MiB) of
//    device memory until the process exits, whether or not the call is used;
//  * problems whose workspace (mlstm_fw_workspace_size) exceeds that size are
//    rejected with MLSTM_ERR_SCRATCH_TOO_SMALL before anything is launched;
//  * all calls share the one array: calls that overlap on the GPU (other
//    streams, other host threads) race with each other and must be serialised
//    by the caller;
//  * the first call in a CUDA context looks up the array's device address
//    (with that context current) and caches it for that context; make that
//    first call before any stream capture.  A cudaDeviceReset ends the
//    context, and the next call looks the address up again in the new one.
// The array keeps whatever the last call left in it.  Nothing needs clearing:
// every scratch byte a call reads was written earlier in the same call.
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_address.h"
#include "mlstm_fw.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

mlstm::DeviceAddressCache g_scratch_cache;

// Device address of g_static_scratch in the current context (looked up once
// per context); nullptr, with the runtime's error cleared, if the lookup
// fails.
void* scratch_address() {
  return mlstm::cached_device_address(
      g_scratch_cache, [](void** p) { return cudaGetSymbolAddress(p, g_static_scratch); });
}

}  // namespace

extern "C" {

size_t mlstm_fw_static_scratch_capacity(void) { return kStaticScratchBytes; }

mlstm_status mlstm_fw_static_scratch(const void* Q, const void* K, const void* V,
                                     const float* i_pre, const float* f_pre, const float* C0,
                                     const float* n0, const float* m0, void* H, float* C_T,
                                     float* n_T, float* m_T, int B, int NH, int T, int DK, int DV,
                                     int chunk_size, mlstm_dtype dtype,
                                     mlstm_gate_mode gate_mode, mlstm_algo algo,
                                     mlstm_stream_t stream) {
  size_t need = 0;
  mlstm_status s = mlstm_fw_workspace_size(B, NH, T, DK, DV, chunk_size, dtype, algo, &need);
  if (s != MLSTM_OK) return s;
  if (need > kStaticScratchBytes) return MLSTM_ERR_SCRATCH_TOO_SMALL;
  void* scratch = scratch_address();
  if (!scratch) return MLSTM_ERR_CUDA;
  return mlstm_fw(Q, K, V, i_pre, f_pre, C0, n0, m0, H, C_T, n_T, m_T, B, NH, T, DK, DV,
                  chunk_size, dtype, gate_mode, algo, scratch, kStaticScratchBytes, stream);
}

}  // extern "C"
