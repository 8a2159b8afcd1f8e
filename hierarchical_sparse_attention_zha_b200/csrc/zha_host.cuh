// zha_host.cuh -- host-side helpers shared by the launchers of libzha: the
// driver's tensor-map encoder (looked up once), the multiprocessor count and
// the dynamic shared-memory attribute of each kernel, cached per device so that
// a decode step does not repeat these queries on every call.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace zha {

// cuTensorMapEncodeTiled through the runtime's driver entry point (the library
// links only the CUDA runtime); nullptr when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Multiprocessors of the current device (queried once per device).
cudaError_t device_sm_count(int* sms);

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) and the largest preferred
// shared-memory carveout for `kernel` on the current device, skipped when an
// earlier call on this device already set at least `bytes`. Kernels without
// dynamic shared memory call it with 0 for the carveout alone.
cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes);

template <typename... Args>
inline cudaError_t ensure_dynamic_smem(void (*kernel)(Args...), size_t bytes) {
  return ensure_dynamic_smem(reinterpret_cast<const void*>(kernel), bytes);
}

}  // namespace zha
