// zha_host.cu -- per-process, per-device host state of the launchers (see
// zha_host.cuh). Every entry is written once under a mutex and read afterwards.
#include <mutex>
#include <unordered_map>

#include "zha_host.cuh"

namespace zha {

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
int g_sms[kMaxDevices] = {};
std::unordered_map<const void*, size_t> g_smem[kMaxDevices];

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

cudaError_t device_sm_count(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_sms[dev] > 0) {
      *sms = g_sms[dev];
      return cudaSuccess;
    }
  }
  int n = 0;
  if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_sms[dev] = n;
  *sms = n;
  return cudaSuccess;
}

cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices)
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  std::lock_guard<std::mutex> lock(g_mutex);
  auto it = g_smem[dev].find(kernel);
  if (it != g_smem[dev].end() && it->second >= bytes) return cudaSuccess;
  if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes))) !=
      cudaSuccess)
    return e;
  // Every kernel asks for the largest shared-memory carveout, so that
  // back-to-back launches of different kernels need no L1 / shared-memory
  // reconfiguration of the SMs between them.
  if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                int(cudaSharedmemCarveoutMaxShared))) != cudaSuccess)
    return e;
  g_smem[dev][kernel] = bytes;
  return cudaSuccess;
}

}  // namespace zha
