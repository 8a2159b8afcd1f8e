// zha_route_noalloc.cu -- zha_route for callers that cannot allocate device
// memory: the routing scratch lives in a fixed array inside the library.
//
// Some callers cannot hand the library a workspace. A plugin running inside an
// inference server that owns all device memory may be forbidden to call
// cudaMalloc. A serving loop with a fixed memory plan cannot allocate per
// request. A plain C host program may have no device allocator of its own.
// For them this file keeps the scratch zha_route needs (per-level scores,
// compacted kept parents and, unless the caller passes its own, the kept
// bitmaps) in one file-scope __device__ array of ZHA_ROUTE_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds that array until the process exits.
#include <cmath>
#include <cstdio>
#include <mutex>
#include <string>

#include "zha_internal.cuh"

// Shared by every call on a device; it keeps the last call's contents.
static __device__ __align__(256) unsigned char g_route_scratch[ZHA_ROUTE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so it must not be handed to a
// kernel; the address is looked up once per device (with that device current)
// and cached.
zha_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    std::string msg = std::string("zha_route_noalloc: cudaGetDevice: ") + cudaGetErrorString(e);
    return zha_report_error(ZHA_ERR_CUDA, msg.c_str());
  }
  if (dev < 0 || dev >= kMaxDevices)
    return zha_report_error(ZHA_ERR_UNSUPPORTED, "zha_route_noalloc: device index above 63");
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || p == nullptr) {
      std::string msg = std::string("zha_route_noalloc: cudaGetSymbolAddress: ") +
                        cudaGetErrorString(e);
      return zha_report_error(ZHA_ERR_CUDA, msg.c_str());
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ZHA_OK;
}

}  // namespace

extern "C" zha_status zha_route_noalloc(const zha_tree* tree, const float* d_Q, int32_t batch,
                                        int64_t n_tokens, float p, int32_t* d_chunk_ids,
                                        int32_t* d_n_chunks, int32_t max_sel,
                                        uint32_t* d_kept_bits, int32_t* d_status, void* stream) {
  zha_status st = zha_check_route_args(tree, d_Q, batch, n_tokens, d_chunk_ids, d_n_chunks, max_sel,
                                       "zha_route_noalloc");
  if (st != ZHA_OK) return st;
  if ((st = zha_check_p(p, "zha_route_noalloc")) != ZHA_OK) return st;
  const zha::Geom& G = tree->geom;
  const zha::RouteLayout lay = zha::route_layout(G, batch, n_tokens);
  const int64_t need = d_kept_bits ? lay.bytes_no_bits : lay.bytes;
  if (need > int64_t(ZHA_ROUTE_NOALLOC_SCRATCH_BYTES)) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "zha_route_noalloc: this call needs %lld bytes of scratch, the library's fixed "
             "scratch holds %lld; use zha_route with a workspace",
             (long long)need, (long long)ZHA_ROUTE_NOALLOC_SCRATCH_BYTES);
    return zha_report_error(ZHA_ERR_CAPACITY, msg);
  }
  void* base = nullptr;
  st = scratch_address(&base);
  if (st != ZHA_OK) return st;
  // Nothing in the scratch has to start at zero: the select kernel clears each
  // level's bitmap before it sets bits, and scores and kept parents are written
  // before they are read within the call.
  char* ws = static_cast<char*>(base);
  float* sigma = reinterpret_cast<float*>(ws);
  int32_t* kp = reinterpret_cast<int32_t*>(ws + zha::round_up(lay.sig_floats * 4, 256));
  uint32_t* bits = d_kept_bits ? d_kept_bits : reinterpret_cast<uint32_t*>(ws + lay.bytes_no_bits);
  cudaError_t e = zha::launch_route(G, d_Q, batch, n_tokens, zha::uniform_top_p(p), d_chunk_ids,
                                    d_n_chunks, max_sel,
                                    bits, sigma, kp, lay, d_status, tree->store,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    std::string msg = std::string("zha_route_noalloc: ") + cudaGetErrorString(e);
    return zha_report_error(ZHA_ERR_CUDA, msg.c_str());
  }
  return ZHA_OK;
}
