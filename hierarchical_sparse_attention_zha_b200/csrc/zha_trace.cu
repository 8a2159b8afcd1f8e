// zha_trace.cu -- optional kernel timing: when enabled (zha_trace_enable), each
// kernel launch of the library is bracketed by two CUDA events recorded on the
// launching stream, so that a caller can read back per-kernel device times
// after it has synchronised. Off by default; when off a launch pays one atomic
// load. The events are created at enable time (host-side driver objects; no
// device memory is allocated).
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "zha_internal.cuh"

namespace zha {

namespace {

struct Rec {
  const char* name;
  int32_t tag;
  cudaEvent_t ev0, ev1;
};

std::atomic<bool> g_on{false};
std::mutex g_mutex;
std::vector<Rec> g_recs;           // events created at enable time
int32_t g_used = 0;                // records taken since the last enable / clear
int32_t g_dropped = 0;
std::string g_filter;              // substring of the kernel name ("" = all)
int32_t g_tag_filter = -1;         // tag to keep (-1 = all)

void destroy_events() {
  for (Rec& r : g_recs) {
    if (r.ev0) cudaEventDestroy(r.ev0);
    if (r.ev1) cudaEventDestroy(r.ev1);
  }
  g_recs.clear();
}

}  // namespace

int trace_begin(const char* name, int32_t tag, cudaStream_t s) {
  if (!g_on.load(std::memory_order_acquire)) return -1;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_filter.empty() && std::strstr(name, g_filter.c_str()) == nullptr) return -1;
  if (g_tag_filter >= 0 && tag != g_tag_filter) return -1;
  if (g_used >= int32_t(g_recs.size())) {
    ++g_dropped;
    return -1;
  }
  const int i = g_used++;
  g_recs[i].name = name;
  g_recs[i].tag = tag;
  cudaEventRecord(g_recs[i].ev0, s);
  return i;
}

void trace_end(int idx, cudaStream_t s) {
  if (idx < 0) return;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (idx < int32_t(g_recs.size())) cudaEventRecord(g_recs[idx].ev1, s);
}

}  // namespace zha

extern "C" {

zha_status zha_trace_enable(int32_t max_records, const char* name_filter, int32_t tag_filter) {
  using namespace zha;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_on.store(false, std::memory_order_release);
  destroy_events();
  g_used = 0;
  g_dropped = 0;
  g_filter = name_filter ? name_filter : "";
  g_tag_filter = tag_filter;
  if (max_records <= 0) return ZHA_OK;
  if (max_records > (1 << 20)) return zha_report_error(ZHA_ERR_INVALID, "zha_trace_enable: max_records above 2^20");
  g_recs.resize(size_t(max_records));
  for (Rec& r : g_recs) {
    r = Rec{"", -1, nullptr, nullptr};
    if (cudaEventCreate(&r.ev0) != cudaSuccess || cudaEventCreate(&r.ev1) != cudaSuccess) {
      destroy_events();
      return zha_report_error(ZHA_ERR_CUDA, "zha_trace_enable: cudaEventCreate failed");
    }
  }
  g_on.store(true, std::memory_order_release);
  return ZHA_OK;
}

int32_t zha_trace_count(void) {
  std::lock_guard<std::mutex> lock(zha::g_mutex);
  return zha::g_used;
}

int32_t zha_trace_dropped(void) {
  std::lock_guard<std::mutex> lock(zha::g_mutex);
  return zha::g_dropped;
}

zha_status zha_trace_read(int32_t i, const char** name, int32_t* tag, float* ms) {
  std::lock_guard<std::mutex> lock(zha::g_mutex);
  if (i < 0 || i >= zha::g_used) return zha_report_error(ZHA_ERR_INVALID, "zha_trace_read: index out of range");
  const zha::Rec& r = zha::g_recs[i];
  if (name) *name = r.name;
  if (tag) *tag = r.tag;
  if (ms) {
    const cudaError_t e = cudaEventElapsedTime(ms, r.ev0, r.ev1);
    if (e != cudaSuccess) {
      std::string msg = std::string("zha_trace_read: ") + cudaGetErrorString(e);
      return zha_report_error(ZHA_ERR_CUDA, msg.c_str());
    }
  }
  return ZHA_OK;
}

void zha_trace_clear(void) {
  std::lock_guard<std::mutex> lock(zha::g_mutex);
  zha::g_used = 0;
  zha::g_dropped = 0;
}

}  // extern "C"
