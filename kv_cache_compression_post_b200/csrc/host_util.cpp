#include "host_util.h"

#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>
#include <vector>

namespace kvb {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::mutex g_info_mu;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}
}  // namespace

namespace {
std::atomic<unsigned long long> g_launches{0};

// Launch tracing: one record per traced launch, its two events taken from a
// per-device pool and given back when the records are read.
struct TraceRec {
  const char* kernel;
  int device;
  cudaEvent_t e0, e1;
  bool closed;
};
std::atomic<bool> g_trace_on{false};
std::mutex g_trace_mu;
std::vector<TraceRec> g_trace;
std::vector<cudaEvent_t> g_event_pool[kMaxDevices];
constexpr size_t kMaxTraceRecords = 1 << 16;

cudaEvent_t pooled_event(int dev) {
  std::vector<cudaEvent_t>& pool = g_event_pool[dev];
  if (!pool.empty()) {
    cudaEvent_t e = pool.back();
    pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

LaunchTrace::LaunchTrace(const char* kernel, cudaStream_t st) : kernel_(kernel), st_(st) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_trace_on.load(std::memory_order_relaxed)) return;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (g_trace.size() >= kMaxTraceRecords) return;
  cudaEvent_t e0 = pooled_event(dev), e1 = pooled_event(dev);
  if (!e0 || !e1) {
    if (e0) g_event_pool[dev].push_back(e0);
    if (e1) g_event_pool[dev].push_back(e1);
    return;
  }
  if (cudaEventRecord(e0, st) != cudaSuccess) {
    g_event_pool[dev].push_back(e0);
    g_event_pool[dev].push_back(e1);
    return;
  }
  slot_ = static_cast<int>(g_trace.size());
  g_trace.push_back(TraceRec{kernel, dev, e0, e1, false});
}

LaunchTrace::~LaunchTrace() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (static_cast<size_t>(slot_) >= g_trace.size()) return;  // records were read meanwhile
  TraceRec& r = g_trace[slot_];
  r.closed = cudaEventRecord(r.e1, st_) == cudaSuccess;
}

bool current_device(DeviceInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_info_mu);
  DeviceInfo& d = g_info[dev];
  if (d.device != dev) {
    DeviceInfo t;
    t.device = dev;
    if (cudaDeviceGetAttribute(&t.n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&t.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&t.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
    d = t;
  }
  *out = d;
  return true;
}

bool make_tmap_bf16(CUtensorMap* m, const void* base, int d, long long rows, int heads, int box_rows) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode || !base || rows <= 0 || heads <= 0 || (d % 64) != 0) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_aug(CUtensorMap* m, const void* base, long long rows, int heads, int box_rows) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode || !base || rows <= 0 || heads <= 0) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[3] = {32, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {64, static_cast<cuuint64_t>(rows) * 64};
  cuuint32_t box[3] = {16, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace kvb

extern "C" unsigned long long kvb_launch_count(void) { return kvb::g_launches.load(std::memory_order_relaxed); }

extern "C" kvb_status kvb_trace_enable(int32_t enable) {
  using namespace kvb;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  for (TraceRec& r : g_trace) {
    g_event_pool[r.device].push_back(r.e0);
    g_event_pool[r.device].push_back(r.e1);
  }
  g_trace.clear();
  g_trace_on.store(enable != 0, std::memory_order_relaxed);
  return KVB_OK;
}

extern "C" kvb_status kvb_trace_read(kvb_trace_record* out, int32_t max_records, int32_t* n_out) {
  using namespace kvb;
  if (!n_out || max_records < 0 || (max_records > 0 && !out)) return KVB_E_INVAL;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  int prev = -1;
  cudaGetDevice(&prev);
  kvb_status result = KVB_OK;
  int32_t n = 0;
  for (TraceRec& r : g_trace) {
    float ms = -1.f;
    if (r.closed && cudaSetDevice(r.device) == cudaSuccess && cudaEventSynchronize(r.e1) == cudaSuccess &&
        cudaEventElapsedTime(&ms, r.e0, r.e1) != cudaSuccess)
      ms = -1.f;
    if (ms < 0.f) result = KVB_E_CUDA;
    if (n < max_records) out[n] = kvb_trace_record{r.kernel, ms, r.device};
    ++n;
    g_event_pool[r.device].push_back(r.e0);
    g_event_pool[r.device].push_back(r.e1);
  }
  g_trace.clear();
  if (prev >= 0) cudaSetDevice(prev);
  *n_out = n;
  return result;
}
