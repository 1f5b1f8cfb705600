// Library-wide state of libtpblock: error messages, counters, the device error word, device
// queries and TMA tensor-map encoding.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <vector>
#include <mutex>
#include <string>

#include "sm100.cuh"
#include "tp_common.cuh"

namespace tp {

namespace {
thread_local std::string t_last_error;
std::atomic<uint64_t> g_reductions{0};
std::atomic<uint64_t> g_launches{0};
__device__ uint32_t d_error_word = 0;
}  // namespace

tp_status set_error(tp_status st, const std::string& msg) {
  t_last_error = msg;
  return st;
}
void clear_error() { t_last_error.clear(); }
void count_launch(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
void count_reduction() { g_reductions.fetch_add(1, std::memory_order_relaxed); }

uint32_t* device_error_word() {
  static uint32_t* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, d_error_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint32_t*>(p);
  }
  return addr[dev];
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

bool tensor_cores_usable() {
  static int cache[64] = {0};  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!cache[dev]) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cache[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cache[dev] == 1;
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

tp_status encode_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t batch, uint64_t outer_stride_bytes,
                              uint64_t batch_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = get_encode_fn();
  if (!fn) return set_error(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (outer_stride_bytes % 16 || batch_stride_bytes % 16)
    return set_error(TP_ERR_INVALID_ARG, "tensor-core operand row stride not a multiple of 16 bytes");
  cuuint64_t dims[3] = {inner, outer, batch};
  cuuint64_t strides[2] = {outer_stride_bytes, batch_stride_bytes};
  cuuint32_t box[3] = {box_inner, box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(TP_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string(r) + ")");
  return TP_OK;
}

namespace {
struct ProfRec {
  std::string label;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::atomic<int> g_prof_on{0};
std::vector<ProfRec> g_prof;
}  // namespace

ProfScope::ProfScope(cudaStream_t s, const char* label) : s_(s), label_(label) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return;
  if (cudaEventCreate(&start_) != cudaSuccess) {
    start_ = nullptr;
    return;
  }
  cudaEventRecord(start_, s_);
}

ProfScope::~ProfScope() {
  if (!start_) return;
  cudaEvent_t end = nullptr;
  if (cudaEventCreate(&end) != cudaSuccess) {
    cudaEventDestroy(start_);
    return;
  }
  cudaEventRecord(end, s_);
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof.push_back({label_, start_, end});
}

}  // namespace tp

namespace tp {
// One warp waits, through the same bounded mbarrier wait the tensor-core kernels use, on a
// barrier that nothing ever completes; after limit_ns the wait gives up, raises the abort flag
// and records DEVERR_WAIT_FULL in the device error word, and the kernel returns.
// A counter that no kernel ever increments (the self-test's cross-CTA wait).
__device__ int32_t g_selftest_counter = 0;

__global__ void wait_selftest_kernel(uint64_t limit_ns, uint32_t* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the mbarrier wait of the pipelines, then the counter wait of the one-launch decode MLP
    sm100::mbar_wait(&bar, 0, &abort_flag, err, DEVERR_WAIT_FULL, limit_ns);
    abort_flag = 0;
    wait_counter_at_least(&g_selftest_counter, 1, &abort_flag, err, DEVERR_WAIT_FLAG, limit_ns);
  }
  __syncthreads();
}
}  // namespace tp

extern "C" {

void tp_profile_enable(int32_t on) { tp::g_prof_on.store(on ? 1 : 0); }

void tp_profile_reset(void) {
  std::lock_guard<std::mutex> g(tp::g_prof_mu);
  for (auto& r : tp::g_prof) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  tp::g_prof.clear();
}

int32_t tp_profile_read(int32_t i, char* label, int32_t label_len, uint64_t* launches,
                        double* total_ms) {
  cudaDeviceSynchronize();
  std::lock_guard<std::mutex> g(tp::g_prof_mu);
  std::vector<std::string> order;
  for (auto& r : tp::g_prof)
    if (std::find(order.begin(), order.end(), r.label) == order.end()) order.push_back(r.label);
  if (i < 0 || i >= static_cast<int32_t>(order.size())) return 0;
  uint64_t n = 0;
  double ms = 0.0;
  for (auto& r : tp::g_prof) {
    if (r.label != order[i]) continue;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess) ms += t;
    ++n;
  }
  if (label && label_len > 0) {
    std::snprintf(label, static_cast<size_t>(label_len), "%s", order[i].c_str());
  }
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  return 1;
}

int32_t tp_profile_read_launch(int32_t i, int64_t j, double* ms) {
  cudaDeviceSynchronize();
  std::lock_guard<std::mutex> g(tp::g_prof_mu);
  std::vector<std::string> order;
  for (auto& r : tp::g_prof)
    if (std::find(order.begin(), order.end(), r.label) == order.end()) order.push_back(r.label);
  if (i < 0 || i >= static_cast<int32_t>(order.size()) || j < 0) return 0;
  int64_t k = 0;
  for (auto& r : tp::g_prof) {
    if (r.label != order[i]) continue;
    if (k++ != j) continue;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return 0;
    if (ms) *ms = t;
    return 1;
  }
  return 0;
}

uint64_t tp_reduction_count(void) { return tp::g_reductions.load(); }
void tp_reset_reduction_count(void) { tp::g_reductions.store(0); }
uint64_t tp_launch_count(void) { return tp::g_launches.load(); }
const char* tp_last_error(void) { return tp::t_last_error.c_str(); }

const char* tp_status_string(int32_t s) {
  switch (s) {
    case TP_OK: return "TP_OK";
    case TP_ERR_INVALID_ARG: return "TP_ERR_INVALID_ARG";
    case TP_ERR_SHAPE: return "TP_ERR_SHAPE";
    case TP_ERR_UNSUPPORTED: return "TP_ERR_UNSUPPORTED";
    case TP_ERR_WORKSPACE: return "TP_ERR_WORKSPACE";
    case TP_ERR_CUDA: return "TP_ERR_CUDA";
    case TP_ERR_TIMEOUT: return "TP_ERR_TIMEOUT";
    default: return "TP_ERR_UNKNOWN";
  }
}

tp_status tp_check_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return tp::set_error(TP_ERR_CUDA, std::string("stream: ") + cudaGetErrorString(e));
  uint32_t* w = tp::device_error_word();
  if (!w) return tp::set_error(TP_ERR_CUDA, "device error word unavailable");
  uint32_t v = 0;
  e = cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess)
    return tp::set_error(TP_ERR_CUDA, std::string("error word: ") + cudaGetErrorString(e));
  if (v) {
    const uint32_t zero = 0;
    cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    return tp::set_error(TP_ERR_TIMEOUT,
                         "a bounded device wait ran out (site bits " + std::to_string(v) + ")");
  }
  return TP_OK;
}

int32_t tp_tensor_core_path_available(void) { return tp::tensor_cores_usable() ? 1 : 0; }

tp_status tp_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  tp::clear_error();
  if (limit_us == 0 || limit_us > 1000000u)
    return tp::set_error(TP_ERR_INVALID_ARG, "limit_us must be in 1 .. 1000000");
  uint32_t* w = tp::device_error_word();
  if (!w) return tp::set_error(TP_ERR_CUDA, "device error word unavailable");
  tp::wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull, w);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

int32_t tp_version(void) { return 100; }  // 0.1.0

}  // extern "C"
