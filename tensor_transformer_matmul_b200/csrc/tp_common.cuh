// Shared host/device helpers of libtpblock: status plumbing, the device error word, launch
// accounting, bf16 conversions and the elementwise functions of the block.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>
#include <string>

#include "tp_block.h"

namespace tp {

// ----------------------------------------------------------------------------------------------
// host-side status helpers (defined in tp_abi.cu)
// ----------------------------------------------------------------------------------------------
tp_status set_error(tp_status st, const std::string& msg);
void clear_error();
void count_launch(uint64_t n = 1);
void count_reduction();

#define TP_CUDA_TRY(expr)                                                                       \
  do {                                                                                          \
    cudaError_t _e = (expr);                                                                    \
    if (_e != cudaSuccess)                                                                      \
      return ::tp::set_error(TP_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(_e));  \
  } while (0)

// Programmatic dependent launch.  A kernel launched with launch_pdl() may start, and run up to
// its pdl_wait(), while the previous kernel on the stream is still finishing (its launch latency
// and set-up overlap that kernel's tail); pdl_wait() returns once the previous kernel has
// completed and its memory is visible, so stream order is kept for everything after it.  Every
// kernel launched this way calls pdl_wait() before it touches global memory, and pdl_trigger()
// to let the next kernel start launching.  Both are no-ops for an ordinary launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// launch_pdl + error check + launch count (inside a function returning tp_status)
#define TP_LAUNCH_PDL(kern, grid, block, smem, stream, ...)                                     \
  do {                                                                                          \
    cudaError_t _e = ::tp::launch_pdl(kern, grid, block, smem, stream, __VA_ARGS__);           \
    if (_e != cudaSuccess)                                                                      \
      return ::tp::set_error(TP_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(_e)); \
    ::tp::count_launch();                                                                       \
  } while (0)

#define TP_LAUNCH_CHECK()                                                                       \
  do {                                                                                          \
    cudaError_t _e = cudaGetLastError();                                                        \
    if (_e != cudaSuccess)                                                                      \
      return ::tp::set_error(TP_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(_e)); \
    ::tp::count_launch();                                                                       \
  } while (0)

// Zero n 32-bit words.  Used instead of a memset for the small counter arrays in front of a
// kernel, so that the stream keeps a chain of programmatically launched kernels.
static __global__ void zero_words_kernel(uint32_t* p, int64_t n) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = 0u;
}
// The same for two arrays in one launch (a GEMM's counters and those of the kernel after it).
static __global__ void zero_words2_kernel(uint32_t* p, int64_t n, uint32_t* q, int64_t m) {
  pdl_wait();
  pdl_trigger();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n + m;
       i += stride) {
    if (i < n) p[i] = 0u;
    else q[i - n] = 0u;
  }
}


// Brackets one kernel launch with CUDA events when tp_profile_enable(1) is in effect.
class ProfScope {
 public:
  ProfScope(cudaStream_t s, const char* label);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;
 private:
  cudaStream_t s_;
  const char* label_;
  cudaEvent_t start_ = nullptr;
};

int num_sms();                    // SM count of the current device (cached per device)
// Decode (swapped, weight-streaming) GEMMs use whole tiles with rotated k order when there are at
// least as many tiles as SMs; with fewer tiles, stream-K gives every SM an equal share.
// Whether a weight-streaming (decode) GEMM uses the stream-K schedule.  Fewer tiles than SMs:
// always (the k-blocks are split evenly).  More: only for up to 16 tokens with long tiles (at
// least 32 k-blocks), where the remainder after whole waves is split and run before the whole
// tiles.  Its fix-ups then overlap the streaming of the whole tiles; with more tokens they are
// longer (more columns per row) and their loads, queued behind the SM's own weight stream, held
// the whole tiles back (measured: up projection 197 vs 166 us at 64 tokens).
inline bool decode_stream_k(int64_t tiles, int64_t tokens, int64_t k_blocks) {
  const int64_t sms = num_sms();
  if (tiles < sms) return true;
  return tiles % sms != 0 && tokens <= 16 && k_blocks >= 32;
}

inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t a) { return (a + 255) & ~size_t(255); }
inline int elem_bytes(int dtype) { return dtype == TP_BF16 ? 2 : 4; }

bool tensor_cores_usable();       // sm_100 device present

// ----------------------------------------------------------------------------------------------
// device error word: written by bounded waits that ran out, read by tp_check_device_error
// ----------------------------------------------------------------------------------------------
enum : uint32_t {
  DEVERR_NONE = 0,
  DEVERR_WAIT_FULL = 1u << 0,      // MMA warp waited too long for a TMA stage
  DEVERR_WAIT_EMPTY = 1u << 1,     // producer waited too long for a free stage
  DEVERR_WAIT_ACC_FULL = 1u << 2,  // epilogue waited too long for an accumulator
  DEVERR_WAIT_ACC_EMPTY = 1u << 3, // MMA warp waited too long for the epilogue
  DEVERR_WAIT_DRAIN = 1u << 4,     // abort path: in-flight copies did not land in time
  DEVERR_WAIT_FLAG = 1u << 5,      // a tile waited too long for another CTA's tiles (decode MLP)
};

// Device address of the error word of the current device (owned by tp_abi.cu).  Kernels get
// it as a parameter; there is no cross-file device symbol.
uint32_t* device_error_word();

// Upper bound for a single device-side wait (nanoseconds of %globaltimer).
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_device_error(uint32_t* word, uint32_t bits) {
  if (word) atomicOr(word, bits);
}

// Acquire load of a 32-bit word at GPU scope (a counter other CTAs publish with a release).
__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *c >= need (another CTA's progress counter).  Gives up when *abort is set
// or after limit_ns; a timeout sets *abort, records site in the device error word and returns
// false.
__device__ __forceinline__ bool wait_counter_at_least(const int32_t* c, int32_t need,
                                                      volatile int* abort, uint32_t* err,
                                                      uint32_t site,
                                                      uint64_t limit_ns = kWaitTimeoutNs) {
  if (ld_acquire_gpu(c) >= need) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t n = 0;
  while (ld_acquire_gpu(c) < need) {
    if ((++n & 15u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort = 1;
        record_device_error(err, site);
        return false;
      }
    }
  }
  return true;
}

// ----------------------------------------------------------------------------------------------
// element conversions
// ----------------------------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ __forceinline__ static float load(const float* p) { return *p; }
  __device__ __forceinline__ static float to_f(float v) { return v; }
  __device__ __forceinline__ static float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  __device__ __forceinline__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// pack two floats into a bf16x2 word (low half = a)
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ----------------------------------------------------------------------------------------------
// the block's elementwise functions (CUDA's expf / erff are called, not re-derived)
// ----------------------------------------------------------------------------------------------
__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }
__device__ __forceinline__ float silu_f(float z) { return z * sigmoid_f(z); }
__device__ __forceinline__ float silu_grad_f(float z) {
  float s = sigmoid_f(z);
  return s * (1.0f + z * (1.0f - s));
}
__device__ __forceinline__ float gelu_f(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752440f));
}
__device__ __forceinline__ float gelu_grad_f(float z) {
  float cdf = 0.5f * (1.0f + erff(z * 0.70710678118654752440f));
  float pdf = 0.39894228040143267794f * expf(-0.5f * z * z);
  return cdf + z * pdf;
}
__device__ __forceinline__ float act_f(int act, float z) {
  switch (act) {
    case TP_ACT_RELU: return z > 0.f ? z : 0.f;
    case TP_ACT_GELU: return gelu_f(z);
    default: return z;
  }
}
__device__ __forceinline__ float act_grad_f(int act, float z) {
  switch (act) {
    case TP_ACT_RELU: return z > 0.f ? 1.f : 0.f;
    case TP_ACT_GELU: return gelu_grad_f(z);
    default: return 1.f;
  }
}

}  // namespace tp
