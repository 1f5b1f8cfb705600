// tp_mlp_fwd_static_ws: the MLP forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: for example a plug-in running inside a host application
// that owns all device memory and hands its plug-ins no allocator, or a latency-critical loop in
// which an allocation (which may synchronize the device) is not allowed.  This entry point gives
// them tp_mlp_fwd without a caller-provided workspace: its scratch lives in a fixed array in the
// library's own device memory, so the caller passes only inputs and outputs.
//
// Costs and rules:
//   * Every GPU that loads the library holds kStaticWsBytes (32 MiB) of device memory for this
//     array until the process exits.
//   * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
//     once per device, with that device current).  Make that first call before any stream
//     capture.
//   * All calls share the one array.  Calls that overlap on the GPU (on different streams, or
//     from different host threads without ordering) race on it; callers must serialise them.
//   * The array keeps whatever the last call left in it.  Nothing needs clearing: every byte of
//     scratch this call reads is written by this call first.
//   * A problem whose workspace (tp_mlp_fwd_workspace) exceeds kStaticWsBytes is rejected with
//     TP_ERR_WORKSPACE before anything is enqueued.
//   * Nothing here allocates: no cudaMalloc, cudaFree or allocating library routine.
#include <mutex>
#include <string>

#include "tp_common.cuh"

namespace {

constexpr size_t kStaticWsBytes = TP_MLP_STATIC_WS_BYTES;  // 32 MiB
static_assert(TP_MLP_STATIC_WS_BYTES == (size_t(32) << 20), "header and library agree");

// File-scope device scratch.  In host code this name is only a host-side stand-in; kernels get
// the device address obtained by cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_mu;
void* g_ws_addr[64] = {nullptr};

tp_status static_ws_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return tp::set_error(TP_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return tp::set_error(TP_ERR_UNSUPPORTED, "device index above 63");
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_ws_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess || !p)
      return tp::set_error(TP_ERR_CUDA, std::string("cudaGetSymbolAddress(static scratch): ") +
                                            cudaGetErrorString(e));
    g_ws_addr[dev] = p;
  }
  *out = g_ws_addr[dev];
  return TP_OK;
}

}  // namespace

extern "C" tp_status tp_mlp_fwd_static_ws(const tp_mlp_desc* desc, const void* x,
                                          const void* w1p, const void* w2p,
                                          const void* residual, void* y, void* stream) {
  tp::clear_error();
  if (!desc) return tp::set_error(TP_ERR_INVALID_ARG, "desc is null");
  const size_t need = tp_mlp_fwd_workspace(desc);
  if (need == 0) {
    // an invalid shape (reported by tp_mlp_fwd) or an empty batch (T = 0, nothing to compute):
    // neither touches scratch
    return tp_mlp_fwd(desc, x, w1p, w2p, residual, y, nullptr, nullptr, nullptr, 0, stream);
  }
  if (need > kStaticWsBytes)
    return tp::set_error(TP_ERR_WORKSPACE,
                         "tp_mlp_fwd_static_ws: this shape needs " + std::to_string(need) +
                             " bytes of scratch; the static scratch holds " +
                             std::to_string(kStaticWsBytes) + " bytes (use tp_mlp_fwd)");
  void* ws = nullptr;
  tp_status st = static_ws_address(&ws);
  if (st != TP_OK) return st;
  return tp_mlp_fwd(desc, x, w1p, w2p, residual, y, nullptr, nullptr, ws, kStaticWsBytes, stream);
}
