// Host side of the tcgen05 GEMM: tensor-map encoding and kernel launch.
#pragma once

#include <cuda.h>
#include <algorithm>

#include "gemm_tc.cuh"
#include "tp_common.cuh"

namespace tp {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
tp_status encode_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t batch, uint64_t outer_stride_bytes,
                              uint64_t batch_stride_bytes, uint32_t box_inner, uint32_t box_outer);

namespace tc {

// One GEMM operand as the kernel sees it: a bf16 tensor [batch][rows][cols] (row-major, strides
// in elements) whose MN and K dimensions are either (rows = MN, cols = K) -- K-major -- or
// (rows = K, cols = MN) -- MN-major.
struct Operand {
  const void* ptr;
  bool mn_major;
  int64_t mn_ext;       // extent of the M (or N) dimension
  int64_t k_ext;        // extent of K
  int64_t batch;        // 1 when shared by all problems
  int64_t row_stride;   // elements between consecutive rows
  int64_t batch_stride; // elements between problems
};

inline tp_status encode_operand(CUtensorMap* map, const Operand& o, int tile_mn) {
  if (reinterpret_cast<uintptr_t>(o.ptr) % 16 != 0)
    return set_error(TP_ERR_INVALID_ARG, "tensor-core operand not 16-byte aligned");
  const uint64_t rs = static_cast<uint64_t>(o.row_stride) * 2;
  const uint64_t bs = o.batch > 1 ? static_cast<uint64_t>(o.batch_stride) * 2
                                  : rs * static_cast<uint64_t>(o.mn_major ? o.k_ext : o.mn_ext);
  if (!o.mn_major)
    return encode_tmap_bf16_3d(map, o.ptr, o.k_ext, o.mn_ext, o.batch, rs, bs, 64,
                               static_cast<uint32_t>(tile_mn));
  return encode_tmap_bf16_3d(map, o.ptr, o.mn_ext, o.k_ext, o.batch, rs, bs, 64, 64);
}

// Launch gemm_kernel<Cfg, Epi> over ``batch`` problems of D = A B^T (M x N, contraction K).
template <class Cfg, class Epi>
tp_status run_gemm(const Operand& a, const Operand& b, int64_t M, int64_t N, int64_t K,
                   int64_t batch, const typename Epi::Params& ep, cudaStream_t stream,
                   const char* label = "gemm", int m_fastest = -1) {
  static_assert(Cfg::A_MN == false || Cfg::A_ROWS % 64 == 0, "A tile");
  if (a.mn_major != Cfg::A_MN || b.mn_major != Cfg::B_MN)
    return set_error(TP_ERR_INVALID_ARG, "operand major does not match the tile config");
  if (M <= 0 || N <= 0 || batch <= 0) return TP_OK;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
    return set_error(TP_ERR_UNSUPPORTED, "GEMM extent above 2^31");
  CUtensorMap ta, tb;
  tp_status st = encode_operand(&ta, a, Cfg::A_ROWS);
  if (st != TP_OK) return st;
  st = encode_operand(&tb, b, Cfg::BN);
  if (st != TP_OK) return st;

  GemmParams gp;
  gp.M = static_cast<int32_t>(M);
  gp.N = static_cast<int32_t>(N);
  gp.K = static_cast<int32_t>(K);
  gp.batch = static_cast<int32_t>(batch);
  gp.m_blocks = static_cast<int32_t>(ceil_div(M, Cfg::A_ROWS));
  gp.n_blocks = static_cast<int32_t>(ceil_div(N, Cfg::BN));
  gp.k_blocks = static_cast<int32_t>(ceil_div(K, kBK));
  gp.m_fastest = m_fastest >= 0 ? m_fastest : (gp.m_blocks <= gp.n_blocks ? 1 : 0);
  gp.a_batched = a.batch > 1 ? 1 : 0;
  gp.b_batched = b.batch > 1 ? 1 : 0;
  gp.err = device_error_word();
  if (gp.k_blocks == 0) return set_error(TP_ERR_INVALID_ARG, "GEMM with K == 0");

  static int attr_set[64] = {0};
  int dev = 0;
  TP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 64 && !attr_set[dev]) {
    TP_CUDA_TRY(cudaFuncSetAttribute(gemm_kernel<Cfg, Epi>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Cfg::SMEM_BYTES));
    attr_set[dev] = 1;
  }
  const int64_t tiles = static_cast<int64_t>(gp.batch) * gp.m_blocks * gp.n_blocks;
  const int grid = static_cast<int>(std::min<int64_t>(tiles, num_sms()));
  ProfScope prof(stream, label);
  gemm_kernel<Cfg, Epi><<<grid, kThreads, Cfg::SMEM_BYTES, stream>>>(ta, tb, gp, ep);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace tc
}  // namespace tp
