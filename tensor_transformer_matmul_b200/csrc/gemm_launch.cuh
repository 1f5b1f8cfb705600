// Host side of the tcgen05 GEMM: tensor-map encoding and kernel launch.
#pragma once

#include <cuda.h>
#include <algorithm>
#include <vector>

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

// Stream-K schedule of one GEMM: every CTA gets an equal contiguous range of the k-blocks of all
// output tiles.  Computed on the host by walking each CTA's segments exactly as the kernel does.
struct SkPlan {
  int grid = 0;             // CTAs (<= SMs, <= k-blocks)
  int slots_per_cta = 0;    // partial-tile slots per CTA
  int max_group_segs = 0;   // most segments any output tile is cut into
  int64_t units = 0;        // k-blocks over the split tiles
  int64_t groups = 0;       // output tiles
  int64_t sk_groups = 0;    // the first sk_groups tiles are split; the rest run whole
  size_t counter_bytes = 0; // arrival counters (256-aligned)
  size_t slot_bytes = 0;    // partial slots
  size_t bytes() const { return counter_bytes + slot_bytes; }
};

template <class Cfg>
SkPlan plan_stream_k(int64_t M, int64_t N, int64_t K, int64_t batch, bool sum_batch, int sms) {
  SkPlan pl;
  const int64_t mb = ceil_div(M, Cfg::A_ROWS), nb = ceil_div(N, Cfg::BN), kb = ceil_div(K, kBK);
  if (M <= 0 || N <= 0 || K <= 0 || batch <= 0) return pl;
  pl.groups = sum_batch ? mb * nb : batch * mb * nb;
  const int64_t U = sum_batch ? batch * kb : kb;
  // With at least a wave of tiles, the whole waves run as whole tiles after the split ranges and
  // only the remainder is split (plus one wave when the remainder alone would be cut into too
  // many pieces).  The fused shard sum splits every tile (each shard's k-range is a segment).
  pl.sk_groups = pl.groups;
  if (!sum_batch && pl.groups > sms) {
    const int64_t r = pl.groups % sms;
    pl.sk_groups = r == 0 ? 0 : (r * 14 >= sms) ? r : r + sms;
  }
  pl.units = pl.sk_groups * U;
  std::vector<int> per_group(static_cast<size_t>(pl.sk_groups), 0);
  // fewer, longer ranges when a tile would otherwise be cut into too many segments (tiny
  // problems spread over many SMs); with whole tiles after the split ones the grid stays at sms
  const int grid0 = pl.sk_groups < pl.groups ? sms : static_cast<int>(std::min<int64_t>(sms, pl.units));
  for (int grid = grid0; grid >= 1; grid = grid / 2) {
    std::fill(per_group.begin(), per_group.end(), 0);
    int spc = 0;
    for (int c = 0; c < grid; ++c) {
      int64_t u = static_cast<int64_t>(c) * pl.units / grid;
      const int64_t end = static_cast<int64_t>(c + 1) * pl.units / grid;
      int n = 0;
      while (u < end) {
        const int64_t g = u / U, o = u - g * U;
        const int64_t lim = sum_batch ? (o / kb + 1) * kb : U;
        const int64_t seg_end = std::min(lim, end - g * U);
        ++n;
        ++per_group[static_cast<size_t>(g)];
        u = g * U + seg_end;
      }
      spc = std::max(spc, n);
    }
    int mx = 0;
    for (int v : per_group) mx = std::max(mx, v);
    pl.grid = grid;
    pl.slots_per_cta = spc;
    pl.max_group_segs = mx;
    if (mx <= kMaxGroupSegs || grid == 1 || pl.sk_groups < pl.groups) break;
  }
  pl.counter_bytes = align256(static_cast<size_t>(pl.groups) * sizeof(int32_t));
  pl.slot_bytes = static_cast<size_t>(pl.grid) * pl.slots_per_cta * Cfg::SLOT_FLOATS * sizeof(float);
  return pl;
}

// Where a stream-K launch keeps its counters and partial slots.
struct StreamKArgs {
  bool sum_batch;     // add the problems (shards) into one output: the fused reduce
  void* ws;           // at least plan_stream_k(...).bytes(), 256-byte aligned
  size_t ws_bytes;
};

// Launch options beyond the shapes.
struct GemmOpts {
  const StreamKArgs* sk = nullptr;   // stream-K schedule (else whole tiles)
  bool rotate_k = false;             // tile-dependent k-loop start (weight streaming)
  // grouped problems (see GemmParams): device arrays of the n groups' row counts, first rows
  // and 128-row block prefix (n + 1 entries); M is then the largest group's row count
  const int32_t* grp_cnt = nullptr;
  const int32_t* grp_off = nullptr;
  const int32_t* grp_mbp = nullptr;
  int grp_n = 0;
  int grp_div = 1;
  bool grp_sum = false;   // sum each group's grp_div problems into one output (in order)
  bool grp_swap = false;  // the group ranges run along N (B rows); grp_mbp counts BN-row blocks
  // words that the kernel after this GEMM needs zeroed: cleared by the launch that zeroes the
  // stream-K counters (one kernel for both), or by a small kernel of their own
  uint32_t* zero_also = nullptr;
  int64_t zero_also_words = 0;
};

// Launch gemm_kernel<Cfg, Epi> over ``batch`` problems of D = A B^T (M x N, contraction K).
// With ``sk`` the stream-K schedule is used (and its counters are zeroed on the stream first, by
// a small kernel).  Both kernels are launched with programmatic dependent launch.
template <class Cfg, class Epi>
tp_status run_gemm(const Operand& a, const Operand& b, int64_t M, int64_t N, int64_t K,
                   int64_t batch, const typename Epi::Params& ep, cudaStream_t stream,
                   const char* label = "gemm", const GemmOpts& opts = GemmOpts(),
                   int m_fastest = -1) {
  const StreamKArgs* sk = opts.sk;
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
  gp.stream_k = 0;
  gp.sum_batch = 0;
  gp.units = 0;
  gp.sk_groups = 0;
  gp.slots_per_cta = 0;
  gp.slots = nullptr;
  gp.counters = nullptr;
  gp.rotate_k = opts.rotate_k ? 1 : 0;
  gp.grp_cnt = opts.grp_cnt;
  gp.grp_off = opts.grp_off;
  gp.grp_mbp = opts.grp_mbp;
  gp.grp_n = opts.grp_n;
  gp.grp_div = opts.grp_div > 0 ? opts.grp_div : 1;
  gp.grp_swap = opts.grp_swap ? 1 : 0;
  if (opts.grp_cnt && opts.grp_sum) gp.sum_batch = 1;
  if (opts.grp_cnt && (sk || Cfg::A_MN || !opts.grp_off || !opts.grp_mbp || opts.grp_n < 1 ||
                       batch != static_cast<int64_t>(opts.grp_n) * gp.grp_div))
    return set_error(TP_ERR_INVALID_ARG,
                     "grouped GEMM: whole tiles, K-major A, n groups x grp_div problems");
  if (opts.grp_cnt && !opts.grp_swap && Cfg::A_ROWS != 128)
    return set_error(TP_ERR_INVALID_ARG, "grouped GEMM: the groups' rows come in 128-row tiles");
  if (opts.grp_cnt && opts.grp_swap && (Cfg::BN != 128 || Cfg::B_MN))
    return set_error(TP_ERR_INVALID_ARG,
                     "swapped grouped GEMM: the groups' rows come in 128-row K-major B tiles");
  int grid_sk = 0;
  if (sk) {
    const SkPlan pl = plan_stream_k<Cfg>(M, N, K, batch, sk->sum_batch, num_sms());
    if (pl.max_group_segs > kMaxGroupSegs)
      return set_error(TP_ERR_UNSUPPORTED, "stream-K: an output tile would need too many segments");
    if (!sk->ws || sk->ws_bytes < pl.bytes())
      return set_error(TP_ERR_WORKSPACE, "stream-K workspace too small");
    gp.stream_k = 1;
    gp.sum_batch = sk->sum_batch ? 1 : 0;
    gp.units = pl.units;
    gp.sk_groups = static_cast<int32_t>(pl.sk_groups);
    gp.slots_per_cta = pl.slots_per_cta;
    gp.counters = static_cast<int32_t*>(sk->ws);
    gp.slots = reinterpret_cast<float*>(static_cast<uint8_t*>(sk->ws) + pl.counter_bytes);
    grid_sk = pl.grid;
    const int64_t words = static_cast<int64_t>(pl.counter_bytes / 4);
    const int64_t extra = opts.zero_also ? opts.zero_also_words : 0;
    TP_LAUNCH_PDL(zero_words2_kernel,
                  dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(words + extra, 256), 64))),
                  dim3(256), 0, stream, static_cast<uint32_t*>(sk->ws), words, opts.zero_also,
                  extra);
  } else if (opts.zero_also && opts.zero_also_words > 0) {
    const int64_t extra = opts.zero_also_words;
    TP_LAUNCH_PDL(zero_words_kernel,
                  dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(extra, 256), 64))),
                  dim3(256), 0, stream, opts.zero_also, extra);
  }

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
  const int grid = sk ? grid_sk : static_cast<int>(std::min<int64_t>(tiles, num_sms()));
  ProfScope prof(stream, label);
  auto* kern = gemm_kernel<Cfg, Epi>;
  TP_LAUNCH_PDL(kern, dim3(grid), dim3(kThreads), Cfg::SMEM_BYTES, stream, ta, tb, gp, ep);
  return TP_OK;
}

}  // namespace tc
}  // namespace tp
