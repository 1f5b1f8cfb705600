// Two-CTA (cta_group::2) tcgen05 GEMM for the large, compute-bound shard GEMMs.
//
//   D[b][m][n] = sum_k A_b(m, k) * B_b(n, k)      (bf16 operands, fp32 accumulator in TMEM)
//
// A cluster of two CTAs on a pair of SMs computes one 256 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256).  CTA r (its rank in the cluster) keeps rows
// 128 r .. 128 r + 127 of the tile's A block and rows 128 r .. 128 r + 127 of its B block in its
// own shared memory; its TMEM receives the accumulator rows of its own A rows, all 256 columns.
// Per SM this is the MMA work of a one-CTA 128 x 256 tile with half of that tile's B traffic:
// the shared-memory bytes written by TMA and read by the tensor core per MMA fall by a third,
// and that traffic is what holds the one-CTA tile below the tensor peak.
//
// Roles (192 threads per CTA, as in the one-CTA kernel of gemm_tc.cuh):
//   warp 0 lane 0, both CTAs -- TMA producer of the CTA's own halves.  The copies signal CTA 0's
//                               "full" barrier (the .cta_group::2 form of the tensor copy), on
//                               which CTA 0 alone announces the byte count of both halves.
//   warp 1 lane 0, CTA 0     -- MMA issuer.  One multicast tcgen05.commit hands a consumed
//                               stage back to both producers, another a finished accumulator to
//                               both epilogues.
//   warps 2..5, both CTAs    -- epilogue of the CTA's 128 accumulator rows; each warp returns
//                               the accumulator by arriving on CTA 0's "acc_empty" barrier.
// Whole tiles only (no stream-K): cluster c takes tiles c, c + C, c + 2C, ... of the
// batch x M x N tile space.  With sum_batch the problems (shards) are summed into one output:
// the tile space is M x N and each tile's k loop runs over the k-blocks of problem 0, then of
// problem 1, ... into the same TMEM accumulator -- the partial-sum reduce, shard by shard in
// order, done in the accumulator.  No copy is multicast: every CTA loads only its own halves.
//
// Every wait is bounded as in the one-CTA kernel.  Both CTAs meet at a cluster barrier before
// TMEM is released and before either exits, so neither CTA's shared memory goes away while the
// other may still signal it.
#pragma once

#include "gemm_launch.cuh"

namespace tp {
namespace tc {

// Compile-time configuration of the pair tile (per CTA: 128 A rows, 128 B rows per stage).
template <bool A_MN_, bool B_MN_, int STAGES_>
struct PairCfg {
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_MN = B_MN_;
  static constexpr int STAGES = STAGES_;
  static constexpr int TILE = 256;                 // output tile is TILE x TILE
  static constexpr int HALF = 128;                 // rows of A and of B held by each CTA
  static constexpr int A_STAGE_BYTES = HALF * kBK * 2;
  static constexpr int B_STAGE_BYTES = HALF * kBK * 2;
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr int ACC_COLS = TILE;            // accumulator columns in each CTA's TMEM
  static constexpr int TMEM_COLS = 2 * ACC_COLS;   // two accumulators
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5) + 32;
  static constexpr int BAR_SPAN = (BAR_BYTES + 127) / 128 * 128;
  static constexpr int EPI_STAGE_FLOATS = 32 * 32;   // per epilogue warp: 32 rows x 32 fp32
  static constexpr int EPI_STAGE_BYTES = 4 * EPI_STAGE_FLOATS * 4;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_SPAN + EPI_STAGE_BYTES;
  static constexpr uint32_t IDESC = sm100::make_idesc_bf16(2 * HALF, TILE, A_MN, B_MN);
  // what the epilogues see: a 128-row x 256-column accumulator, as a one-CTA 128 x 256 tile
  static constexpr int BN = TILE;
  static constexpr int A_SUB = 1;
  static constexpr int A_ROWS = HALF;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Tiles of at most this many k-blocks store fp32 accumulators through the staging tiles.
constexpr int kStageMaxKBlocks = 48;

namespace pair {

// arrive on an mbarrier given by its shared::cluster address (possibly in the peer CTA)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   bar_cluster_addr)
               : "memory");
}
// 3-D tiled load into this CTA's shared memory whose completion bytes go to an mbarrier in
// either CTA of the pair (given by its shared::cluster address).
__device__ __forceinline__ void tma_load_3d_pair(const CUtensorMap* map, uint32_t bar_cluster_addr,
                                                 void* dst, int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(sm100::smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// TMEM allocation shared by the pair: the same warp of both CTAs executes it.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   sm100::smem_addr(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]^T, issued by one thread of CTA 0.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this shared offset in every CTA of ``mask`` when all MMAs issued
// so far by this thread have completed.
__device__ __forceinline__ void umma_commit_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(sm100::smem_addr(bar)),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          sm100::smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void decode_tile(int t, const GemmParams& gp, int& b, int& mb, int& nb) {
  if (gp.sum_batch) {
    b = 0;
    decode_mn(t, gp, mb, nb);
    return;
  }
  const int per = gp.m_blocks * gp.n_blocks;
  b = t / per;
  decode_mn(t - b * per, gp, mb, nb);
}
// k-blocks of one tile: all problems' with sum_batch
__device__ __forceinline__ int tile_k_blocks(const GemmParams& gp) {
  return gp.sum_batch ? gp.batch * gp.k_blocks : gp.k_blocks;
}

}  // namespace pair

template <class Cfg, class Epi>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tma_a,
                     const __grid_constant__ CUtensorMap tma_b, const GemmParams gp,
                     const typename Epi::Params ep) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + Cfg::STAGES * Cfg::A_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(b_smem + Cfg::STAGES * Cfg::B_STAGE_BYTES);
  uint64_t* empty = full + Cfg::STAGES;
  uint64_t* acc_full = empty + Cfg::STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2], used in CTA 0
  uint64_t* drain = acc_empty + 2;           // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // the epilogue warps' staging tiles, after the barriers: used when a tile's k loop is short
  // (the epilogue's stores then bound the kernel); with a long k loop the epilogue is hidden
  // behind the next tile's MMAs and its direct stores measured faster
  float* epi_stage = pair::tile_k_blocks(gp) <= kStageMaxKBlocks
                         ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + Cfg::BAR_SPAN)
                         : nullptr;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int cluster = static_cast<int>(blockIdx.x >> 1);
  const int nclusters = static_cast<int>(gridDim.x >> 1);
  const int tiles = (gp.sum_batch ? 1 : gp.batch) * gp.m_blocks * gp.n_blocks;
  const int nk = pair::tile_k_blocks(gp);

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full[s], 1);    // CTA 0's producer announces both halves' bytes
      mbar_init(&empty[s], 1);   // one multicast commit per consumed stage
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * kEpiWarps);   // the epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tma_a);
    tma_prefetch_desc(&tma_b);
  }
  if (warp == 1) {
    pair::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    pair::tmem_relinquish();
  }
  // barrier initialisation and the TMEM address are visible to both CTAs from here on
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0;
      uint32_t last_parity = 0;
      bool ok = true;
      const uint32_t full0 = map_to_rank(smem_addr(full), 0);
      for (int t = cluster; ok && t < tiles; t += nclusters) {
        int b, mb, nb;
        pair::decode_tile(t, gp, b, mb, nb);
        const int m0 = mb * Cfg::TILE + Cfg::HALF * static_cast<int>(rank);
        const int n0 = nb * Cfg::TILE + Cfg::HALF * static_cast<int>(rank);
        int bu = b, kb = 0;   // problem and k-block of step u
        for (int u = 0; u < nk; ++u, ++kb) {
          if (kb == gp.k_blocks) {   // sum_batch: on to the next problem's k-blocks
            kb = 0;
            ++bu;
          }
          const int za = gp.a_batched ? bu : 0;
          const int zb = gp.b_batched ? bu : 0;
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, gp.err, DEVERR_WAIT_EMPTY)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * Cfg::STAGE_BYTES);
          const uint32_t fb = full0 + static_cast<uint32_t>(stage) * 8u;
          const int k0 = kb * kBK;
          uint8_t* sa = a_smem + stage * Cfg::A_STAGE_BYTES;
          uint8_t* sb = b_smem + stage * Cfg::B_STAGE_BYTES;
          if (Cfg::A_MN) {
#pragma unroll
            for (int j = 0; j < Cfg::HALF / 64; ++j)
              pair::tma_load_3d_pair(&tma_a, fb, sa + j * 64 * kBK * 2, m0 + 64 * j, k0, za);
          } else {
            pair::tma_load_3d_pair(&tma_a, fb, sa, k0, m0, za);
          }
          if (Cfg::B_MN) {
#pragma unroll
            for (int j = 0; j < Cfg::HALF / 64; ++j)
              pair::tma_load_3d_pair(&tma_b, fb, sb + j * 64 * kBK * 2, n0 + 64 * j, k0, zb);
          } else {
            pair::tma_load_3d_pair(&tma_b, fb, sb, k0, n0, zb);
          }
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (ok) {
        // the MMA's last releases of this CTA's stages must land before the CTA can exit
        for (int s = 0; s < Cfg::STAGES; ++s)
          if (issued_mask & (1u << s))
            if (!mbar_wait(&empty[s], (last_parity >> s) & 1u, abort_flag, gp.err,
                           DEVERR_WAIT_EMPTY))
              break;
      } else if (rank == 0) {
        // copies of both CTAs signal CTA 0's barriers: let every announced phase land
        for (int s = 0; s < Cfg::STAGES; ++s)
          if (issued_mask & (1u << s)) drain_wait(&full[s], (last_parity >> s) & 1u, gp.err);
      } else {
        // this CTA's copies signal CTA 0: give the ones in flight time to land
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------------ MMA issuer (CTA 0)
      int stage = 0;
      uint32_t phase = 0;
      int it_n = 0;
      bool ok = true;
      bool issued_any = false;
      for (int t = cluster; ok && t < tiles; t += nclusters) {
        const int acc = it_n & 1;
        const uint32_t acc_phase = (it_n >> 1) & 1;
        ++it_n;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, gp.err,
                       DEVERR_WAIT_ACC_EMPTY)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * Cfg::ACC_COLS;
        for (int u = 0; u < nk; ++u) {
          if (!mbar_wait(&full[stage], phase, abort_flag, gp.err, DEVERR_WAIT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(a_smem + stage * Cfg::A_STAGE_BYTES);
          const uint32_t b_addr = smem_addr(b_smem + stage * Cfg::B_STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t adesc =
                Cfg::A_MN ? make_sdesc_sw128(a_addr + kk * (kUmmaK * 128), 64 * kBK * 2, 1024)
                          : make_sdesc_sw128(a_addr + kk * (kUmmaK * 2), 16, 1024);
            const uint64_t bdesc =
                Cfg::B_MN ? make_sdesc_sw128(b_addr + kk * (kUmmaK * 128), 64 * kBK * 2, 1024)
                          : make_sdesc_sw128(b_addr + kk * (kUmmaK * 2), 16, 1024);
            pair::umma_f16(d_tmem, adesc, bdesc, Cfg::IDESC, (u > 0 || kk != 0) ? 1u : 0u);
          }
          issued_any = true;
          pair::umma_commit_mc(&empty[stage], 0x3);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        pair::umma_commit_mc(&acc_full[acc], 0x3);
      }
      if (ok) {
        // both epilogues' last hand-backs land on this CTA's barriers before it can exit
        const int uses[2] = {(it_n + 1) >> 1, it_n >> 1};
        for (int a = 0; a < 2; ++a)
          if (uses[a] > 0 &&
              !mbar_wait(&acc_empty[a], static_cast<uint32_t>(uses[a] - 1) & 1u, abort_flag,
                         gp.err, DEVERR_WAIT_ACC_EMPTY))
            break;
      } else if (issued_any) {
        pair::umma_commit(drain);
        drain_wait(drain, 0, gp.err);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int quarter = warp & 3;   // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t acc_empty0 = map_to_rank(smem_addr(acc_empty), 0);
    int it_n = 0;
    for (int t = cluster; t < tiles; t += nclusters) {
      const int acc = it_n & 1;
      const uint32_t acc_phase = (it_n >> 1) & 1;
      ++it_n;
      int ok = 0;
      if (lane == 0)
        ok = mbar_wait(&acc_full[acc], acc_phase, abort_flag, gp.err, DEVERR_WAIT_ACC_FULL);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!epi_bar_and(ok)) break;
      tc_fence_after();
      int b, mb, nb;
      pair::decode_tile(t, gp, b, mb, nb);
      TmemSrc tsrc;
      tsrc.taddr = tmem_base + acc * Cfg::ACC_COLS + (static_cast<uint32_t>(quarter * 32) << 16);
      EpiCtx ctx;
      ctx.row = row;
      ctx.b = b;
      ctx.m0 = mb * Cfg::TILE + Cfg::HALF * static_cast<int>(rank);
      ctx.n0 = nb * Cfg::TILE;
      ctx.stage = epi_stage ? epi_stage + quarter * Cfg::EPI_STAGE_FLOATS : nullptr;
      Epi::template run<Cfg>(ep, gp, ctx, tsrc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair::mbar_arrive_cluster(acc_empty0 + static_cast<uint32_t>(acc) * 8u);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    pair::tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// Clusters of two that can be resident at once for this kernel (cached per device).
template <class Cfg, class Epi>
tp_status pair_clusters(int* out) {
  static int cached[64] = {0};
  int dev = 0;
  TP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 64 && cached[dev] > 0) {
    *out = cached[dev];
    return TP_OK;
  }
  auto* kern = gemm_pair_kernel<Cfg, Epi>;
  TP_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   Cfg::SMEM_BYTES));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  TP_CUDA_TRY(cudaOccupancyMaxActiveClusters(&n, kern, &cfg));
  if (n < 1) return set_error(TP_ERR_UNSUPPORTED, "no cluster of two CTAs fits on this device");
  if (dev < 64) cached[dev] = n;
  *out = n;
  return TP_OK;
}

// Launch gemm_pair_kernel<Cfg, Epi> over ``batch`` problems of D = A B^T (M x N, contraction K):
// one cluster of two CTAs per resident pair of SMs, persistent over the 256 x 256 tiles, with
// programmatic dependent launch.
template <class Cfg, class Epi>
tp_status run_gemm_pair(const Operand& a, const Operand& b, int64_t M, int64_t N, int64_t K,
                        int64_t batch, const typename Epi::Params& ep, cudaStream_t stream,
                        const char* label = "gemm", int m_fastest = -1,
                        bool sum_batch = false) {
  if (a.mn_major != Cfg::A_MN || b.mn_major != Cfg::B_MN)
    return set_error(TP_ERR_INVALID_ARG, "operand major does not match the tile config");
  if (M <= 0 || N <= 0 || batch <= 0) return TP_OK;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
    return set_error(TP_ERR_UNSUPPORTED, "GEMM extent above 2^31");
  CUtensorMap ta, tb;
  tp_status st = encode_operand(&ta, a, Cfg::HALF);
  if (st != TP_OK) return st;
  st = encode_operand(&tb, b, Cfg::HALF);
  if (st != TP_OK) return st;

  GemmParams gp = {};
  gp.M = static_cast<int32_t>(M);
  gp.N = static_cast<int32_t>(N);
  gp.K = static_cast<int32_t>(K);
  gp.batch = static_cast<int32_t>(batch);
  gp.m_blocks = static_cast<int32_t>(ceil_div(M, Cfg::TILE));
  gp.n_blocks = static_cast<int32_t>(ceil_div(N, Cfg::TILE));
  gp.k_blocks = static_cast<int32_t>(ceil_div(K, kBK));
  gp.m_fastest = m_fastest >= 0 ? m_fastest : (gp.m_blocks <= gp.n_blocks ? 1 : 0);
  gp.a_batched = a.batch > 1 ? 1 : 0;
  gp.b_batched = b.batch > 1 ? 1 : 0;
  gp.err = device_error_word();
  gp.sum_batch = sum_batch ? 1 : 0;
  if (gp.k_blocks == 0) return set_error(TP_ERR_INVALID_ARG, "GEMM with K == 0");
  const int64_t tiles = static_cast<int64_t>(sum_batch ? 1 : gp.batch) * gp.m_blocks * gp.n_blocks;
  if (tiles > INT32_MAX || static_cast<int64_t>(gp.batch) * gp.k_blocks > INT32_MAX)
    return set_error(TP_ERR_UNSUPPORTED, "too many output tiles");

  int resident = 0;
  st = pair_clusters<Cfg, Epi>(&resident);
  if (st != TP_OK) return st;
  const int clusters = static_cast<int>(std::min<int64_t>(tiles, resident));

  ProfScope prof(stream, label);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel<Cfg, Epi>, ta, tb, gp, ep);
  if (e != cudaSuccess)
    return set_error(TP_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
  count_launch();
  return TP_OK;
}

}  // namespace tc
}  // namespace tp
