// One-launch decode MLP (swapped tensor-core tiles, up to 64 tokens, separate shard reduce).
//
// "How does tensor parallelism split a transformer feed-forward block's two matmuls": each shard
// i computes act(x W1_i) W2_i, the column-parallel up projection followed by the row-parallel down
// projection, and the p partials are summed afterwards.  In decode both projections only stream
// their weights once, so the two GEMMs are one persistent kernel here: a single work list holds
// the up-projection tiles (activation in the epilogue, h to memory) followed by the down-
// projection tiles ordered by shard (fp32 partials, summed by the reduce kernel afterwards).
// Each CTA takes the next item from a device counter when it has issued all loads of its previous
// one, so down tiles start on the SMs that finished their up tiles first and both weight streams
// run back to back, without the wave tail of each GEMM (224 up tiles and 512 down tiles on 148
// SMs in the workload's shape).
//
// Dependency: a down tile of shard i reads h_i, written by the up tiles of shard i (h column c
// belongs to shard c / Fsp, and up tile u writes columns [128u, 128u + 128)).  After its h stores
// an up tile's epilogue threads fence, and one of them adds 1 to the shard's counter; a down
// tile's producer waits (bounded) until its shard's counter is complete, then orders its tensor
// loads of h after that acquire with a proxy fence.  Every item a CTA waits for was taken earlier,
// by a CTA that is running and whose up tiles wait for nothing, so the waits always end; a CTA
// that has not started has taken no item.
//
// Roles and pipeline as in gemm_tc.cuh (TMA producer, MMA issuer, four epilogue warps, two TMEM
// accumulators, bounded mbarrier waits).  The work items reach the MMA issuer and the epilogue
// warps through a small shared-memory queue filled by the producer.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "gemm_tc.cuh"
#include "sm100.cuh"
#include "tp_common.cuh"

namespace tp {
namespace mlpdec {

using tc::kBK;
using tc::kUmmaK;
using tc::kEpiWarps;
using tc::kThreads;

// A stage holds two 128 x 64 weight boxes and up to two token boxes: an up tile of SwiGLU loads its
// gate and up rows of one k-block, every other item two k-blocks of 128 rows, so each stage keeps
// 32 KB of weights in flight whatever the item.
template <int BN_, int UP_SUB_>
struct Cfg {
  static constexpr int BN = BN_;            // tokens per tile (N of the MMAs)
  static constexpr int UP_SUB = UP_SUB_;    // 128-row MMAs per up tile (2: SwiGLU gate + up)
  static constexpr int UP_KPACK = 2 / UP_SUB;   // k-blocks per stage of an up tile
  static constexpr int DN_KPACK = 2;            // k-blocks per stage of a down tile
  static constexpr int BOX_A = 128 * kBK * 2;   // one 128 x 64 weight box
  static constexpr int BOX_B = BN * kBK * 2;    // one BN x 64 token box
  static constexpr int A_STAGE_BYTES = 2 * BOX_A;
  static constexpr int B_STAGE_BYTES = 2 * BOX_B;
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES < 8 ? (200 * 1024) / STAGE_BYTES : 8;
  static constexpr int ACC_COLS = UP_SUB * BN;
  static constexpr int TMEM_COLS = (2 * ACC_COLS <= 32) ? 32 : (2 * ACC_COLS <= 64) ? 64
                                   : (2 * ACC_COLS <= 128) ? 128 : (2 * ACC_COLS <= 256) ? 256 : 512;
  static constexpr int QUEUE = 4;           // work items between the producer and the consumers
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5 + 2 * QUEUE) + 4 * QUEUE + 32;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr uint32_t IDESC = sm100::make_idesc_bf16(128, BN, false, false);
  // the tile configurations whose epilogues the two kinds of item reuse
  using UpTile = tc::TileCfg<BN, UP_SUB, false, false, STAGES>;
  using DownTile = tc::TileCfg<BN, 1, false, false, STAGES>;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(2 * ACC_COLS <= 512, "two accumulators must fit in TMEM");
};

struct Params {
  int32_t n_up;           // up tiles: 128 * UP_SUB packed W1 rows each, all of K = d
  int32_t up_kb;          // k-blocks of an up tile
  int32_t up_per_shard;   // up tiles per shard (Fsp / 128)
  int32_t n_dn;           // down tiles: p shards x dn_mb blocks of 128 output features
  int32_t dn_mb;          // 128-row blocks of d
  int32_t dn_kb;          // k-blocks of a down tile (Fsp / 64)
  int32_t* counters;      // [0]: items handed out after the first gridDim.x (each CTA starts at
                          // its index); [1 + i]: finished up tiles of shard i (zeroed)
  uint32_t* err;          // device error word
  tc::EpiHiddenParams up;      // h (and the saved pre-activations), swapped
  tc::EpiStoreF32::Params dn;  // fp32 partials [p][T][d], swapped
};

// orders this thread's generic-proxy accesses with its tensor (async-proxy) accesses
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

template <class C>
__global__ void __launch_bounds__(kThreads, 1)
    mlp_decode_kernel(const __grid_constant__ CUtensorMap tma_w1,
                      const __grid_constant__ CUtensorMap tma_x,
                      const __grid_constant__ CUtensorMap tma_w2,
                      const __grid_constant__ CUtensorMap tma_h, const Params pr) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + C::STAGES * C::A_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(b_smem + C::STAGES * C::B_STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint64_t* drain = acc_empty + 2;          // [1]
  uint64_t* q_full = drain + 1;             // [QUEUE]
  uint64_t* q_empty = q_full + C::QUEUE;    // [QUEUE]
  volatile int* q_item = reinterpret_cast<volatile int*>(q_empty + C::QUEUE);   // [QUEUE]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(q_item) + C::QUEUE);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = pr.n_up + pr.n_dn;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int q = 0; q < C::QUEUE; ++q) {
      mbar_init(&q_full[q], 1);
      mbar_init(&q_empty[q], 1 + kEpiWarps);   // the MMA issuer and each epilogue warp
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tma_w1);
    tma_prefetch_desc(&tma_x);
    tma_prefetch_desc(&tma_w2);
    tma_prefetch_desc(&tma_h);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above may overlap the previous kernel's tail; global memory only from here on
  // (the TMA producer waits below, after requesting its first weight tiles)
  if (threadIdx.x != 0) pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      int stage = 0, slot = 0;
      uint32_t phase = 0, qphase = 0;
      uint32_t issued_mask = 0, last_parity = 0;
      bool ok = true;
      // Item of step i of a tile: stage count, k-rotation, first k-block and k-block count.
      auto up_stage = [&](int item, int i, int& kb0, int& nkb) {
        const int nst = (pr.up_kb + C::UP_KPACK - 1) / C::UP_KPACK;
        const int rot = static_cast<int>((static_cast<int64_t>(item) * 37) % nst);
        int si = i + rot;
        if (si >= nst) si -= nst;
        kb0 = si * C::UP_KPACK;
        nkb = pr.up_kb - kb0 < C::UP_KPACK ? pr.up_kb - kb0 : C::UP_KPACK;
      };
      auto up_bytes = [&](int nkb) {
        return C::UP_SUB == 2 ? static_cast<uint32_t>(2 * C::BOX_A + C::BOX_B)
                              : static_cast<uint32_t>(nkb * (C::BOX_A + C::BOX_B));
      };
      auto load_w1 = [&](int st, int kb0, int nkb, int m0) {
        uint8_t* sa = a_smem + st * C::A_STAGE_BYTES;
        if (C::UP_SUB == 2) {
          tma_load_3d(&tma_w1, &full[st], sa, kb0 * kBK, m0, 0);   // gate and up rows: one box
        } else {
          for (int j = 0; j < nkb; ++j)
            tma_load_3d(&tma_w1, &full[st], sa + j * C::BOX_A, (kb0 + j) * kBK, m0, 0);
        }
      };
      // The first item is this CTA's index (the counter hands out the rest).  When it is an up
      // tile, its first stages of W1 -- a weight no earlier kernel writes -- are requested
      // before the programmatic-launch wait and stream while the previous kernel finishes; x
      // follows after the wait.
      const int first = static_cast<int>(blockIdx.x) < n_items ? static_cast<int>(blockIdx.x) : -1;
      int pre = 0;
      if (first >= 0 && first < pr.n_up) {
        const int nst = (pr.up_kb + C::UP_KPACK - 1) / C::UP_KPACK;
        pre = nst < C::STAGES ? nst : C::STAGES;
        for (int i = 0; i < pre; ++i) {
          int kb0, nkb;
          up_stage(first, i, kb0, nkb);
          mbar_arrive_expect_tx(&full[i], up_bytes(nkb));
          load_w1(i, kb0, nkb, first * 128 * C::UP_SUB);
          issued_mask |= 1u << i;   // phase 0
        }
      }
      pdl_wait();
      bool first_taken = false;
      while (ok) {
        int item = first;
        if (first_taken) {
          item = static_cast<int>(gridDim.x) + atomicAdd(pr.counters, 1);
          if (item >= n_items) item = -1;
        }
        first_taken = true;
        // publish the item to the MMA issuer and the epilogue warps
        if (!mbar_wait(&q_empty[slot], qphase ^ 1u, abort_flag, pr.err, DEVERR_WAIT_EMPTY)) {
          ok = false;
          break;
        }
        q_item[slot] = item;
        mbar_arrive(&q_full[slot]);
        if (++slot == C::QUEUE) {
          slot = 0;
          qphase ^= 1u;
        }
        if (item < 0) break;
        const bool up = item < pr.n_up;
        const int t = up ? item : item - pr.n_up;
        const int shard = up ? 0 : t / pr.dn_mb;
        const int m0 = up ? t * 128 * C::UP_SUB : (t - shard * pr.dn_mb) * 128;
        const int kb_all = up ? pr.up_kb : pr.dn_kb;
        const int kpack = up ? C::UP_KPACK : C::DN_KPACK;
        const int nst = (kb_all + kpack - 1) / kpack;   // stages of this item
        const int rot = static_cast<int>((static_cast<int64_t>(item) * 37) % nst);
        if (!up) {
          // h of this shard must be complete before its tensor loads
          if (!wait_counter_at_least(pr.counters + 1 + shard, pr.up_per_shard, abort_flag,
                                     pr.err, DEVERR_WAIT_FLAG)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();
        }
        for (int i = 0; i < nst; ++i) {
          int si = i + rot;
          if (si >= nst) si -= nst;
          const int kb0 = si * kpack;
          const int nkb = kb_all - kb0 < kpack ? kb_all - kb0 : kpack;
          uint8_t* sb = b_smem + stage * C::B_STAGE_BYTES;
          if (pre > 0) {
            --pre;   // this stage's W1 tile and byte count went out before the wait
          } else {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, pr.err, DEVERR_WAIT_EMPTY)) {
              ok = false;
              break;
            }
            if (up) {
              mbar_arrive_expect_tx(&full[stage], up_bytes(nkb));
              load_w1(stage, kb0, nkb, m0);
            } else {
              uint8_t* sa = a_smem + stage * C::A_STAGE_BYTES;
              mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(nkb * (C::BOX_A + C::BOX_B)));
              for (int j = 0; j < nkb; ++j)
                tma_load_3d(&tma_w2, &full[stage], sa + j * C::BOX_A, (kb0 + j) * kBK, m0, shard);
            }
          }
          if (up) {
            // x: one box per k-block of the stage
            if (C::UP_SUB == 2) {
              tma_load_3d(&tma_x, &full[stage], sb, kb0 * kBK, 0, 0);
            } else {
              for (int j = 0; j < nkb; ++j)
                tma_load_3d(&tma_x, &full[stage], sb + j * C::BOX_B, (kb0 + j) * kBK, 0, 0);
            }
          } else {
            for (int j = 0; j < nkb; ++j)
              tma_load_3d(&tma_h, &full[stage], sb + j * C::BOX_B, (kb0 + j) * kBK, 0, shard);
          }
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let every copy already issued land before the CTA can exit
        for (int s = 0; s < C::STAGES; ++s)
          if (issued_mask & (1u << s)) tc::drain_wait(&full[s], (last_parity >> s) & 1u, pr.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      int stage = 0, slot = 0, it_n = 0;
      uint32_t phase = 0, qphase = 0;
      bool ok = true, issued_any = false;
      while (ok) {
        if (!mbar_wait(&q_full[slot], qphase, abort_flag, pr.err, DEVERR_WAIT_FULL)) {
          ok = false;
          break;
        }
        const int item = q_item[slot];
        mbar_arrive(&q_empty[slot]);
        if (++slot == C::QUEUE) {
          slot = 0;
          qphase ^= 1u;
        }
        if (item < 0) break;
        const bool up = item < pr.n_up;
        const int kb_all = up ? pr.up_kb : pr.dn_kb;
        const int kpack = up ? C::UP_KPACK : C::DN_KPACK;
        const int nst = (kb_all + kpack - 1) / kpack;
        const int rot = static_cast<int>((static_cast<int64_t>(item) * 37) % nst);
        const int acc = it_n & 1;
        const uint32_t acc_phase = (it_n >> 1) & 1;
        ++it_n;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, pr.err,
                       DEVERR_WAIT_ACC_EMPTY)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_base = tmem_base + acc * C::ACC_COLS;
        for (int i = 0; i < nst; ++i) {
          if (!mbar_wait(&full[stage], phase, abort_flag, pr.err, DEVERR_WAIT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(a_smem + stage * C::A_STAGE_BYTES);
          const uint32_t b_addr = smem_addr(b_smem + stage * C::B_STAGE_BYTES);
          int si = i + rot;
          if (si >= nst) si -= nst;
          const int kb0 = si * kpack;
          const int nkb = kb_all - kb0 < kpack ? kb_all - kb0 : kpack;
          if (up && C::UP_SUB == 2) {
            // gate rows accumulate in columns [0, BN), up rows in [BN, 2 BN)
#pragma unroll
            for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
              const uint64_t bdesc = make_sdesc_sw128(b_addr + kk * (kUmmaK * 2), 16, 1024);
#pragma unroll
              for (int s = 0; s < 2; ++s) {
                const uint64_t adesc =
                    make_sdesc_sw128(a_addr + s * C::BOX_A + kk * (kUmmaK * 2), 16, 1024);
                umma_f16(d_base + s * C::BN, adesc, bdesc, C::IDESC, (i > 0 || kk != 0) ? 1u : 0u);
              }
            }
          } else {
            for (int j = 0; j < nkb; ++j) {
#pragma unroll
              for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                const uint64_t bdesc =
                    make_sdesc_sw128(b_addr + j * C::BOX_B + kk * (kUmmaK * 2), 16, 1024);
                const uint64_t adesc =
                    make_sdesc_sw128(a_addr + j * C::BOX_A + kk * (kUmmaK * 2), 16, 1024);
                umma_f16(d_base, adesc, bdesc, C::IDESC, (i > 0 || j > 0 || kk != 0) ? 1u : 0u);
              }
            }
          }
          issued_any = true;
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
      }
      if (!ok && issued_any) {
        // every MMA issued so far must finish before TMEM is released
        umma_commit(drain);
        tc::drain_wait(drain, 0, pr.err);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    int slot = 0, it_n = 0;
    uint32_t qphase = 0;
    const tc::GemmParams no_gp = {};
    while (true) {
      int item = -1, ok = 0;
      if (lane == 0) {
        ok = mbar_wait(&q_full[slot], qphase, abort_flag, pr.err, DEVERR_WAIT_ACC_FULL);
        if (ok) {
          item = q_item[slot];
          mbar_arrive(&q_empty[slot]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      item = __shfl_sync(0xffffffffu, item, 0);
      if (!tc::epi_bar_and(ok)) break;
      if (++slot == C::QUEUE) {
        slot = 0;
        qphase ^= 1u;
      }
      if (item < 0) break;
      const bool up = item < pr.n_up;
      const int t = up ? item : item - pr.n_up;
      const int acc = it_n & 1;
      const uint32_t acc_phase = (it_n >> 1) & 1;
      ++it_n;
      ok = 0;
      if (lane == 0)
        ok = mbar_wait(&acc_full[acc], acc_phase, abort_flag, pr.err, DEVERR_WAIT_ACC_FULL);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!tc::epi_bar_and(ok)) break;
      tc_fence_after();
      tc::TmemSrc tsrc;
      tsrc.taddr = tmem_base + acc * C::ACC_COLS + (static_cast<uint32_t>(quarter * 32) << 16);
      tc::EpiCtx ctx;
      ctx.row = row;
      ctx.n0 = 0;
      if (up) {
        ctx.b = 0;
        ctx.m0 = t * 128 * C::UP_SUB;
        tc::EpiHiddenSwap::template run<typename C::UpTile>(pr.up, no_gp, ctx, tsrc);
      } else {
        const int shard = t / pr.dn_mb;
        ctx.b = shard;
        ctx.m0 = (t - shard * pr.dn_mb) * 128;
        tc::EpiStoreF32::template run<typename C::DownTile>(pr.dn, no_gp, ctx, tsrc);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (up) {
        // h of this tile is stored: publish it to the down tiles of its shard
        fence_proxy_async_global();
        __threadfence();
        tc::epi_bar();
        if (threadIdx.x == 64) atomicAdd(pr.counters + 1 + t / pr.up_per_shard, 1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace mlpdec
}  // namespace tp
