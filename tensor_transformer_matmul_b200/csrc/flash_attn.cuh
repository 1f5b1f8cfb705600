// Prefill attention on the tensor cores (sm_100a): each CTA computes one 128-row query tile of
// one query head, attending over its KV head with an online softmax ("Tensor Parallelism"
// (klaylearn), Notes: attention is computed locally over the shard's heads; the same page names
// FlashAttention's tiling of QK, softmax and V as the way to cut its HBM traffic).
//
//   S  = Q K_b^T                (tcgen05.mma, Q and K K-major in smem, S fp32 in TMEM)
//   m' = max(m, rowmax(S)),  P = exp(S - m') (bf16, written to smem in the UMMA K-major layout),
//   l  = l * exp(m - m') + rowsum(P),  O = O * exp(m - m')  (O fp32 in TMEM, rescaled only when
//        some row's maximum moved)
//   O += P V_b                  (tcgen05.mma, V read MN-major straight from its [key][dim] tile)
//   out = O / l
//
// 128 threads: thread t owns query row t of the tile (TMEM lane t).  Thread 0 also issues the TMA
// loads and the MMAs.  K/V blocks of 64 keys are double buffered; with head_dim 128 the bf16 P of
// a block is written over that block's K tile (K is dead once S is computed), which keeps a CTA
// under 100 KB of shared memory so two CTAs share an SM and one's softmax overlaps the other's
// MMAs.  All waits are bounded.
#pragma once

#include <cuda.h>

#include "gemm_launch.cuh"
#include "sm100.cuh"
#include "tp_common.cuh"

namespace tp {
namespace fa {

constexpr int kRows = 128;   // query rows per tile
constexpr int kKeys = 64;    // keys per K/V block
constexpr int kThreads = 128;

template <int HD>
struct Smem {
  static constexpr int SUB = HD / 64;                 // 64-wide swizzle sub-tiles along the head dim
  static constexpr int QTILE = kRows * 128;           // Q sub-tile: 128 rows x 128 bytes
  static constexpr int KTILE = kKeys * 128;           // K or V sub-tile: 64 rows x 128 bytes
  static constexpr int PTILE = kRows * 128;           // P: 128 rows x 64 keys (bf16)
  static constexpr bool P_IN_K = SUB * KTILE >= PTILE;   // P reuses the block's K buffer
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + SUB * QTILE;   // 2 buffers
  static constexpr int V_OFF = K_OFF + 2 * SUB * KTILE;
  static constexpr int P_OFF = V_OFF + 2 * SUB * KTILE;   // used only when !P_IN_K
  static constexpr int BAR_OFF = P_OFF + (P_IN_K ? 0 : PTILE);
  static constexpr int BYTES = BAR_OFF + 128 + 1024;  // barriers + alignment slack
  static constexpr int KV_BYTES = 2 * SUB * KTILE;    // one K block + one V block
  static constexpr uint32_t TMEM_COLS = 256;          // S (64 cols) + O (from col 128)
};

struct Params {
  int32_t s;          // tokens per sequence
  int32_t n_q, qh, kh, hd, group;   // heads: total Q, per shard Q, per shard KV, dim, n_q/n_kv
  int32_t R_a;        // packed qkv columns per shard
  int32_t n_qt;       // query tiles per sequence
  int32_t causal;
  float scale_log2;   // log2(e) / sqrt(hd)
  __nv_bfloat16* o;   // [b*s][n_q*hd]
  uint32_t* err;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 2)
    flash_fwd_kernel(const __grid_constant__ CUtensorMap tma_qkv, const Params P) {
  using namespace sm100;
  using L = Smem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bar + 0;
  uint64_t* kv_full = bar + 1;   // [2]
  uint64_t* s_done = bar + 3;
  uint64_t* o_done = bar + 4;
  uint64_t* drain = bar + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int j = blockIdx.x;                          // query head
  const int qt = P.n_qt - 1 - static_cast<int>(blockIdx.y);   // heaviest causal tiles first
  const int bi = blockIdx.z;
  const int shard = j / P.qh, jl = j - shard * P.qh;
  const int g = j / P.group;                         // KV head (global)
  const int gl = g - shard * P.kh;
  const int q_col = shard * P.R_a + jl * HD;
  const int k_col = shard * P.R_a + (P.qh + gl) * HD;
  const int v_col = shard * P.R_a + (P.qh + P.kh + gl) * HD;
  const int q0 = qt * kRows;
  const int n_kb_all = (P.s + kKeys - 1) / kKeys;
  const int nkb = P.causal ? min((q0 + kRows) / kKeys, n_kb_all) : n_kb_all;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(&kv_full[0], 1);
    mbar_init(&kv_full[1], 1);
    mbar_init(s_done, 1);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tma_qkv);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  uint8_t* sQ = smem + L::Q_OFF;
  uint8_t* sK = smem + L::K_OFF;
  uint8_t* sV = smem + L::V_OFF;

  auto load_kv = [&](int kb) {
    const int buf = kb & 1;
    mbar_arrive_expect_tx(&kv_full[buf], L::KV_BYTES);
#pragma unroll
    for (int c = 0; c < L::SUB; ++c) {
      tma_load_3d(&tma_qkv, &kv_full[buf], sK + (buf * L::SUB + c) * L::KTILE, k_col + 64 * c,
                  kb * kKeys, bi);
      tma_load_3d(&tma_qkv, &kv_full[buf], sV + (buf * L::SUB + c) * L::KTILE, v_col + 64 * c,
                  kb * kKeys, bi);
    }
  };

  uint32_t issued_kv = 0;       // blocks whose loads were issued (thread 0 only)
  if (tid == 0) {
    mbar_arrive_expect_tx(q_full, L::SUB * L::QTILE);
#pragma unroll
    for (int c = 0; c < L::SUB; ++c) {   // a Q sub-tile is two 64-row boxes
      tma_load_3d(&tma_qkv, q_full, sQ + c * L::QTILE, q_col + 64 * c, q0, bi);
      tma_load_3d(&tma_qkv, q_full, sQ + c * L::QTILE + L::KTILE, q_col + 64 * c, q0 + 64, bi);
    }
    load_kv(0);
    issued_kv = 1;
    if (nkb > 1) {
      load_kv(1);
      issued_kv = 2;
    }
  }

  // instruction descriptors: S = Q K^T (both K-major); O += P V (P K-major, V MN-major)
  constexpr uint32_t IDESC_S = make_idesc_bf16(128, kKeys, false, false);
  constexpr uint32_t IDESC_O = make_idesc_bf16(128, HD, false, true);

  const int row = tid;                 // query row within the tile
  const int q_abs = q0 + row;
  float m_run = -INFINITY, l_run = 0.f;
  bool issued_mma = false;
  // every wait result is made warp-uniform (the TMEM loads are warp-collective) and, once per
  // key block, CTA-uniform, so on a timeout all threads leave the loop together
  bool ok = __syncthreads_and(mbar_wait(q_full, 0, abort_flag, P.err, DEVERR_WAIT_FULL) ? 1 : 0);

  for (int kb = 0; kb < nkb && ok; ++kb) {
    const int buf = kb & 1;
    bool w = __all_sync(0xffffffffu,
                        mbar_wait(&kv_full[buf], (kb >> 1) & 1, abort_flag, P.err, DEVERR_WAIT_FULL));
    if (w && tid == 0) {
      tc_fence_after();
      const uint32_t qa = smem_addr(sQ), ka = smem_addr(sK + buf * L::SUB * L::KTILE);
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t koff = (kk & 3) * 32;
        umma_f16(tS, make_sdesc_sw128(qa + (kk >> 2) * L::QTILE + koff, 16, 1024),
                 make_sdesc_sw128(ka + (kk >> 2) * L::KTILE + koff, 16, 1024), IDESC_S,
                 kk > 0 ? 1u : 0u);
      }
      umma_commit(s_done);
      issued_mma = true;
    }
    if (w) w = __all_sync(0xffffffffu, mbar_wait(s_done, kb & 1, abort_flag, P.err,
                                                   DEVERR_WAIT_ACC_FULL));
    float sv[kKeys];
    if (w) {
      tc_fence_after();
      // ---- online softmax on this thread's row of S
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tS + lane_base + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(r[e]);
      }
      const int k_base = kb * kKeys;
      const bool need_mask = (k_base + kKeys > P.s) || (P.causal && k_base + kKeys - 1 > q0);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        if (need_mask) {
          const int k_abs = k_base + c;
          if (k_abs >= P.s || (P.causal && k_abs > q_abs)) sv[c] = -INFINITY;
        }
        mx = fmaxf(mx, sv[c]);
      }
      const float m_new = fmaxf(m_run, mx);
      const float alpha = (m_run == -INFINITY) ? 0.f : exp2f((m_run - m_new) * P.scale_log2);
      const float mscaled = (m_new == -INFINITY) ? 0.f : m_new * P.scale_log2;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        const float pv = exp2f(sv[c] * P.scale_log2 - mscaled);   // exp2(-inf) = 0 when masked
        sv[c] = pv;
        rs += pv;
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;

      // ---- the previous P V must be finished before P and O are touched again
      if (kb > 0) {
        w = __all_sync(0xffffffffu, mbar_wait(o_done, (kb - 1) & 1, abort_flag, P.err,
                                              DEVERR_WAIT_ACC_EMPTY));
        if (w) {
          tc_fence_after();
          if (tid == 0 && kb + 1 < nkb) {
            load_kv(kb + 1);   // buffer (kb+1)&1 held block kb-1, whose MMAs are complete
            issued_kv = kb + 2;
          }
          // rescale O only in warps where some row's maximum moved
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
              uint32_t r[32];
              tmem_ld_32x32b_x32(tO + lane_base + c * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              tmem_st_32x32b_x32(tO + lane_base + c * 32, r);
            }
            tmem_wait_st();
          }
        }
      }
    }
    // P of this block: over its K tile (dead after S) or in its own buffer
    uint8_t* sP = L::P_IN_K ? sK + buf * L::SUB * L::KTILE : smem + L::P_OFF;
    if (w) {
      // ---- P (bf16) into smem, K-major with the 128-byte swizzle: row `row`, 64 keys
#pragma unroll
      for (int ch = 0; ch < kKeys / 8; ++ch) {
        uint4 v4;
        v4.x = pack_bf16x2(sv[ch * 8 + 0], sv[ch * 8 + 1]);
        v4.y = pack_bf16x2(sv[ch * 8 + 2], sv[ch * 8 + 3]);
        v4.z = pack_bf16x2(sv[ch * 8 + 4], sv[ch * 8 + 5]);
        v4.w = pack_bf16x2(sv[ch * 8 + 6], sv[ch * 8 + 7]);
        *reinterpret_cast<uint4*>(sP + row * 128 + ((ch ^ (row & 7)) << 4)) = v4;
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    if (!__syncthreads_and(w ? 1 : 0)) {
      ok = false;
      break;
    }
    if (tid == 0) {
      tc_fence_after();
      const uint32_t pa = smem_addr(sP), va = smem_addr(sV + buf * L::SUB * L::KTILE);
#pragma unroll
      for (int kk = 0; kk < kKeys / 16; ++kk) {
        const uint64_t adesc = make_sdesc_sw128(pa + kk * 32, 16, 1024);
        // V tile: 64-dim blocks of 64 key rows (LBO = one sub-tile), 16 keys per MMA
        const uint64_t bdesc = make_sdesc_sw128(va + kk * 16 * 128, L::KTILE, 1024);
        umma_f16(tO, adesc, bdesc, IDESC_O, (kb > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(o_done);
    }
  }

  if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (nkb - 1) & 1, abort_flag, P.err,
                                                 DEVERR_WAIT_ACC_EMPTY));
  if (ok) {
    tc_fence_after();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    const bool live = q_abs < P.s;
    __nv_bfloat16* dst = P.o + (static_cast<int64_t>(bi) * P.s + q_abs) * (P.n_q * HD) + j * HD;
#pragma unroll
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tO + lane_base + c * 32, r);
      tmem_wait_ld();
      if (live) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(r[8 * qd + 0]) * inv, __uint_as_float(r[8 * qd + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(r[8 * qd + 2]) * inv, __uint_as_float(r[8 * qd + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(r[8 * qd + 4]) * inv, __uint_as_float(r[8 * qd + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(r[8 * qd + 6]) * inv, __uint_as_float(r[8 * qd + 7]) * inv);
          d4[qd] = w;
        }
      }
    }
  } else if (tid == 0) {
    // abort path: let issued copies and MMAs land before the CTA leaves (bounded waits)
    const uint64_t t0 = globaltimer_ns();
    auto bounded = [&](uint64_t* b, uint32_t par) {
      while (!mbar_try_wait(b, par))
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
          record_device_error(P.err, DEVERR_WAIT_DRAIN);
          return;
        }
    };
    bounded(q_full, 0);
    // only the most recent load into each buffer can still be in flight
    for (uint32_t kb = issued_kv >= 2 ? issued_kv - 2 : 0; kb < issued_kv; ++kb)
      bounded(&kv_full[kb & 1], (kb >> 1) & 1);
    if (issued_mma) {
      umma_commit(drain);
      bounded(drain, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

// Host launcher: qkv [b][s][p*R_a] bf16 (packed per shard: Q heads, K heads, V heads), o out.
template <int HD>
inline tp_status launch(const void* qkv, int64_t b, int64_t s, int n_q, int qh, int kh, int group,
                        int64_t R_a, int p, int causal, void* o, cudaStream_t st) {
  using L = Smem<HD>;
  CUtensorMap map;
  const uint64_t cols = static_cast<uint64_t>(p) * R_a;
  tp_status r = encode_tmap_bf16_3d(&map, qkv, cols, static_cast<uint64_t>(s),
                                    static_cast<uint64_t>(b), cols * 2,
                                    cols * 2 * static_cast<uint64_t>(s), 64, kKeys);
  if (r != TP_OK) return r;
  static int attr_set[64] = {0};
  int dev = 0;
  TP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 64 && !attr_set[dev]) {
    TP_CUDA_TRY(cudaFuncSetAttribute(flash_fwd_kernel<HD>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES));
    attr_set[dev] = 1;
  }
  Params P;
  P.s = static_cast<int32_t>(s);
  P.n_q = n_q; P.qh = qh; P.kh = kh; P.hd = HD; P.group = group;
  P.R_a = static_cast<int32_t>(R_a);
  P.n_qt = static_cast<int32_t>(ceil_div(s, kRows));
  P.causal = causal;
  P.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
  P.o = static_cast<__nv_bfloat16*>(o);
  P.err = device_error_word();
  dim3 grid(static_cast<unsigned>(n_q), static_cast<unsigned>(P.n_qt), static_cast<unsigned>(b));
  ProfScope prof(st, "attn_prefill");
  flash_fwd_kernel<HD><<<grid, kThreads, L::BYTES, st>>>(map, P);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace fa
}  // namespace tp
