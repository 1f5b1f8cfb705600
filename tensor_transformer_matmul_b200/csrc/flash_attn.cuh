// Prefill attention on the tensor cores (sm_100a): each CTA computes one 128-row query tile of
// one query head, attending over its KV head with an online softmax ("Tensor Parallelism"
// (klaylearn), Notes: attention is computed locally over the shard's heads; the same page names
// FlashAttention's tiling of QK, softmax and V as the way to cut its HBM traffic).
//
//   S  = Q K_b^T                (tcgen05.mma, Q and K K-major in smem, S fp32 in TMEM)
//   m' = max(m, rowmax(S)),  P = exp(S - m') (bf16),
//   l  = l * exp(m - m') + rowsum(P),  O = O * exp(m - m')  (O fp32 in TMEM; m is only moved when
//        the row maximum grew by more than 2^8, so the rescale is rare)
//   O += P V_b                  (tcgen05.mma, V read MN-major straight from its [key][dim] tile)
//   out = O / l
//
// 128 threads, thread t owning query row t of the tile (TMEM lane t).  Thread 0 also issues the
// TMA loads and the MMAs.  Key blocks are 128 keys, so every MMA is 128 x 128.  S and P share 128
// TMEM columns (the bf16 P of a block is written over its S and read from there as the A operand
// of P V, so P never touches shared memory) and O takes the other 128.  Thread 0 issues
// S(kb+1) = Q K(kb+1)^T right behind P(kb) V(kb): the MMAs of a CTA run in issue order, so S(kb+1)
// overwrites P(kb) only after P(kb) V(kb) has read it, and S(kb+1) done means P(kb) V(kb) is done
// too.  Q, K and V each have one shared-memory buffer: K(kb+1) is fetched as soon as S(kb) is
// done, V(kb+1) as soon as S(kb+1) is, each well ahead of its use.  A CTA needs 96 KB of shared
// memory and 256 TMEM columns, so two CTAs share an SM and one's softmax runs while the other's
// MMAs do.
//
// The special-function unit computes 16 exponentials per clock per SM, which for this tile shape
// is as slow as the tensor core, so three pairs of P values in eight are computed on the FMA pipe:
// 2^x = 2^n * 2^f with n = round(x), f in [-1/2, 1/2], 2^f by a degree-3 polynomial (minimax fit
// for relative error, max error 7.5e-5, below bf16's rounding of P), and n added to the exponent.
// All waits are bounded; a timeout sets the abort flag, drains what was issued and leaves.
#pragma once

#include <cuda.h>

#include "gemm_launch.cuh"
#include "sm100.cuh"
#include "tp_common.cuh"

namespace tp {
namespace fa {

constexpr int kRows = 128;   // query rows per tile
constexpr int kKeys = 128;   // keys per K/V block
constexpr int kThreads = 128;

template <int HD>
struct Smem {
  static constexpr int SUB = HD / 64;                 // 64-wide swizzle sub-tiles along the head dim
  static constexpr int TILE = 128 * 128;              // one sub-tile: 128 rows x 128 bytes
  static constexpr int BLOCK = SUB * TILE;            // Q tile, or one K or V block
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + BLOCK;
  static constexpr int V_OFF = K_OFF + BLOCK;
  static constexpr int BAR_OFF = V_OFF + BLOCK;
  static constexpr int BYTES = BAR_OFF + 128 + 1024;  // barriers + alignment slack
  static constexpr uint32_t TMEM_COLS = 256;          // S/P at column 0, O at column 128
};

constexpr float kRescaleLog2 = 8.f;   // growth of a row maximum (log2 units) that forces a rescale
// 2^f ~= kP0 + f (kP1 + f (kP2 + f kP3)) on [-1/2, 1/2]
constexpr float kP0 = 0.9999281168f, kP1 = 0.6932609677f, kP2 = 0.2426105440f, kP3 = 0.0551713221f;
constexpr float kRoundMagic = 12582912.f;   // 1.5 * 2^23: x + magic has round(x) in its low bits
// pairs of P values (index mod 8) computed on the FMA pipe; the rest use the special-function unit.
// Three of eight balances the two when two warps share a sub-partition: a pair costs 16 cycles
// of the 4-lane-per-clock unit, or about twice the issue slots on the FMA pipe.
constexpr uint32_t kPolyPairs = (1u << 1) | (1u << 4) | (1u << 6);

struct Params {
  int32_t s;          // tokens per sequence
  int32_t n_q, qh, kh, hd, group;   // heads: total Q, per shard Q, per shard KV, dim, n_q/n_kv
  int32_t R_a;        // packed qkv columns per shard
  int32_t n_qt;       // query tiles per sequence
  int32_t causal;
  float scale_log2;   // log2(e) / sqrt(hd)
  __nv_bfloat16* o;   // [b*s][n_q*hd]
  float* lse;         // optional [b*s][n_q]: log2 of each row's softmax denominator (scaled units)
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
// 2^x with the special-function unit (PTX ex2.approx.ftz.f32: results below 2^-126 flush to 0,
// 2^-inf = 0); a softmax term that small does not change the sum.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Packed pairs of fp32 (PTX .f32x2 arithmetic, sm_100): one instruction for two lanes of work.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint64_t fsub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// (2^x0, 2^x1) on the FMA pipe; inputs below -125 (masked keys at -inf included) give about
// 2^-125, which no softmax sum notices.
__device__ __forceinline__ void exp2_poly_x2(float x0, float x1, float& y0, float& y1) {
  const uint64_t x = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t magic = f2_pack(kRoundMagic, kRoundMagic);
  const uint64_t j = fadd2(x, magic);
  const uint64_t f = fsub2(x, fsub2(j, magic));
  uint64_t q = ffma2(f2_pack(kP3, kP3), f, f2_pack(kP2, kP2));
  q = ffma2(q, f, f2_pack(kP1, kP1));
  q = ffma2(q, f, f2_pack(kP0, kP0));
  float j0, j1, q0, q1;
  f2_unpack(j, j0, j1);
  f2_unpack(q, q0, q1);
  y0 = __uint_as_float(__float_as_uint(q0) + __float_as_uint(j0) * (1u << 23));
  y1 = __uint_as_float(__float_as_uint(q1) + __float_as_uint(j1) * (1u << 23));
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16: A (M x 16, K-major) sits in TMEM, row i in lane i,
// two bf16 per 32-bit column (lower k in the low half).  Issued by a single thread.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
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
  uint64_t* k_full = bar + 1;    // K block landed (one phase per block)
  uint64_t* v_full = bar + 2;    // V block landed
  uint64_t* s_full = bar + 3;    // S = Q K^T done
  uint64_t* p_full = bar + 4;    // P stored in TMEM and O rescaled (128 arrivals)
  uint64_t* pv_done = bar + 5;   // O += P V done: S/P columns and the V buffer are free again
  uint64_t* drain = bar + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 7);
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
  const int nkb = P.causal ? min(qt + 1, n_kb_all) : n_kb_all;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(k_full, 1);
    mbar_init(v_full, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, kThreads);
    mbar_init(pv_done, 1);
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
  // everything above may overlap the previous kernel's tail; global memory only from here on
  pdl_wait();
  pdl_trigger();
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  uint8_t* sQ = smem + L::Q_OFF;
  uint8_t* sK = smem + L::K_OFF;
  uint8_t* sV = smem + L::V_OFF;
  auto wait = [&](uint64_t* b, uint32_t par, uint32_t site) {
    return mbar_wait(b, par, abort_flag, P.err, site);
  };

  // ---- thread 0: loads and MMAs
  uint32_t n_k = 0, n_v = 0;    // K / V loads issued (thread 0)
  bool issued_mma = false;
  auto load_block = [&](uint64_t* full, uint8_t* dst, int col, int row) {
    mbar_arrive_expect_tx(full, L::BLOCK);
#pragma unroll
    for (int c = 0; c < L::SUB; ++c) tma_load_3d(&tma_qkv, full, dst + c * L::TILE, col + 64 * c, row, bi);
  };
  auto issue_s = [&]() {
    constexpr uint32_t IDESC_S = make_idesc_bf16(128, kKeys, false, false);
    tc_fence_after();
    const uint32_t qa = smem_addr(sQ), ka = smem_addr(sK);
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const uint32_t off = (kk >> 2) * L::TILE + (kk & 3) * 32;
      umma_f16(tS, make_sdesc_sw128(qa + off, 16, 1024), make_sdesc_sw128(ka + off, 16, 1024),
               IDESC_S, kk > 0 ? 1u : 0u);
    }
    umma_commit(s_full);
    issued_mma = true;
  };
  auto issue_pv = [&](int kb) {
    constexpr uint32_t IDESC_O = make_idesc_bf16(128, HD, false, true);
    tc_fence_after();
    const uint32_t va = smem_addr(sV);
#pragma unroll
    for (int kk = 0; kk < kKeys / 16; ++kk) {
      // P: 16 keys = 8 TMEM columns; V: 64-dim blocks of 128 key rows (LBO = one sub-tile)
      umma_f16_tmem_a(tO, tS + kk * 8, make_sdesc_sw128(va + kk * 16 * 128, L::TILE, 1024),
                      IDESC_O, (kb > 0 || kk > 0) ? 1u : 0u);
    }
    umma_commit(pv_done);
  };

  bool ok = true;
  if (tid == 0) {
    load_block(q_full, sQ, q_col, q0);
    load_block(k_full, sK, k_col, 0);
    ++n_k;
    load_block(v_full, sV, v_col, 0);
    ++n_v;
    if (wait(q_full, 0, DEVERR_WAIT_FULL) && wait(k_full, 0, DEVERR_WAIT_FULL)) issue_s();
  }

  // ---- softmax: every thread one row; wait results are made warp-uniform (the TMEM loads and
  // stores are warp-collective)
  const int q_abs = q0 + tid;
  float m_run = -INFINITY, l_run = 0.f;
  for (int kb = 0; kb < nkb; ++kb) {
    const uint32_t par = kb & 1;
    // S(kb) done: the MMAs run in issue order, so P(kb-1) V(kb-1) is done too and O is final
    // for a rescale
    ok = __all_sync(0xffffffffu, wait(s_full, par, DEVERR_WAIT_ACC_FULL));
    if (!ok) break;
    tc_fence_after();
    if (tid == 0) {
      if (kb + 1 < nkb) {   // the K buffer is free once S(kb) is done
        load_block(k_full, sK, k_col, (kb + 1) * kKeys);
        ++n_k;
      }
      if (kb > 0) {         // and the V buffer once P(kb-1) V(kb-1) is
        load_block(v_full, sV, v_col, kb * kKeys);
        ++n_v;
      }
    }
    float sv[kKeys];
    {
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tS + lane_base + c * 32, r[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(r[c][e]);
    }
    const int k_base = kb * kKeys;
    if ((k_base + kKeys > P.s) || (P.causal && k_base + kKeys - 1 > q0)) {
      // keys of this row inside the block: beyond the sequence or the causal limit -> -inf
      const int lim = (P.causal ? min(P.s, q_abs + 1) : P.s) - k_base;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) sv[c] = c < lim ? sv[c] : -INFINITY;
    }
    float mx;
    {   // row maximum: 8 partial maxima, two new keys per three-input max
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = sv[i];
#pragma unroll
      for (int c = 8; c < kKeys; c += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmax3(m8[i], sv[c + i], sv[c + 8 + i]);
      mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
    }
    // The reference maximum m moves only on the first block or when the block's maximum
    // exceeds it by more than 2^8 in the exp2 domain, so O and l are rarely rescaled; P then
    // stays below 2^8 and O / l is the same whichever m was used.
    float alpha = 1.f;
    if (m_run == -INFINITY || (mx - m_run) * P.scale_log2 > kRescaleLog2) {
      alpha = (m_run == -INFINITY) ? 0.f : exp2f((m_run - mx) * P.scale_log2);
      m_run = mx;
    }
    const float mscaled = (m_run == -INFINITY) ? 0.f : m_run * P.scale_log2;
    uint32_t pk[kKeys / 2];
    float rs;
    {   // P = 2^(s*scale - m) two keys at a time; row sum in 4 packed partial sums
      const uint64_t scale2 = f2_pack(P.scale_log2, P.scale_log2);
      const uint64_t negm2 = f2_pack(-mscaled, -mscaled);
      uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int c = 0; c < kKeys / 2; ++c) {
        float x0, x1, p0, p1;
        f2_unpack(ffma2(f2_pack(sv[2 * c], sv[2 * c + 1]), scale2, negm2), x0, x1);
        if (kPolyPairs & (1u << (c & 7))) {
          exp2_poly_x2(x0, x1, p0, p1);
        } else {
          p0 = ex2_approx(x0);   // 2^-inf = 0 for masked keys
          p1 = ex2_approx(x1);
        }
        acc[c & 3] = fadd2(acc[c & 3], f2_pack(p0, p1));
        pk[c] = pack_bf16x2(p0, p1);
      }
      const uint64_t a2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      float a, bb;
      f2_unpack(a2, a, bb);
      rs = a + bb;
    }
    l_run = l_run * alpha + rs;
    // P(kb) as bf16 over the first half of the S columns
    tmem_st_32x32b_x32(tS + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
    tmem_st_32x32b_x32(tS + lane_base + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
    if (kb > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tO + lane_base + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
        tmem_st_32x32b_x32(tO + lane_base + c * 32, r);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(p_full);
    if (tid == 0) {
      // every row has stored P(kb) and rescaled O: O += P(kb) V(kb), and right behind it S(kb+1),
      // which overwrites P(kb) only after P(kb) V(kb) has read it (issue order)
      bool t = wait(p_full, par, DEVERR_WAIT_ACC_FULL) && wait(v_full, par, DEVERR_WAIT_FULL);
      if (t) issue_pv(kb);
      if (t && kb + 1 < nkb && wait(k_full, (kb + 1) & 1, DEVERR_WAIT_FULL)) issue_s();
    }
  }
  tmem_wait_st();
  if (ok) ok = __all_sync(0xffffffffu, wait(pv_done, (nkb - 1) & 1, DEVERR_WAIT_ACC_EMPTY));
  if (ok) {
    tc_fence_after();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    // p = 2^(s * scale_log2 - lse) reproduces the softmax (used by the backward pass)
    if (P.lse && q_abs < P.s)
      P.lse[(static_cast<int64_t>(bi) * P.s + q_abs) * P.n_q + j] =
          (m_run == -INFINITY ? 0.f : m_run * P.scale_log2) + log2f(l_run);
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
  }
  __syncthreads();
  if (*abort_flag && tid == 0) {
    // let issued copies and MMAs land before the CTA leaves (bounded waits); each buffer has at
    // most its latest load in flight
    const uint64_t t0 = globaltimer_ns();
    auto bounded = [&](uint64_t* bb, uint32_t pp) {
      while (!mbar_try_wait(bb, pp))
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
          record_device_error(P.err, DEVERR_WAIT_DRAIN);
          return;
        }
    };
    bounded(q_full, 0);
    if (n_k) bounded(k_full, (n_k - 1) & 1);
    if (n_v) bounded(v_full, (n_v - 1) & 1);
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
                        int64_t R_a, int p, int causal, void* o, cudaStream_t st,
                        float* lse = nullptr) {
  using L = Smem<HD>;
  CUtensorMap map;
  const uint64_t cols = static_cast<uint64_t>(p) * R_a;
  tp_status r = encode_tmap_bf16_3d(&map, qkv, cols, static_cast<uint64_t>(s),
                                    static_cast<uint64_t>(b), cols * 2,
                                    cols * 2 * static_cast<uint64_t>(s), 64, 128);
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
  P.lse = lse;
  P.err = device_error_word();
  dim3 grid(static_cast<unsigned>(n_q), static_cast<unsigned>(P.n_qt), static_cast<unsigned>(b));
  ProfScope prof(st, "attn_prefill");
  TP_LAUNCH_PDL(flash_fwd_kernel<HD>, grid, dim3(kThreads), static_cast<size_t>(L::BYTES), st,
                map, P);
  return TP_OK;
}

}  // namespace fa
}  // namespace tp
