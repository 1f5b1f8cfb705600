// Attention backward on the tensor cores (sm_100a), head_dim 64 or 128, bf16.
//
//   With P = softmax(S), S = Q K^T / sqrt(hd) (causal mask), O = P V, the row log-sum-exp of
//   the forward and D = rowsum(dO * O):
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  dK = dS^T Q / sqrt(hd),  dQ = dS K / sqrt(hd)
//   ("Tensor Parallelism" (klaylearn), Notes: attention is local to the shard's heads, so each
//   shard differentiates its own heads; a KV head collects dK and dV from every query head of
//   its group.)
//
// Two kernels, neither with atomics (each output tile is summed by one CTA in a fixed order):
//   * dK/dV: one CTA per (128-key block, KV head, query head of its group, sequence).  It walks
//     the 64-query blocks that see its keys; per step S^T = K Q^T and dP^T = V dO^T land in one
//     of two TMEM buffers, the 256 compute threads (one key row and one half of the 64 queries
//     each) turn them into P^T and dS^T, written back as bf16 over their own TMEM columns, and
//     dV += P^T dO, dK += dS^T Q accumulate in TMEM with P^T and dS^T as the TMEM A operands
//     (dO and Q read MN-major).  A ninth warp issues the MMAs and loads, so the next step's
//     S^T/dP^T are ready while the threads work on this one; Q and dO stream through a ring of
//     four 64-row slots.  The per-head shares are added afterwards.
//   * dQ: one CTA per (128-query block, query head, sequence).  It walks the key blocks its
//     queries see; per step S = Q K^T and dP = dO V^T land in TMEM, the threads (one query row
//     and one half of the 128 keys each) write dS back over S, and dQ += dS K accumulates in
//     TMEM (K read MN-major).  K and V are double buffered.
// In the dQ kernel thread 0 issues the TMA loads and the MMAs; TMEM holds three 128-column fp32
// tiles.  The next step's S/dP MMAs are issued right behind this step's dQ MMAs: the MMAs run
// in issue order, so they overwrite dS only after it has been read, and their completion also
// means the previous step's MMAs are done.  The dK/dV kernel's issuing warp uses the same
// order, two steps ahead: step it's dV/dK MMAs, then step it+2's S^T/dP^T into the buffer they
// have just read.
// The two thread halves (warps 0-3 and 4-7) read the same TMEM lanes and split a step's columns
// in two; half h packs its bf16 results into the first half of its own columns, which only it
// reads, so the halves need no ordering between them.
// Every wait is bounded; a timeout sets the abort flag, drains what was issued and leaves, and
// the loop exit is CTA-uniform.
#pragma once

#include <cuda.h>

#include "flash_attn.cuh"
#include "gemm_launch.cuh"
#include "sm100.cuh"
#include "tp_common.cuh"

namespace tp {
namespace fb {

constexpr int kBlk = 128;       // query rows and key rows per block
constexpr int kThreads = 256;   // two threads per row: each takes half of the block's columns

// TMEM column (from the tile's start) of the packed bf16 pair holding columns 2i and 2i+1 of a
// 128-column block: half h = i / 32 of the threads writes its 32 packed columns at 64 h
__device__ __forceinline__ uint32_t packed_col(int i) {
  return static_cast<uint32_t>(i + (i >> 5) * 32);
}

// 2^x with the MUFU approximation (flushes subnormal results to zero); the probabilities it
// feeds are rounded to bf16 right after
__device__ __forceinline__ float exp2_fast(float x) { return fa::ex2_approx(x); }

struct Params {
  int32_t s;                    // tokens per sequence
  int32_t n_q, qh, kh, group;   // heads: total Q, per shard Q, per shard KV, n_q / n_kv
  int32_t R_a;                  // packed qkv columns per shard
  int32_t n_blk;                // 128-row blocks per sequence
  int32_t causal;
  int64_t ld;                   // qkv and dqkv row length (p * R_a)
  float scale_log2, scale;      // log2(e) / sqrt(hd), 1 / sqrt(hd)
  const float* lse;             // [b*s][n_q], log2 units of the scaled scores
  const float* D;               // [b*s][n_q]
  __nv_bfloat16* dqkv;
  float* part_kv;               // split > 1: fp32 partial dK, dV [split][b*s][n_kv][2][hd]
  int32_t split;                // CTAs sharing one key block's query heads
  uint32_t* err;
};

template <int HD>
struct Tiles {
  static constexpr int SUB = HD / 64;           // 64-column swizzle sub-tiles along the head dim
  static constexpr int TILE = kBlk * 128;       // one sub-tile: 128 rows x 128 bytes
  static constexpr int BLOCK = SUB * TILE;      // one 128-row head tile
};

__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  sm100::tmem_ld_32x32b_x32(taddr, r);
  sm100::tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]);
}

// 32 bf16 values (16 words) of this lane's row into TMEM columns taddr .. taddr+15
__device__ __forceinline__ void st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]),
      "r"(w[15])
      : "memory");
}

// bounded drain of what thread 0 issued, on the abort path
struct Drain {
  uint64_t t0;
  uint32_t* err;
  __device__ void operator()(uint64_t* bar, uint32_t par) const {
    while (!sm100::mbar_try_wait(bar, par))
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
        record_device_error(err, DEVERR_WAIT_DRAIN);
        return;
      }
  }
};

// ================================================================================ dK and dV
// Steps of 64 queries.  S^T/dP^T have two TMEM buffers of 64 + 64 columns next to dV and dK
// (128 each), so the MMAs of step it+1 are already done while the 256 compute threads turn step
// it into P^T/dS^T.  A ninth warp issues: when all 256 threads have stored step it's P^T/dS^T
// (an mbarrier of 256 arrivals) its elected thread issues step it's dV/dK MMAs and then step
// it+2's S^T/dP^T into the same buffer (issue order keeps the overwrite behind the reads), so
// the compute threads never wait for the issue.  Q and dO stream through a ring of kRing 64-row
// slots, loaded three steps ahead.
constexpr int kQStep = 64;   // queries per step of the dK/dV kernel (keys per step of dQ)
constexpr int kRing = 4;     // 64-row Q/dO (K/V) slots
constexpr int kThreadsIssue = kThreads + 32;   // compute threads plus the issuing warp
constexpr int kIssuer = kThreads;              // the issuing thread

// barrier 1 over the 256 compute threads (the issuing warp does not take part), returning the
// AND of v over them
__device__ __forceinline__ int compute_bar_and(int v) {
  int out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\tselp.s32 %0, 1, 0, q;\n\t}\n"
      : "=r"(out)
      : "r"(v), "n"(kThreads)
      : "memory");
  return out;
}

template <int HD>
struct Tiles64 {
  static constexpr int TILE = kQStep * 128;           // one 64-row, 128-byte-wide sub-tile
  static constexpr int BLOCK = Tiles<HD>::SUB * TILE; // one 64-row head tile
};

// TMEM column, from a 64-column buffer's start, of the packed bf16 pairs that the k-th
// 16-row MMA step reads: half h of the threads packs its 32 rows into columns 32 h .. 32 h + 15
__device__ __forceinline__ uint32_t packed_col64(int kk) {
  return static_cast<uint32_t>(32 * (kk >> 1) + 8 * (kk & 1));
}

template <int HD>
__global__ void __launch_bounds__(kThreadsIssue, 1)
    flash_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tma_qkv,
                         const __grid_constant__ CUtensorMap tma_q64,
                         const __grid_constant__ CUtensorMap tma_do64, const Params P) {
  using namespace sm100;
  using L = Tiles<HD>;
  using Q = Tiles64<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + L::BLOCK;
  uint8_t* sQ = sV + L::BLOCK;            // [kRing] slots
  uint8_t* sDO = sQ + kRing * Q::BLOCK;   // [kRing] slots
  float* lse_s = reinterpret_cast<float*>(sDO + kRing * Q::BLOCK);   // [2][kQStep]
  float* D_s = lse_s + 2 * kQStep;                                     // [2][kQStep]
  uint64_t* bar = reinterpret_cast<uint64_t*>(D_s + 2 * kQStep);
  uint64_t* kv_full = bar + 0;
  uint64_t* qd_full = bar + 1;            // [kRing]
  uint64_t* s_full = qd_full + kRing;     // [2]
  uint64_t* m_done = s_full + 2;          // [2]
  uint64_t* p_ready = m_done + 2;         // [2]: the 256 threads' P^T/dS^T of a step stored
  uint64_t* drain = p_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int kb = blockIdx.x, bi = blockIdx.z;
  const int g = blockIdx.y / P.split, sp = blockIdx.y - g * P.split;   // KV head, head slice
  const int heads = P.group / P.split, a0 = sp * heads;                 // query heads of this CTA
  const int shard = g / P.kh, gl = g - shard * P.kh;
  const int k_col = shard * P.R_a + (P.qh + gl) * HD;
  const int v_col = shard * P.R_a + (P.qh + P.kh + gl) * HD;
  const int k0 = kb * kBlk;
  const int n64 = (P.s + kQStep - 1) / kQStep;
  const int qb0 = P.causal ? k0 / kQStep : 0;   // first 64-query block that sees these keys
  const int nqb = n64 - qb0;
  const int n_iter = heads * nqb;

  if (tid == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < kRing; ++i) mbar_init(&qd_full[i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&m_done[i], 1);
      mbar_init(&p_ready[i], kThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tma_qkv);
    tma_prefetch_desc(&tma_q64);
    tma_prefetch_desc(&tma_do64);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // buffer b: S^T at 128 b, dP^T at 128 b + 64; dV at 256, dK at 384
  const uint32_t tdV = tmem + 256, tdK = tmem + 384;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const int row = tid & (kBlk - 1);
  const int half = tid >> 7;   // queries 32 half .. 32 half + 31 of a step
  const int k_abs = k0 + row;
  auto wait = [&](uint64_t* b, uint32_t par, uint32_t site) {
    return mbar_wait(b, par, abort_flag, P.err, site);
  };
  constexpr uint32_t IDESC_S = make_idesc_bf16(128, kQStep, false, false);   // S^T, dP^T
  constexpr uint32_t IDESC_KN = make_idesc_bf16(128, HD, false, true);       // dV, dK

  // step it -> (query head, 64-query block)
  auto head_of = [&](int it) { return g * P.group + a0 + it / nqb; };
  auto block_of = [&](int it) { return qb0 + it % nqb; };
  uint32_t nq[kRing] = {0, 0, 0, 0};   // Q/dO loads issued per slot (issuing thread)
  bool any_mma = false;
  auto load_qd = [&](int it) {
    const int r = it % kRing, j = head_of(it), jl = j - shard * P.qh;
    const int q_col = shard * P.R_a + jl * HD, q0 = block_of(it) * kQStep;
    mbar_arrive_expect_tx(&qd_full[r], 2 * Q::BLOCK);
#pragma unroll
    for (int c = 0; c < L::SUB; ++c) {
      tma_load_3d(&tma_q64, &qd_full[r], sQ + r * Q::BLOCK + c * Q::TILE, q_col + 64 * c, q0, bi);
      tma_load_3d(&tma_do64, &qd_full[r], sDO + r * Q::BLOCK + c * Q::TILE, j * HD + 64 * c, q0,
                  bi);
    }
    ++nq[r];
  };
  // S^T = K Q(it)^T and dP^T = V dO(it)^T into buffer it & 1 (issuing thread)
  auto issue_s = [&](int it) {
    const int b = it & 1, r = it % kRing;
    const uint32_t tS = tmem + 128 * b, tdP = tS + 64;
    const uint32_t ka = smem_addr(sK), va = smem_addr(sV), qa = smem_addr(sQ + r * Q::BLOCK),
                   da = smem_addr(sDO + r * Q::BLOCK);
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const uint32_t ok_ = (kk >> 2) * L::TILE + (kk & 3) * 32;
      const uint32_t oq = (kk >> 2) * Q::TILE + (kk & 3) * 32;
      umma_f16(tS, make_sdesc_sw128(ka + ok_, 16, 1024), make_sdesc_sw128(qa + oq, 16, 1024),
               IDESC_S, kk > 0 ? 1u : 0u);
      umma_f16(tdP, make_sdesc_sw128(va + ok_, 16, 1024), make_sdesc_sw128(da + oq, 16, 1024),
               IDESC_S, kk > 0 ? 1u : 0u);
    }
    umma_commit(&s_full[b]);
    any_mma = true;
  };
  // log-sum-exp and D of a step's 64 queries, double-buffered in shared memory: thread t < 64
  // loads step it+1's pair while step it runs and stores it before the step's barrier
  auto row_data = [&](int it, float& l, float& dd) {
    const int t_abs = block_of(it) * kQStep + tid;
    const bool valid = t_abs < P.s;
    const int64_t ri = (static_cast<int64_t>(bi) * P.s + t_abs) * P.n_q + head_of(it);
    l = valid ? P.lse[ri] : 0.f;
    dd = valid ? P.D[ri] : 0.f;
  };
  if (tid < kQStep) {
    float l, dd;
    row_data(0, l, dd);
    lse_s[tid] = l;
    D_s[tid] = dd;
  }
  bool ok = true;
  __syncthreads();   // step 0's row data is in shared memory
  if (tid >= kThreads) {
    // ------------------------------------------------------------------ issuing warp
    if (tid == kIssuer) {
      mbar_arrive_expect_tx(kv_full, 2 * L::BLOCK);
#pragma unroll
      for (int c = 0; c < L::SUB; ++c) {
        tma_load_3d(&tma_qkv, kv_full, sK + c * L::TILE, k_col + 64 * c, k0, bi);
        tma_load_3d(&tma_qkv, kv_full, sV + c * L::TILE, v_col + 64 * c, k0, bi);
      }
      for (int m = 0; m < kRing - 1 && m < n_iter; ++m) load_qd(m);
      ok = wait(&qd_full[0], 0, DEVERR_WAIT_FULL) && wait(kv_full, 0, DEVERR_WAIT_FULL);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      if (ok && n_iter > 1) {
        ok = wait(&qd_full[1], 0, DEVERR_WAIT_FULL);
        if (ok) {
          tc_fence_after();
          issue_s(1);
        }
      }
      for (int it = 0; ok && it < n_iter; ++it) {
        const int b = it & 1, r = it % kRing;
        const uint32_t tS = tmem + 128 * b, tdP = tS + 64;
        ok = wait(&p_ready[b], (it >> 1) & 1, DEVERR_WAIT_ACC_EMPTY);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qa = smem_addr(sQ + r * Q::BLOCK), da = smem_addr(sDO + r * Q::BLOCK);
#pragma unroll
        for (int kk = 0; kk < kQStep / 16; ++kk) {
          // A: 16 queries = 8 TMEM columns of P^T / dS^T; B: the [query][dim] tiles read
          // MN-major (N = dim), 16 query rows per MMA
          fa::umma_f16_tmem_a(tdV, tS + packed_col64(kk),
                              make_sdesc_sw128(da + kk * 16 * 128, Q::TILE, 1024), IDESC_KN,
                              (it > 0 || kk > 0) ? 1u : 0u);
          fa::umma_f16_tmem_a(tdK, tdP + packed_col64(kk),
                              make_sdesc_sw128(qa + kk * 16 * 128, Q::TILE, 1024), IDESC_KN,
                              (it > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&m_done[b]);
        // step it+2's S^T and dP^T into this buffer, behind the MMAs that read it
        if (it + 2 < n_iter) {
          ok = wait(&qd_full[(it + 2) % kRing], ((it + 2) / kRing) & 1, DEVERR_WAIT_FULL);
          if (!ok) break;
          tc_fence_after();
          issue_s(it + 2);
        }
        // step it+3's Q and dO into the slot of step it-1, whose dV/dK MMAs are then done
        if (it + kRing - 1 < n_iter) {
          if (it >= 1) ok = wait(&m_done[b ^ 1], ((it - 1) >> 1) & 1, DEVERR_WAIT_ACC_EMPTY);
          if (!ok) break;
          load_qd(it + kRing - 1);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ compute threads
    for (int it = 0; it < n_iter; ++it) {
      const int b = it & 1;
      const uint32_t tS = tmem + 128 * b, tdP = tS + 64;
      const int q0 = block_of(it) * kQStep;
      const float* lse_c = lse_s + b * kQStep;
      const float* D_c = D_s + b * kQStep;
      float nl = 0.f, nd = 0.f;
      if (tid < kQStep && it + 1 < n_iter) row_data(it + 1, nl, nd);
      // S^T(it) done (issued two steps back, or before the loop)
      ok = __all_sync(0xffffffffu, ok && wait(&s_full[b], (it >> 1) & 1, DEVERR_WAIT_ACC_FULL));
      // ---- P^T and dS^T for this key row against this thread's 32 of the step's queries,
      // written as bf16 over the first half of its own S^T / dP^T columns (read before
      // overwrite)
      if (ok) {
        tc_fence_after();
        // no mask: every query is valid and (causal) at or after every key of the block
        const bool plain =
            q0 + kQStep <= P.s && k0 + kBlk <= P.s && (!P.causal || q0 >= k0 + kBlk);
        uint32_t rs[32], rd[32];
        tmem_ld_32x32b_x32(tS + lane_base + 32 * half, rs);
        tmem_ld_32x32b_x32(tdP + lane_base + 32 * half, rd);
        tmem_wait_ld();
        uint32_t pw[16], dw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int c0 = 32 * half + e;
          const float4 l4 = *reinterpret_cast<const float4*>(lse_c + c0);
          const float4 d4 = *reinterpret_cast<const float4*>(D_c + c0);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
          float pr[4], ds[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            pr[u] = exp2_fast(__uint_as_float(rs[e + u]) * P.scale_log2 - lv[u]);
            if (!plain) {
              const int q_abs = q0 + c0 + u;
              if (q_abs >= P.s || k_abs >= P.s || (P.causal && k_abs > q_abs)) pr[u] = 0.f;
            }
            ds[u] = pr[u] * (__uint_as_float(rd[e + u]) - dv[u]);
          }
          pw[e >> 1] = pack_bf16x2(pr[0], pr[1]);
          pw[(e >> 1) + 1] = pack_bf16x2(pr[2], pr[3]);
          dw[e >> 1] = pack_bf16x2(ds[0], ds[1]);
          dw[(e >> 1) + 1] = pack_bf16x2(ds[2], ds[3]);
        }
        st16(tS + lane_base + 32 * half, pw);
        st16(tdP + lane_base + 32 * half, dw);
        fa::tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_ready[b]);
      }
      if (tid < kQStep && it + 1 < n_iter) {
        lse_s[(b ^ 1) * kQStep + tid] = nl;
        D_s[(b ^ 1) * kQStep + tid] = nd;
      }
      // the next step's row data is stored, this step's is read by all; all agree on ok
      if (!compute_bar_and(ok ? 1 : 0)) {
        ok = false;
        break;
      }
    }
    if (ok)
      ok = __all_sync(0xffffffffu, wait(&m_done[(n_iter - 1) & 1], ((n_iter - 1) >> 1) & 1,
                                        DEVERR_WAIT_ACC_EMPTY));
  }
  if (ok && tid < kThreads) {
    tc_fence_after();
    const bool live = k_abs < P.s;
    const int64_t t = static_cast<int64_t>(bi) * P.s + k_abs;
    __nv_bfloat16* rowp = P.dqkv + t * P.ld;
    // split > 1: this CTA's share of dK (unscaled) and dV, added up by the combine kernel
    const int64_t n_tok = static_cast<int64_t>(gridDim.z) * P.s;
    const int n_kv = static_cast<int>(gridDim.y) / P.split;
    float* prow = P.part_kv + ((static_cast<int64_t>(sp) * n_tok + t) * n_kv + g) * 2 * HD;
#pragma unroll 1
    for (int c = half * (HD / 2); c < (half + 1) * (HD / 2); c += 32) {
      float v[32];
      ld32(tdK + lane_base + c, v);
      if (P.split > 1) {
        if (live) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(prow + c)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= P.scale;
        if (live) tc::store_bf16x32(rowp + k_col + c, v);
      }
      ld32(tdV + lane_base + c, v);
      if (P.split > 1) {
        if (live) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(prow + HD + c)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      } else if (live) {
        tc::store_bf16x32(rowp + v_col + c, v);
      }
    }
  }
  __syncthreads();
  if (*abort_flag && tid == kIssuer) {
    const Drain dr{globaltimer_ns(), P.err};
    dr(kv_full, 0);
    for (int r = 0; r < kRing; ++r)
      if (nq[r]) dr(&qd_full[r], (nq[r] - 1) & 1);
    if (any_mma) {
      umma_commit(drain);
      dr(drain, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ======================================================================================= dQ
template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    flash_bwd_dq_kernel(const __grid_constant__ CUtensorMap tma_qkv,
                        const __grid_constant__ CUtensorMap tma_do, const Params P) {
  using namespace sm100;
  using L = Tiles<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = sQ + L::BLOCK;
  uint8_t* sK = sDO + L::BLOCK;      // [2] buffers
  uint8_t* sV = sK + 2 * L::BLOCK;   // [2] buffers
  uint64_t* bar = reinterpret_cast<uint64_t*>(sV + 2 * L::BLOCK);
  uint64_t* qd_full = bar + 0;
  uint64_t* kv_full = bar + 1;       // [2]
  uint64_t* s_full = bar + 3;
  uint64_t* m_done = bar + 4;
  uint64_t* drain = bar + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qb = P.causal ? P.n_blk - 1 - static_cast<int>(blockIdx.x) : blockIdx.x;
  const int j = blockIdx.y, bi = blockIdx.z;
  const int shard = j / P.qh, jl = j - shard * P.qh;
  const int g = j / P.group, gl = g - shard * P.kh;
  const int q_col = shard * P.R_a + jl * HD;
  const int k_col = shard * P.R_a + (P.qh + gl) * HD;
  const int v_col = shard * P.R_a + (P.qh + P.kh + gl) * HD;
  const int q0 = qb * kBlk;
  const int nkb = P.causal ? qb + 1 : P.n_blk;

  if (tid == 0) {
    mbar_init(qd_full, 1);
    mbar_init(&kv_full[0], 1);
    mbar_init(&kv_full[1], 1);
    mbar_init(s_full, 1);
    mbar_init(m_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tma_qkv);
    tma_prefetch_desc(&tma_do);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const int row = tid & (kBlk - 1);
  const int half = tid >> 7;   // columns 64 half .. 64 half + 63
  const int q_abs = q0 + row;
  const bool q_live = q_abs < P.s;
  const int64_t ri = (static_cast<int64_t>(bi) * P.s + q_abs) * P.n_q + j;
  const float lse_r = q_live ? P.lse[ri] : 0.f;
  const float D_r = q_live ? P.D[ri] : 0.f;
  auto wait = [&](uint64_t* b, uint32_t par, uint32_t site) {
    return mbar_wait(b, par, abort_flag, P.err, site);
  };
  constexpr uint32_t IDESC_KK = make_idesc_bf16(128, 128, false, false);   // S, dP
  constexpr uint32_t IDESC_KN = make_idesc_bf16(128, HD, false, true);     // dQ

  uint32_t nk[2] = {0, 0};   // K/V loads issued per buffer (thread 0)
  bool any_mma = false;
  auto load_kv = [&](int kb) {
    const int b = kb & 1;
    mbar_arrive_expect_tx(&kv_full[b], 2 * L::BLOCK);
#pragma unroll
    for (int c = 0; c < L::SUB; ++c) {
      tma_load_3d(&tma_qkv, &kv_full[b], sK + b * L::BLOCK + c * L::TILE, k_col + 64 * c,
                  kb * kBlk, bi);
      tma_load_3d(&tma_qkv, &kv_full[b], sV + b * L::BLOCK + c * L::TILE, v_col + 64 * c,
                  kb * kBlk, bi);
    }
    ++nk[b];
  };
  // S = Q K(kb)^T and dP = dO V(kb)^T (thread 0)
  auto issue_s = [&](int kb) {
    const int b = kb & 1;
    const uint32_t qa = smem_addr(sQ), da = smem_addr(sDO), ka = smem_addr(sK + b * L::BLOCK),
                   va = smem_addr(sV + b * L::BLOCK);
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const uint32_t off = (kk >> 2) * L::TILE + (kk & 3) * 32;
      umma_f16(tS, make_sdesc_sw128(qa + off, 16, 1024), make_sdesc_sw128(ka + off, 16, 1024),
               IDESC_KK, kk > 0 ? 1u : 0u);
      umma_f16(tdP, make_sdesc_sw128(da + off, 16, 1024), make_sdesc_sw128(va + off, 16, 1024),
               IDESC_KK, kk > 0 ? 1u : 0u);
    }
    umma_commit(s_full);
    any_mma = true;
  };
  bool ok = true;
  if (tid == 0) {
    mbar_arrive_expect_tx(qd_full, 2 * L::BLOCK);
#pragma unroll
    for (int c = 0; c < L::SUB; ++c) {
      tma_load_3d(&tma_qkv, qd_full, sQ + c * L::TILE, q_col + 64 * c, q0, bi);
      tma_load_3d(&tma_do, qd_full, sDO + c * L::TILE, j * HD + 64 * c, q0, bi);
    }
    load_kv(0);
    if (nkb > 1) load_kv(1);
    ok = wait(&kv_full[0], 0, DEVERR_WAIT_FULL) && wait(qd_full, 0, DEVERR_WAIT_FULL);
    if (ok) {
      tc_fence_after();
      issue_s(0);
    }
  }
  __syncthreads();
  for (int kb = 0; kb < nkb; ++kb) {
    const int k0 = kb * kBlk;
    // S(kb) done: the MMAs run in issue order, so dQ of the previous step is done too and the
    // other K/V buffer is free for step kb+1
    ok = __all_sync(0xffffffffu, ok && wait(s_full, kb & 1, DEVERR_WAIT_ACC_FULL));
    if (ok && tid == 0 && kb >= 1 && kb + 1 < nkb) load_kv(kb + 1);
    // ---- dS for this query row against this thread's 64 of the block's 128 keys, bf16 over
    // the first half of this half's S columns (all of this thread's S and dP are read before
    // any of them is overwritten)
    if (ok) {
      tc_fence_after();
      // no mask inside the block: every key is valid and (causal) before every query
      const bool plain = q0 + kBlk <= P.s && k0 + kBlk <= P.s && (!P.causal || k0 < q0);
      float sv[64], dp[64];
      {
        uint32_t r[4][32];
        tmem_ld_32x32b_x32(tS + lane_base + 64 * half, r[0]);
        tmem_ld_32x32b_x32(tS + lane_base + 64 * half + 32, r[1]);
        tmem_ld_32x32b_x32(tdP + lane_base + 64 * half, r[2]);
        tmem_ld_32x32b_x32(tdP + lane_base + 64 * half + 32, r[3]);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          sv[e] = __uint_as_float(r[e >> 5][e & 31]);
          dp[e] = __uint_as_float(r[2 + (e >> 5)][e & 31]);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int c0 = 64 * half + 32 * c;
        uint32_t dw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float ds[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            float pr = exp2_fast(sv[32 * c + e + u] * P.scale_log2 - lse_r);
            if (!plain) {
              const int k_abs = k0 + c0 + e + u;
              if (!q_live || k_abs >= P.s || (P.causal && k_abs > q_abs)) pr = 0.f;
            }
            ds[u] = pr * (dp[32 * c + e + u] - D_r);
          }
          dw[e >> 1] = pack_bf16x2(ds[0], ds[1]);
        }
        st16(tS + lane_base + packed_col(c0 / 2), dw);
      }
      fa::tmem_wait_st();
    }
    tc_fence_before();
    // every thread's dS is stored; all agree on ok
    if (!__syncthreads_and(ok ? 1 : 0)) {
      ok = false;
      break;
    }
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ka = smem_addr(sK + (kb & 1) * L::BLOCK);
#pragma unroll
      for (int kk = 0; kk < kBlk / 16; ++kk) {
        // A: 16 keys = 8 TMEM columns of dS; B: the [key][dim] K tile read MN-major
        fa::umma_f16_tmem_a(tdQ, tS + packed_col(kk * 8),
                            make_sdesc_sw128(ka + kk * 16 * 128, L::TILE, 1024), IDESC_KN,
                            (kb > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(m_done);
      // the next step's S and dP right behind: they overwrite dS only after this MMA has read
      // it (issue order)
      if (kb + 1 < nkb) {
        ok = wait(&kv_full[(kb + 1) & 1], ((kb + 1) >> 1) & 1, DEVERR_WAIT_FULL);
        if (ok) {
          tc_fence_after();
          issue_s(kb + 1);
        }
      }
    }
  }
  if (!__syncthreads_and(ok ? 1 : 0)) ok = false;
  if (ok) ok = __all_sync(0xffffffffu, wait(m_done, (nkb - 1) & 1, DEVERR_WAIT_ACC_EMPTY));
  if (ok) {
    tc_fence_after();
    __nv_bfloat16* rowp = P.dqkv + (static_cast<int64_t>(bi) * P.s + q_abs) * P.ld + q_col;
#pragma unroll 1
    for (int c = half * (HD / 2); c < (half + 1) * (HD / 2); c += 32) {
      float v[32];
      ld32(tdQ + lane_base + c, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] *= P.scale;
      if (q_live) tc::store_bf16x32(rowp + c, v);
    }
  }
  __syncthreads();
  if (*abort_flag && tid == 0) {
    const Drain dr{globaltimer_ns(), P.err};
    dr(qd_full, 0);
    for (int b = 0; b < 2; ++b)
      if (nk[b]) dr(&kv_full[b], (nk[b] - 1) & 1);
    if (any_mma) {
      umma_commit(drain);
      dr(drain, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// dK = scale * sum_sp partial dK, dV = sum_sp partial dV, slices added in order; bf16 into dqkv.
// One thread per 4 consecutive dims of one (token, KV head).
template <int HD>
__global__ void __launch_bounds__(256) combine_kv_kernel(const float* part, int split,
                                                         int64_t n_tok, int n_kv, int kh,
                                                         int qh, int64_t R_a, int64_t ld,
                                                         float scale, __nv_bfloat16* dqkv) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  constexpr int V4 = HD / 4;
  if (idx >= n_tok * n_kv * 2 * V4) return;
  const int e4 = static_cast<int>(idx % V4);
  const int which = static_cast<int>((idx / V4) & 1);   // 0: dK, 1: dV
  const int64_t tg = idx / (2 * V4);
  const int g = static_cast<int>(tg % n_kv);
  const int64_t t = tg / n_kv;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sp = 0; sp < split; ++sp) {
    const float4 v = reinterpret_cast<const float4*>(
        part + ((static_cast<int64_t>(sp) * n_tok + t) * n_kv + g) * 2 * HD + which * HD)[e4];
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  const float f = which == 0 ? scale : 1.f;
  const int shard = g / kh, gl = g - shard * kh;
  __nv_bfloat16* dst = dqkv + t * ld + shard * R_a + (qh + which * kh + gl) * HD + 4 * e4;
  reinterpret_cast<uint2*>(dst)[0] = make_uint2(pack_bf16x2(acc.x * f, acc.y * f),
                                                pack_bf16x2(acc.z * f, acc.w * f));
}

template <int HD>
constexpr int dkv_smem() {
  return 2 * Tiles<HD>::BLOCK + 2 * kRing * Tiles64<HD>::BLOCK + 4 * kQStep * 4 + 128 + 1024;
}
// at least 120 KB, so that no second CTA (which would wait for the 512 TMEM columns) shares an SM
template <int HD>
constexpr int dq_smem() {
  return 6 * Tiles<HD>::BLOCK + 128 + 1024 > 120 * 1024 ? 6 * Tiles<HD>::BLOCK + 128 + 1024
                                                         : 120 * 1024;
}
template <int HD>
constexpr int dkv_smem_padded() { return dkv_smem<HD>() > 120 * 1024 ? dkv_smem<HD>() : 120 * 1024; }

// Host launcher.  qkv and dqkv [b][s][p*R_a] bf16 (packed per shard: Q heads, K heads, V heads),
// dO [b][s][n_q*HD] bf16, lse and D [b*s][n_q] fp32.
template <int HD>
inline tp_status launch_bwd(const void* qkv, const void* dO, const float* lse, const float* D,
                            void* dqkv, int64_t b, int64_t s, int n_q, int qh, int kh, int group,
                            int64_t R_a, int p, int causal, float* part_kv, cudaStream_t st) {
  CUtensorMap mq, md;
  const uint64_t cols = static_cast<uint64_t>(p) * R_a;
  tp_status r = encode_tmap_bf16_3d(&mq, qkv, cols, static_cast<uint64_t>(s),
                                    static_cast<uint64_t>(b), cols * 2,
                                    cols * 2 * static_cast<uint64_t>(s), 64, kBlk);
  if (r != TP_OK) return r;
  const uint64_t dcols = static_cast<uint64_t>(n_q) * HD;
  r = encode_tmap_bf16_3d(&md, dO, dcols, static_cast<uint64_t>(s), static_cast<uint64_t>(b),
                          dcols * 2, dcols * 2 * static_cast<uint64_t>(s), 64, kBlk);
  if (r != TP_OK) return r;
  // 64-row boxes of the same tensors: the dK/dV kernel's query steps
  CUtensorMap mq64, md64;
  r = encode_tmap_bf16_3d(&mq64, qkv, cols, static_cast<uint64_t>(s), static_cast<uint64_t>(b),
                          cols * 2, cols * 2 * static_cast<uint64_t>(s), 64, kQStep);
  if (r != TP_OK) return r;
  r = encode_tmap_bf16_3d(&md64, dO, dcols, static_cast<uint64_t>(s), static_cast<uint64_t>(b),
                          dcols * 2, dcols * 2 * static_cast<uint64_t>(s), 64, kQStep);
  if (r != TP_OK) return r;
  static int attr_set[64] = {0};
  int dev = 0;
  TP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 64 && !attr_set[dev]) {
    TP_CUDA_TRY(cudaFuncSetAttribute(flash_bwd_dkv_kernel<HD>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, dkv_smem_padded<HD>()));
    TP_CUDA_TRY(cudaFuncSetAttribute(flash_bwd_dq_kernel<HD>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, dq_smem<HD>()));
    attr_set[dev] = 1;
  }
  Params P;
  P.s = static_cast<int32_t>(s);
  P.n_q = n_q; P.qh = qh; P.kh = kh; P.group = group;
  P.R_a = static_cast<int32_t>(R_a);
  P.n_blk = static_cast<int32_t>(ceil_div(s, kBlk));
  P.causal = causal;
  P.ld = static_cast<int64_t>(cols);
  P.scale = 1.0f / sqrtf(static_cast<float>(HD));
  P.scale_log2 = P.scale * 1.4426950408889634f;
  P.lse = lse;
  P.D = D;
  P.dqkv = static_cast<__nv_bfloat16*>(dqkv);
  P.err = device_error_word();
  const int n_kv = n_q / group;
  // one CTA per query head of the group when the workspace slice is given (more CTAs than the
  // key blocks times KV heads alone); their fp32 shares are added in order afterwards
  P.split = (part_kv && group > 1) ? group : 1;
  P.part_kv = part_kv;
  ProfScope prof(st, "attn_bwd_flash");
  flash_bwd_dkv_kernel<HD><<<dim3(static_cast<unsigned>(P.n_blk),
                                  static_cast<unsigned>(n_kv * P.split), static_cast<unsigned>(b)),
                             kThreadsIssue, dkv_smem_padded<HD>(), st>>>(mq, mq64, md64, P);
  TP_LAUNCH_CHECK();
  if (P.split > 1) {
    const int64_t n_tok = b * s;
    const int64_t work = n_tok * n_kv * 2 * (HD / 4);
    combine_kv_kernel<HD><<<static_cast<unsigned>(ceil_div(work, 256)), 256, 0, st>>>(
        part_kv, P.split, n_tok, n_kv, kh, qh, R_a, P.ld, P.scale, P.dqkv);
    TP_LAUNCH_CHECK();
  }
  flash_bwd_dq_kernel<HD><<<dim3(static_cast<unsigned>(P.n_blk), static_cast<unsigned>(n_q),
                                 static_cast<unsigned>(b)),
                            kThreads, dq_smem<HD>(), st>>>(mq, md, P);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace fb
}  // namespace tp
