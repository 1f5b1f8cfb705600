// Backward pass of the tensor-parallel GQA attention block (prefill, bf16).
//
//   "Tensor Parallelism" (klaylearn), Notes: Q/K/V column-parallel, attention local to the
//   shard's heads, output projection row-parallel.  "How does tensor parallelism split a
//   transformer feed-forward block's two matmuls", "The backward pass": dY is replicated, each
//   shard's weight gradients need no exchange, the input gradient is the sum of per-shard
//   partials; the same page notes the pattern carries over to multi-head attention.
//
// Per shard i, with O_i the shard's attention output and dY replicated:
//   dWo_i = O_i^T dY                      (no exchange)
//   dO_i  = dY Wo_i^T
//   (dQ, dK, dV) of every head from dO, Q, K, V, O and the forward's row log-sum-exp:
//       P = softmax(S), dV = P^T dO, dP = dO V^T, D = rowsum(dO * O), dS = P * (dP - D),
//       dQ = dS K / sqrt(hd), dK = dS^T Q / sqrt(hd); a KV head collects the dK, dV of every
//       query head of its group
//   dWqkv_i = x^T [dQ dK dV]_i             (no exchange)
//   dx = sum_i [dQ dK dV]_i Wqkv_i         (per-shard partials, summed in shard order)
//
// The forward quantities Q, K, V, O and the log-sum-exp are recomputed from x (the forward call
// keeps no activations).  The GEMMs run on the tcgen05 core.  dQ, dK and dV run in the tcgen05
// kernels of flash_bwd.cuh for head_dim 64 and 128, otherwise in SIMT kernels (one warp per query
// row and head for dQ, one per key row and KV head for dK and dV).  Each output is summed by one
// CTA or warp in a fixed order; no atomics.
#pragma once

#include "attn.cuh"
#include "flash_bwd.cuh"

namespace tp {
namespace attn {

// D[t][j] = sum_e dO[t][j][e] O[t][j][e]; one warp per (token, query head).
template <typename T>
__global__ void __launch_bounds__(128) bwd_rowdot_kernel(const T* o, const T* dO, int64_t tokens,
                                                        int n_q, int hd, float* D) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= tokens * n_q) return;
  const T* a = o + wid * hd;   // o and dO rows are [tokens][n_q][hd]
  const T* b = dO + wid * hd;
  float acc = 0.f;
  for (int e = lane; e < hd; e += 32) acc = fmaf(to_f(a[e]), to_f(b[e]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) D[wid] = acc;
}

constexpr int kBwdMaxPerLane = 8;   // head_dim <= 256

// dQ of query head j at token t: sum over the visible keys of dS * k, times 1/sqrt(hd).
template <typename T>
__global__ void __launch_bounds__(128) bwd_dq_kernel(const T* qkv, const T* dO, QkvIdx ix,
                                                     const float* lse2, const float* D,
                                                     int64_t b, int64_t s, int n_q, int causal,
                                                     float scale_log2, float scale, T* dqkv) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= b * s * n_q) return;
  const int j = static_cast<int>(wid % n_q);
  const int64_t t = wid / n_q;
  const int64_t bi = t / s, pos = t - bi * s;
  const int g = j / ix.group;
  const int per = (ix.hd + 31) / 32;
  float q[kBwdMaxPerLane], go[kBwdMaxPerLane], dq[kBwdMaxPerLane];
#pragma unroll
  for (int r = 0; r < kBwdMaxPerLane; ++r) {
    const int e = lane + 32 * r;
    const bool in = r < per && e < ix.hd;
    q[r] = in ? to_f(qkv[ix.q(t, j) + e]) * scale_log2 : 0.f;
    go[r] = in ? to_f(dO[(t * n_q + j) * ix.hd + e]) : 0.f;
    dq[r] = 0.f;
  }
  const float lse = lse2[t * n_q + j], dd = D[t * n_q + j];
  const int64_t last = causal ? pos : s - 1;
  for (int64_t kp = 0; kp <= last; ++kp) {
    const int64_t tk = bi * s + kp;
    const int64_t kb = ix.k(tk, g), vb = ix.v(tk, g);
    float sc = 0.f, dp = 0.f, kv[kBwdMaxPerLane];
#pragma unroll
    for (int r = 0; r < kBwdMaxPerLane; ++r) {
      const int e = lane + 32 * r;
      kv[r] = 0.f;
      if (r < per && e < ix.hd) {
        kv[r] = to_f(qkv[kb + e]);
        sc = fmaf(q[r], kv[r], sc);
        dp = fmaf(go[r], to_f(qkv[vb + e]), dp);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      sc += __shfl_xor_sync(0xffffffffu, sc, off);
      dp += __shfl_xor_sync(0xffffffffu, dp, off);
    }
    const float ds = exp2f(sc - lse) * (dp - dd);
#pragma unroll
    for (int r = 0; r < kBwdMaxPerLane; ++r) dq[r] = fmaf(ds, kv[r], dq[r]);
  }
#pragma unroll
  for (int r = 0; r < kBwdMaxPerLane; ++r) {
    const int e = lane + 32 * r;
    if (r < per && e < ix.hd) dqkv[ix.q(t, j) + e] = from_f<T>(dq[r] * scale);
  }
}

// dK and dV of KV head g at key token tk: sums over every query head of the group and every
// query that sees the key, in query-then-head order.
template <typename T>
__global__ void __launch_bounds__(128) bwd_dkv_kernel(const T* qkv, const T* dO, QkvIdx ix,
                                                      const float* lse2, const float* D,
                                                      int64_t b, int64_t s, int n_q, int n_kv,
                                                      int causal, float scale_log2, float scale,
                                                      T* dqkv) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= b * s * n_kv) return;
  const int g = static_cast<int>(wid % n_kv);
  const int64_t tk = wid / n_kv;
  const int64_t bi = tk / s, kpos = tk - bi * s;
  const int per = (ix.hd + 31) / 32;
  float kk[kBwdMaxPerLane], vv[kBwdMaxPerLane], dk[kBwdMaxPerLane], dv[kBwdMaxPerLane];
#pragma unroll
  for (int r = 0; r < kBwdMaxPerLane; ++r) {
    const int e = lane + 32 * r;
    const bool in = r < per && e < ix.hd;
    kk[r] = in ? to_f(qkv[ix.k(tk, g) + e]) * scale_log2 : 0.f;
    vv[r] = in ? to_f(qkv[ix.v(tk, g) + e]) : 0.f;
    dk[r] = dv[r] = 0.f;
  }
  const int64_t first = causal ? kpos : 0;
  for (int64_t qp = first; qp < s; ++qp) {
    const int64_t t = bi * s + qp;
    for (int a = 0; a < ix.group; ++a) {
      const int j = g * ix.group + a;
      const int64_t qb = ix.q(t, j), ob = (t * n_q + j) * ix.hd;
      float sc = 0.f, dp = 0.f, qv[kBwdMaxPerLane], gv[kBwdMaxPerLane];
#pragma unroll
      for (int r = 0; r < kBwdMaxPerLane; ++r) {
        const int e = lane + 32 * r;
        qv[r] = gv[r] = 0.f;
        if (r < per && e < ix.hd) {
          qv[r] = to_f(qkv[qb + e]);
          gv[r] = to_f(dO[ob + e]);
          sc = fmaf(qv[r], kk[r], sc);
          dp = fmaf(gv[r], vv[r], dp);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sc += __shfl_xor_sync(0xffffffffu, sc, off);
        dp += __shfl_xor_sync(0xffffffffu, dp, off);
      }
      const float pr = exp2f(sc - lse2[t * n_q + j]);
      const float ds = pr * (dp - D[t * n_q + j]);
#pragma unroll
      for (int r = 0; r < kBwdMaxPerLane; ++r) {
        dk[r] = fmaf(ds, qv[r], dk[r]);
        dv[r] = fmaf(pr, gv[r], dv[r]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kBwdMaxPerLane; ++r) {
    const int e = lane + 32 * r;
    if (r < per && e < ix.hd) {
      dqkv[ix.k(tk, g) + e] = from_f<T>(dk[r] * scale);
      dqkv[ix.v(tk, g) + e] = from_f<T>(dv[r]);
    }
  }
}

}  // namespace attn

// Workspace of the backward pass (offsets into the caller's buffer, 256-byte aligned).
struct AttnBwdLayout {
  size_t qkv, o, dO, dqkv, lse, D, part, sk, bytes;
};

inline AttnBwdLayout attn_bwd_layout(const AttnLayout& L) {
  AttnBwdLayout B;
  const size_t qkvb = static_cast<size_t>(L.tokens * L.p * L.R_a) * 2;
  const size_t ob = static_cast<size_t>(L.tokens * L.n_q * L.hd) * 2;
  const size_t rowb = static_cast<size_t>(L.tokens * L.n_q) * 4;
  // the dX partials; before them, the per-query-head dK/dV shares of the flash kernels
  const size_t partb = std::max(static_cast<size_t>(L.p * L.tokens * L.h),
                                static_cast<size_t>(L.tokens * L.n_q * 2 * L.hd)) * 4;
  B.qkv = 0;
  B.o = B.qkv + align256(qkvb);
  B.dO = B.o + align256(ob);
  B.dqkv = B.dO + align256(ob);
  B.lse = B.dqkv + align256(qkvb);
  B.D = B.lse + align256(rowb);
  B.part = B.D + align256(rowb);
  B.sk = B.part + align256(partb);
  B.bytes = B.sk + align256(attn_sk_bytes(L));
  return B;
}

// ``sp``: the sequence-parallel form -- the dx partials are reduce-scattered into
// sp->y (the shards' token slices) instead of summed into dx.
inline tp_status attn_backward(const AttnLayout& L, const void* x, const void* wqkv,
                               const void* wo_p, const void* dy, void* dx, float* dwqkv_p,
                               float* dwo_p, void* ws, cudaStream_t s,
                               const seqpar::SpOut* sp = nullptr) {
  using tc::Operand;
  using tc::TileCfg;
  using BF = __nv_bfloat16;
  const AttnBwdLayout B = attn_bwd_layout(L);
  uint8_t* w = static_cast<uint8_t*>(ws);
  BF* qkv = reinterpret_cast<BF*>(w + B.qkv);
  BF* o = reinterpret_cast<BF*>(w + B.o);
  BF* dO = reinterpret_cast<BF*>(w + B.dO);
  BF* dqkv = reinterpret_cast<BF*>(w + B.dqkv);
  float* lse = reinterpret_cast<float*>(w + B.lse);
  float* D = reinterpret_cast<float*>(w + B.D);
  float* part = reinterpret_cast<float*>(w + B.part);
  const int64_t T = L.tokens, P = L.p, K = static_cast<int64_t>(L.qh) * L.hd;
  const int64_t nqhd = static_cast<int64_t>(L.n_q) * L.hd;
  tp_status st;
  // forward quantities: qkv = x Wqkv, O and the row log-sum-exp
  if ((st = attn_tc::qkv_proj(L, x, wqkv, qkv, w + B.sk, B.bytes - B.sk, s)) != TP_OK) return st;
  if ((st = attn_core<BF>(L, qkv, o, nullptr, nullptr, nullptr, nullptr, s, lse)) != TP_OK)
    return st;
  // dO_i = dY Wo_i^T into the [tokens][n_q hd] layout of O (shard i at column i qh hd)
  {
    const Operand a{dy, false, T, L.h, 1, L.h, 0};
    const Operand bo{wo_p, true, K, L.h, P, K, L.h * K};
    tc::EpiStoreBf16::Params ep;
    ep.out = dO;
    ep.ld = nqhd;
    ep.col_off = K;
    ep.rows_valid = static_cast<int32_t>(T);
    ep.cols_valid = static_cast<int32_t>(K);
    st = K % 256 == 0
             ? tc::run_gemm_pair<attn_tc::PP<false, true>, tc::EpiStoreBf16>(
                   a, bo, T, K, L.h, P, ep, s, "attn_do_gemm")
             : tc::run_gemm<TileCfg<128, 1, false, true, 6>, tc::EpiStoreBf16>(
                   a, bo, T, K, L.h, P, ep, s, "attn_do_gemm");
    if (st != TP_OK) return st;
  }
  // dWo_i[n][c] = sum_t dY[t][n] O_i[t][c]   (no exchange between shards)
  {
    const Operand a{dy, true, L.h, T, 1, L.h, 0};
    const Operand bo{o, true, K, T, P, nqhd, K};
    tc::EpiStoreF32::Params ep;
    ep.out = dwo_p;
    ep.ld = K;
    ep.batch_stride = L.h * K;
    ep.rows_valid = static_cast<int32_t>(L.h);
    ep.cols_valid = static_cast<int32_t>(K);
    ep.swap = 0;
    st = K % 256 == 0
             ? tc::run_gemm_pair<attn_tc::PP<true, true>, tc::EpiStoreF32>(
                   a, bo, L.h, K, T, P, ep, s, "attn_dwo_gemm")
             : tc::run_gemm<TileCfg<128, 1, true, true, 6>, tc::EpiStoreF32>(
                   a, bo, L.h, K, T, P, ep, s, "attn_dwo_gemm");
    if (st != TP_OK) return st;
  }
  // dQ, dK, dV of every head: tcgen05 kernels for head_dim 64/128, SIMT kernels otherwise
  {
#define return_if_error(expr)          \
  do {                                 \
    tp_status _r = (expr);             \
    if (_r != TP_OK) return _r;        \
  } while (0)
    attn::QkvIdx ix{P * L.R_a, L.R_a, L.qh, L.kh, L.hd, L.n_q / L.n_kv};
    const float scale = 1.0f / sqrtf(static_cast<float>(L.hd));
    const float scale_log2 = scale * 1.4426950408889634f;
    const int64_t rows = T * L.n_q, krows = T * L.n_kv;
    if (ceil_div(rows * 32, 128) > INT32_MAX) return set_error(TP_ERR_UNSUPPORTED, "grid too large");
    {
      ProfScope prof(s, "attn_bwd_rowdot");
      attn::bwd_rowdot_kernel<BF><<<static_cast<unsigned>(ceil_div(rows * 32, 128)), 128, 0, s>>>(
          o, dO, T, L.n_q, L.hd, D);
      TP_LAUNCH_CHECK();
    }
    const int group = L.n_q / L.n_kv;
    if ((L.hd == 128 || L.hd == 64) && L.b <= 65535 && L.s <= INT32_MAX) {
      if (L.hd == 128)
        return_if_error(fb::launch_bwd<128>(qkv, dO, lse, D, dqkv, L.b, L.s, L.n_q, L.qh, L.kh,
                                            group, L.R_a, L.p, L.causal, part, s));
      else
        return_if_error(fb::launch_bwd<64>(qkv, dO, lse, D, dqkv, L.b, L.s, L.n_q, L.qh, L.kh,
                                           group, L.R_a, L.p, L.causal, part, s));
    } else {
    ProfScope prof(s, "attn_bwd_core");
    attn::bwd_dq_kernel<BF><<<static_cast<unsigned>(ceil_div(rows * 32, 128)), 128, 0, s>>>(
        qkv, dO, ix, lse, D, L.b, L.s, L.n_q, L.causal, scale_log2, scale, dqkv);
    TP_LAUNCH_CHECK();
    attn::bwd_dkv_kernel<BF><<<static_cast<unsigned>(ceil_div(krows * 32, 128)), 128, 0, s>>>(
        qkv, dO, ix, lse, D, L.b, L.s, L.n_q, L.n_kv, L.causal, scale_log2, scale, dqkv);
    TP_LAUNCH_CHECK();
    }
  }
#undef return_if_error
  // dWqkv_i[r][k] = sum_t dqkv_i[t][r] x[t][k]   (no exchange between shards)
  {
    const Operand a{dqkv, true, L.R_a, T, P, P * L.R_a, L.R_a};
    const Operand bx{x, true, L.h, T, 1, L.h, 0};
    tc::EpiStoreF32::Params ep;
    ep.out = dwqkv_p;
    ep.ld = L.h;
    ep.batch_stride = L.R_a * L.h;
    ep.rows_valid = static_cast<int32_t>(L.R_a);
    ep.cols_valid = static_cast<int32_t>(L.h);
    ep.swap = 0;
    st = tc::run_gemm_pair<attn_tc::PP<true, true>, tc::EpiStoreF32>(
        a, bx, L.R_a, L.h, T, P, ep, s, "attn_dwqkv_gemm");
    if (st != TP_OK) return st;
  }
  // dx_i = dqkv_i Wqkv_i (partials), then dx = sum_i dx_i in shard order; with
  // TP_REDUCE_FUSED the GEMM adds the shards in its accumulator and writes dx itself
  {
    const Operand a{dqkv, false, T, L.R_a, P, P * L.R_a, L.R_a};
    const Operand bw{wqkv, true, L.h, L.R_a, P, L.h, L.R_a * L.h};
    if (L.reduce_mode == TP_REDUCE_FUSED && !sp) {
      tc::EpiReduceOut::Params ep;
      ep.out = dx;
      ep.residual = nullptr;
      ep.ld = L.h;
      ep.rows_valid = static_cast<int32_t>(T);
      ep.cols_valid = static_cast<int32_t>(L.h);
      ep.out_bf16 = 1;
      ep.swap = 0;
      return tc::run_gemm_pair<attn_tc::PP<false, true>, tc::EpiReduceOut>(
          a, bw, T, L.h, L.R_a, P, ep, s, "attn_dx_gemm", -1, true);
    }
    tc::EpiStoreF32::Params ep;
    ep.out = part;
    ep.ld = L.h;
    ep.batch_stride = T * L.h;
    ep.rows_valid = static_cast<int32_t>(T);
    ep.cols_valid = static_cast<int32_t>(L.h);
    ep.swap = 0;
    st = tc::run_gemm_pair<attn_tc::PP<false, true>, tc::EpiStoreF32>(
        a, bw, T, L.h, L.R_a, P, ep, s, "attn_dx_gemm");
    if (st != TP_OK) return st;
  }
  if (sp)   // the all-gather's gradient: dx reduce-scattered into the token slices
    return seqpar::reduce_scatter(part, L.p, T, L.h, nullptr, sp->y, TP_BF16, nullptr,
                                  TP_BF16, L.norm_eps, s);
  return reduce::launch(part, TP_F32, L.p, T * L.h, nullptr, dx, TP_BF16, s);
}

inline tp_status attn_unpack_grads(const AttnLayout& L, const float* dwqkv_p, const float* dwo_p,
                                   float* dwq, float* dwk, float* dwv, float* dwo,
                                   cudaStream_t s) {
  pack::ColMap cm{};
  cm.kind = 2;
  cm.R = L.R_a;
  cm.q_rows = static_cast<int64_t>(L.qh) * L.hd;
  cm.k_rows = static_cast<int64_t>(L.kh) * L.hd;
  cm.src[0] = dwq; cm.src[1] = dwk; cm.src[2] = dwv;
  cm.ld[0] = static_cast<int64_t>(L.n_q) * L.hd;
  cm.ld[1] = cm.ld[2] = static_cast<int64_t>(L.n_kv) * L.hd;
  const int64_t rows = L.p * L.R_a;
  dim3 blk(32, 8);
  dim3 g1(static_cast<unsigned>(ceil_div(rows, 32)), static_cast<unsigned>(ceil_div(L.h, 32)), 1);
  if (!pack::grid_ok(g1.x, g1.y, 1)) return set_error(TP_ERR_UNSUPPORTED, "unpack grid too large");
  pack::unpack_cols_kernel<<<g1, blk, 0, s>>>(dwqkv_p, rows, L.h, cm, dwq, dwk, dwv);
  TP_LAUNCH_CHECK();
  const int64_t K = static_cast<int64_t>(L.qh) * L.hd;
  dim3 g2(static_cast<unsigned>(ceil_div(L.h, 32)), static_cast<unsigned>(ceil_div(K, 32)),
          static_cast<unsigned>(L.p));
  if (!pack::grid_ok(g2.x, g2.y, g2.z)) return set_error(TP_ERR_UNSUPPORTED, "unpack grid too large");
  pack::unpack_rows_kernel<<<g2, blk, 0, s>>>(dwo_p, L.p, L.h, K, K, dwo, L.h);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace tp
