// Tensor-parallel MLP block: packing, forward, backward.
//
// "How does tensor parallelism split a transformer feed-forward block's two matmuls across
// devices?": column-parallel first matmul with the activation local to each shard, row-parallel
// second matmul producing full-shape partial sums, one reduction; backward with per-shard weight
// gradients and a reduced input gradient.  "Tensor Parallelism" (klaylearn), Notes: up/gate
// projections sharded column-wise.
//
// All p shards live on this GPU.  Because x is replicated, the column-parallel matmuls of all
// shards are one GEMM over the concatenated packed weights (their outputs are the column slices
// h_i, laid side by side); the row-parallel matmul is a batched GEMM with one problem per shard,
// each producing its own full-shape partial y_i; the partials are then summed in shard order.
#include <algorithm>

#include "gemm_launch.cuh"
#include "gemm_pair.cuh"
#include "mlp_decode.cuh"
#include "moe.cuh"
#include "pack.cuh"
#include "reduce.cuh"
#include "seqpar.cuh"
#include "simt.cuh"
#include "tp_common.cuh"

namespace tp {
namespace {

using tc::Operand;
using tc::TileCfg;

constexpr int stages_for(int bn, int a_sub) {
  return std::min(8, (200 * 1024) / (128 * a_sub * 64 * 2 + bn * 64 * 2));
}

struct MlpLayout {
  int64_t T, d, F, Fs, Fsp, R;
  int p, act, dtype, eb, y_dtype, reduce_mode;
  float norm_eps;
  bool tc;                      // bf16 with 16-byte rows: the tensor-core path
  size_t w1p_bytes, w2p_bytes;
  size_t saved_z_off, saved_h_off, saved_bytes;
  size_t fz_off, fh_off, fpart_off, fsk_off, fwd_ws;
  size_t bdh_off, bdz_off, bpart_off, bwd_ws;
};

template <class C> struct Tag { using type = C; };
// 256 x 256 tiles on SM pairs (cta_group::2): the prefill and backward GEMMs
template <bool A_MN, bool B_MN>
using PP = tc::PairCfg<A_MN, B_MN, 6>;
template <int BN, int ASUB>
using KK = TileCfg<BN, ASUB, false, false, stages_for(BN, ASUB)>;

// Swapped GEMMs put the weights on the 128-row M side and the T tokens on N: pick N by T.
template <int ASUB, class F>
auto by_tokens(int64_t T, F&& f) {
  if (T <= 16) return f(Tag<KK<16, ASUB>>{});
  if (T <= 64) return f(Tag<KK<64, ASUB>>{});
  return f(Tag<KK<128, ASUB>>{});
}

constexpr int64_t kSwapMaxT = 128;   // token counts up to this use the swapped (decode) tiles

// stream-K plans of the forward GEMMs (bytes of counters + partial slots); empty if unused
// output tiles of the swapped (decode) up and down GEMMs
int64_t up_tiles(const MlpLayout& L) {
  return ceil_div(L.p * L.R, L.act == TP_ACT_SWIGLU ? 256 : 128);
}
int64_t down_tiles(const MlpLayout& L) { return L.p * ceil_div(L.d, 128); }

// The one-launch decode MLP (csrc/mlp_decode.cuh): tensor-core path, 1..64 tokens, separate
// shard reduce.  Its counters (next work item, finished up tiles per shard) sit in the stream-K
// region, which the separate up and down GEMMs would otherwise use.
bool fused_decode_ok(const MlpLayout& L) {
  return L.tc && L.T >= 1 && L.T <= 64 && L.reduce_mode == TP_REDUCE_SEPARATE;
}
size_t fused_decode_bytes(const MlpLayout& L) {
  return fused_decode_ok(L) ? align256(static_cast<size_t>(1 + L.p) * sizeof(int32_t)) : 0;
}

size_t up_sk_bytes(const MlpLayout& L) {
  if (L.T > kSwapMaxT || !decode_stream_k(up_tiles(L), L.T, ceil_div(L.d, 64))) return 0;
  const int64_t rows = L.p * L.R;
  auto f = [&](auto tag) {
    return tc::plan_stream_k<typename decltype(tag)::type>(rows, L.T, L.d, 1, false, num_sms()).bytes();
  };
  return L.act == TP_ACT_SWIGLU ? by_tokens<2>(L.T, f) : by_tokens<1>(L.T, f);
}
size_t down_sk_bytes(const MlpLayout& L) {
  const bool fused = L.reduce_mode == TP_REDUCE_FUSED;
  if (L.T > kSwapMaxT) return 0;   // prefill: whole pair tiles, the fused sum in the accumulator
  if (!fused && !decode_stream_k(down_tiles(L), L.T, ceil_div(L.Fsp, 64))) return 0;
  return by_tokens<1>(L.T, [&](auto tag) {
    return tc::plan_stream_k<typename decltype(tag)::type>(L.d, L.T, L.Fsp, L.p, fused, num_sms()).bytes();
  });
}

tp_status layout_of(const tp_mlp_desc* desc, MlpLayout* L) {
  if (!desc) return set_error(TP_ERR_INVALID_ARG, "desc is null");
  if (desc->T < 0) return set_error(TP_ERR_SHAPE, "T must be >= 0");
  if (desc->d < 1 || desc->d_ff < 1) return set_error(TP_ERR_SHAPE, "d and d_ff must be >= 1");
  if (desc->p < 1) return set_error(TP_ERR_SHAPE, "p must be >= 1");
  if (desc->d_ff % desc->p) return set_error(TP_ERR_SHAPE, "p must divide d_ff");
  if (desc->act < TP_ACT_IDENTITY || desc->act > TP_ACT_SWIGLU)
    return set_error(TP_ERR_INVALID_ARG, "unknown activation");
  if (desc->dtype != TP_F32 && desc->dtype != TP_BF16)
    return set_error(TP_ERR_INVALID_ARG, "dtype must be TP_F32 or TP_BF16");
  if (desc->reduce_mode != TP_REDUCE_SEPARATE && desc->reduce_mode != TP_REDUCE_FUSED)
    return set_error(TP_ERR_INVALID_ARG, "unknown reduce_mode");
  if (desc->flags & ~TP_FLAG_F32_RESIDUAL) return set_error(TP_ERR_INVALID_ARG, "unknown flags");
  L->y_dtype = (desc->flags & TP_FLAG_F32_RESIDUAL) ? TP_F32 : desc->dtype;
  L->T = desc->T; L->d = desc->d; L->F = desc->d_ff; L->p = desc->p;
  L->act = desc->act; L->dtype = desc->dtype; L->eb = elem_bytes(desc->dtype);
  L->reduce_mode = desc->reduce_mode;
  L->norm_eps = desc->norm_eps > 0.f ? desc->norm_eps : 1e-5f;
  L->tc = desc->dtype == TP_BF16 && desc->d % 8 == 0;
  L->Fs = L->F / L->p;
  L->Fsp = round_up(L->Fs, 128);
  L->R = (L->act == TP_ACT_SWIGLU) ? 2 * L->Fsp : L->Fsp;
  const int64_t P = L->p;
  L->w1p_bytes = static_cast<size_t>(P * L->R * L->d) * L->eb;
  L->w2p_bytes = static_cast<size_t>(P * L->d * L->Fsp) * L->eb;
  const size_t zb = static_cast<size_t>(L->T * P * L->R) * L->eb;
  const size_t hb = static_cast<size_t>(L->T * P * L->Fsp) * L->eb;
  const size_t partb = static_cast<size_t>(P * L->T * L->d) * 4;
  L->saved_z_off = 0;
  L->saved_h_off = align256(zb);
  L->saved_bytes = L->saved_h_off + align256(hb);
  if (L->tc) {
    // h, the stream-K region (shared by the up and down GEMMs, which run one after the other),
    // then the fp32 partials when they are reduced by a separate kernel
    L->fz_off = 0;
    L->fh_off = 0;
    L->fsk_off = align256(hb);
    const size_t sk = L->T > 0 ? std::max({up_sk_bytes(*L), down_sk_bytes(*L),
                                           fused_decode_bytes(*L)})
                               : 0;
    L->fpart_off = L->fsk_off + align256(sk);
    const size_t pb = L->reduce_mode == TP_REDUCE_FUSED ? 0 : partb;
    L->fwd_ws = L->fpart_off + align256(pb);
  } else {
    L->fz_off = 0;
    L->fh_off = align256(zb);
    L->fpart_off = L->fh_off + align256(hb);
    L->fsk_off = L->fpart_off;
    L->fwd_ws = L->fpart_off + align256(partb);
  }
  const size_t dhb = static_cast<size_t>(L->T * P * L->Fsp) * 4;
  L->bdh_off = 0;
  L->bdz_off = align256(dhb);
  L->bpart_off = L->bdz_off + align256(zb);
  L->bwd_ws = L->bpart_off + align256(partb);
  return TP_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

uint8_t* off(void* base, size_t o) { return static_cast<uint8_t*>(base) + o; }

// ------------------------------------------------------------------------------ tensor cores

tp_status tc_up(const MlpLayout& L, const void* x, const void* w1p, void* h, void* z,
                void* sk_ws, size_t sk_bytes, cudaStream_t s) {
  const int64_t rows = L.p * L.R;
  tc::EpiHidden::Params ep;
  ep.h = static_cast<__nv_bfloat16*>(h);
  ep.z = static_cast<__nv_bfloat16*>(z);
  ep.ld_h = L.p * L.Fsp;
  ep.ld_z = L.p * L.R;
  ep.tokens = static_cast<int32_t>(L.T);
  ep.rows = static_cast<int32_t>(rows);
  ep.act = L.act;
  const Operand xo{x, false, L.T, L.d, 1, L.d, 0};
  const Operand wo{w1p, false, rows, L.d, 1, L.d, 0};
  if (L.T <= kSwapMaxT) {
    // decode: weights stream once, every SM takes an equal share of their k-blocks
    ep.swap = 1;
    const tc::StreamKArgs sk{false, sk_ws, sk_bytes};
    tc::GemmOpts opt;
    opt.sk = decode_stream_k(up_tiles(L), L.T, ceil_div(L.d, 64)) ? &sk : nullptr;
    opt.rotate_k = true;
    auto f = [&](auto tag) {
      return tc::run_gemm<typename decltype(tag)::type, tc::EpiHiddenSwap>(wo, xo, rows, L.T, L.d, 1, ep,
                                                                       s, "mlp_up_gemm", opt);
    };
    return L.act == TP_ACT_SWIGLU ? by_tokens<2>(L.T, f) : by_tokens<1>(L.T, f);
  }
  ep.swap = 0;
  return tc::run_gemm_pair<PP<false, false>, tc::EpiHidden>(xo, wo, L.T, rows, L.d, 1, ep, s,
                                                            "mlp_up_gemm");
}

// Row-parallel down projection.  Separate reduce: partial[i] = h_i W2_i (fp32, [p][T][d]).
// Fused reduce: y = residual + sum_i h_i W2_i written directly (shards added in order).
tp_status tc_down(const MlpLayout& L, const void* h, const void* w2p, float* part,
                  const void* residual, void* y, void* sk_ws, size_t sk_bytes, cudaStream_t s) {
  const Operand ho{h, false, L.T, L.Fsp, L.p, L.p * L.Fsp, L.Fsp};
  const Operand wo{w2p, false, L.d, L.Fsp, L.p, L.Fsp, L.d * L.Fsp};
  const bool swap = L.T <= kSwapMaxT;
  if (L.reduce_mode == TP_REDUCE_FUSED) {
    tc::EpiReduceOut::Params ep;
    ep.out = y;
    ep.residual = residual;
    ep.ld = L.d;
    ep.rows_valid = static_cast<int32_t>(L.T);
    ep.cols_valid = static_cast<int32_t>(L.d);
    ep.out_bf16 = L.y_dtype == TP_BF16 ? 1 : 0;
    ep.swap = swap ? 1 : 0;
    const tc::StreamKArgs sk{true, sk_ws, sk_bytes};
    tc::GemmOpts opt;
    opt.sk = &sk;
    opt.rotate_k = swap;
    if (swap)
      return by_tokens<1>(L.T, [&](auto tag) {
        return tc::run_gemm<typename decltype(tag)::type, tc::EpiReduceOut>(
            wo, ho, L.d, L.T, L.Fsp, L.p, ep, s, "mlp_down_gemm", opt);
      });
    // prefill: each 256 x 256 tile runs the k-blocks of shard 0, 1, ..., p-1 into one
    // accumulator, so the shard sum never leaves TMEM
    return tc::run_gemm_pair<PP<false, false>, tc::EpiReduceOut>(ho, wo, L.T, L.d, L.Fsp, L.p, ep,
                                                                 s, "mlp_down_gemm", -1, true);
  }
  tc::EpiStoreF32::Params ep;
  ep.out = part;
  ep.ld = L.d;
  ep.batch_stride = L.T * L.d;
  ep.rows_valid = static_cast<int32_t>(L.T);
  ep.cols_valid = static_cast<int32_t>(L.d);
  if (swap) {
    ep.swap = 1;
    const tc::StreamKArgs sk{false, sk_ws, sk_bytes};
    tc::GemmOpts opt;
    opt.sk = decode_stream_k(down_tiles(L), L.T, ceil_div(L.Fsp, 64)) ? &sk : nullptr;
    opt.rotate_k = true;
    return by_tokens<1>(L.T, [&](auto tag) {
      return tc::run_gemm<typename decltype(tag)::type, tc::EpiStoreF32>(
          wo, ho, L.d, L.T, L.Fsp, L.p, ep, s, "mlp_down_gemm", opt);
    });
  }
  ep.swap = 0;
  return tc::run_gemm_pair<PP<false, false>, tc::EpiStoreF32>(ho, wo, L.T, L.d, L.Fsp, L.p, ep, s,
                                                              "mlp_down_gemm");
}

// Up and down projections of a decode call as one persistent launch (mlp_decode.cuh): h (and z
// when saved) as tc_up writes them, fp32 partials [p][T][d] as tc_down writes them.
template <int BN, int UP_SUB>
tp_status run_mlp_decode(const MlpLayout& L, const void* x, const void* w1p, const void* w2p,
                         void* h, void* z, float* part, void* counters, cudaStream_t s) {
  using C = mlpdec::Cfg<BN, UP_SUB>;
  const int64_t rows = L.p * L.R;
  const uint64_t d = static_cast<uint64_t>(L.d), Fsp = static_cast<uint64_t>(L.Fsp);
  const uint64_t P = static_cast<uint64_t>(L.p), T = static_cast<uint64_t>(L.T);
  CUtensorMap m_w1, m_x, m_w2, m_h;
  tp_status st;
  // packed W1 [p*R][d] (K-major), one box = the tile's 128 * UP_SUB rows
  if ((st = encode_tmap_bf16_3d(&m_w1, w1p, d, static_cast<uint64_t>(rows), 1, d * 2,
                                d * 2 * static_cast<uint64_t>(rows), 64, 128 * UP_SUB)) != TP_OK)
    return st;
  // x [T][d]: token rows past T read as zeros
  if ((st = encode_tmap_bf16_3d(&m_x, x, d, T, 1, d * 2, d * 2 * T, 64, BN)) != TP_OK) return st;
  // packed W2 [p][d][Fsp]
  if ((st = encode_tmap_bf16_3d(&m_w2, w2p, Fsp, d, P, Fsp * 2, d * Fsp * 2, 64, 128)) != TP_OK)
    return st;
  // h [T][p*Fsp] seen as [p][T][Fsp]: shard i's columns are its k range
  if ((st = encode_tmap_bf16_3d(&m_h, h, Fsp, T, P, P * Fsp * 2, Fsp * 2, 64, BN)) != TP_OK)
    return st;
  mlpdec::Params pr;
  pr.n_up = static_cast<int32_t>(rows / (128 * UP_SUB));
  pr.up_kb = static_cast<int32_t>(ceil_div(L.d, 64));
  pr.up_per_shard = static_cast<int32_t>(L.Fsp / 128);
  pr.dn_mb = static_cast<int32_t>(ceil_div(L.d, 128));
  pr.n_dn = static_cast<int32_t>(L.p * pr.dn_mb);
  pr.dn_kb = static_cast<int32_t>(L.Fsp / 64);
  pr.counters = static_cast<int32_t*>(counters);
  pr.err = device_error_word();
  pr.up.h = static_cast<__nv_bfloat16*>(h);
  pr.up.z = static_cast<__nv_bfloat16*>(z);
  pr.up.ld_h = L.p * L.Fsp;
  pr.up.ld_z = rows;
  pr.up.tokens = static_cast<int32_t>(L.T);
  pr.up.rows = static_cast<int32_t>(rows);
  pr.up.act = L.act;
  pr.up.swap = 1;
  pr.dn.out = part;
  pr.dn.ld = L.d;
  pr.dn.batch_stride = L.T * L.d;
  pr.dn.rows_valid = static_cast<int32_t>(L.T);
  pr.dn.cols_valid = static_cast<int32_t>(L.d);
  pr.dn.swap = 1;
  TP_LAUNCH_PDL(zero_words_kernel, dim3(1), dim3(256), 0, s, static_cast<uint32_t*>(counters),
                static_cast<int64_t>(1 + L.p));
  auto* kern = mlpdec::mlp_decode_kernel<C>;
  static int attr_set[64] = {0};
  int dev = 0;
  TP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 64 && !attr_set[dev]) {
    TP_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::SMEM_BYTES));
    attr_set[dev] = 1;
  }
  ProfScope prof(s, "mlp_decode_gemm");
  TP_LAUNCH_PDL(kern, dim3(static_cast<unsigned>(num_sms())), dim3(tc::kThreads),
                static_cast<size_t>(C::SMEM_BYTES), s, m_w1, m_x, m_w2, m_h, pr);
  return TP_OK;
}

tp_status mlp_decode(const MlpLayout& L, const void* x, const void* w1p, const void* w2p, void* h,
                     void* z, float* part, void* counters, cudaStream_t s) {
  const bool swiglu = L.act == TP_ACT_SWIGLU;
  if (L.T <= 16)
    return swiglu ? run_mlp_decode<16, 2>(L, x, w1p, w2p, h, z, part, counters, s)
                  : run_mlp_decode<16, 1>(L, x, w1p, w2p, h, z, part, counters, s);
  return swiglu ? run_mlp_decode<64, 2>(L, x, w1p, w2p, h, z, part, counters, s)
                : run_mlp_decode<64, 1>(L, x, w1p, w2p, h, z, part, counters, s);
}

// With TP_REDUCE_FUSED the dx GEMM sums the shards in its accumulator and writes dx itself
// (``dx``); otherwise it writes the fp32 partials to ``part`` for the separate reduce.
tp_status tc_backward(const MlpLayout& L, const void* dy, const void* x, const void* z,
                      const void* h, const void* w1p, const void* w2p, void* dz, float* dw1p,
                      float* dw2p, float* part, void* dx, bool dx_f32, cudaStream_t s) {
  const int64_t P = L.p;
  tp_status st;
  // (1) dH_i = dY W2_i^T with the activation backward fused: dz in w1p row order
  {
    const Operand a{dy, false, L.T, L.d, 1, L.d, 0};
    const Operand b{w2p, true, L.Fsp, L.d, P, L.Fsp, L.d * L.Fsp};
    tc::EpiActBwd::Params ep;
    ep.z = static_cast<const __nv_bfloat16*>(z);
    ep.dz = static_cast<__nv_bfloat16*>(dz);
    ep.ld = P * L.R;
    ep.R = static_cast<int32_t>(L.R);
    ep.tokens = static_cast<int32_t>(L.T);
    ep.act = L.act;
    if (L.Fsp % 256 == 0)
      st = tc::run_gemm_pair<PP<false, true>, tc::EpiActBwd>(a, b, L.T, L.Fsp, L.d, P, ep, s,
                                                             "mlp_dh_gemm");
    else
      st = tc::run_gemm<TileCfg<128, 1, false, true, stages_for(128, 1)>, tc::EpiActBwd>(
          a, b, L.T, L.Fsp, L.d, P, ep, s, "mlp_dh_gemm");
    if (st != TP_OK) return st;
  }
  // (2) dW2_i[n][c] = sum_t dY[t][n] h_i[t][c]   (no exchange between shards)
  {
    const Operand a{dy, true, L.d, L.T, 1, L.d, 0};
    const Operand b{h, true, L.Fsp, L.T, P, P * L.Fsp, L.Fsp};
    tc::EpiStoreF32::Params ep;
    ep.out = dw2p;
    ep.ld = L.Fsp;
    ep.batch_stride = L.d * L.Fsp;
    ep.rows_valid = static_cast<int32_t>(L.d);
    ep.cols_valid = static_cast<int32_t>(L.Fsp);
    ep.swap = 0;
    if (L.Fsp % 256 == 0)
      st = tc::run_gemm_pair<PP<true, true>, tc::EpiStoreF32>(a, b, L.d, L.Fsp, L.T, P, ep, s,
                                                              "mlp_dw2_gemm");
    else
      st = tc::run_gemm<TileCfg<128, 1, true, true, stages_for(128, 1)>, tc::EpiStoreF32>(
          a, b, L.d, L.Fsp, L.T, P, ep, s, "mlp_dw2_gemm");
    if (st != TP_OK) return st;
  }
  // (3) dW1_i[r][k] = sum_t dz_i[t][r] x[t][k]   (no exchange between shards)
  {
    const Operand a{dz, true, L.R, L.T, P, P * L.R, L.R};
    const Operand b{x, true, L.d, L.T, 1, L.d, 0};
    tc::EpiStoreF32::Params ep;
    ep.out = dw1p;
    ep.ld = L.d;
    ep.batch_stride = L.R * L.d;
    ep.rows_valid = static_cast<int32_t>(L.R);
    ep.cols_valid = static_cast<int32_t>(L.d);
    ep.swap = 0;
    st = tc::run_gemm_pair<PP<true, true>, tc::EpiStoreF32>(a, b, L.R, L.d, L.T, P, ep, s,
                                                            "mlp_dw1_gemm");
    if (st != TP_OK) return st;
  }
  // (4) dx_i = dz_i W1_i^T  (partials, summed by the caller; or summed here when fused)
  {
    const Operand a{dz, false, L.T, L.R, P, P * L.R, L.R};
    const Operand b{w1p, true, L.d, L.R, P, L.d, L.R * L.d};
    if (L.reduce_mode == TP_REDUCE_FUSED) {
      tc::EpiReduceOut::Params ep;
      ep.out = dx;
      ep.residual = nullptr;
      ep.ld = L.d;
      ep.rows_valid = static_cast<int32_t>(L.T);
      ep.cols_valid = static_cast<int32_t>(L.d);
      ep.out_bf16 = dx_f32 ? 0 : 1;
      ep.swap = 0;
      return tc::run_gemm_pair<PP<false, true>, tc::EpiReduceOut>(a, b, L.T, L.d, L.R, P, ep, s,
                                                                  "mlp_dx_gemm", -1, true);
    }
    tc::EpiStoreF32::Params ep;
    ep.out = part;
    ep.ld = L.d;
    ep.batch_stride = L.T * L.d;
    ep.rows_valid = static_cast<int32_t>(L.T);
    ep.cols_valid = static_cast<int32_t>(L.d);
    ep.swap = 0;
    st = tc::run_gemm_pair<PP<false, true>, tc::EpiStoreF32>(a, b, L.T, L.d, L.R, P, ep, s,
                                                             "mlp_dx_gemm");
  }
  return st;
}

// ------------------------------------------------------------------------------ SIMT path
template <typename T>
tp_status simt_forward(const MlpLayout& L, const void* x, const void* w1p, const void* w2p,
                       void* z, void* h, float* part, cudaStream_t s) {
  const int64_t P = L.p;
  simt::GemmArgs g{};
  g.a = x; g.a_bs = 0; g.a_sm = L.d; g.a_sk = 1;
  g.b = w1p; g.b_bs = 0; g.b_sm = L.d; g.b_sk = 1;
  g.out = z; g.o_bs = 0; g.o_sm = P * L.R; g.o_sn = 1;
  g.M = L.T; g.N = P * L.R; g.K = L.d; g.batch = 1; g.out_f32 = 0;
  tp_status st = simt::gemm<T>(g, s);
  if (st != TP_OK) return st;
  const int64_t total = L.T * P * L.Fsp;
  {
    ProfScope prof(s, "simt_act");
    simt::act_fwd_kernel<T><<<simt::elementwise_grid(total), 256, 0, s>>>(
        static_cast<const T*>(z), static_cast<T*>(h), L.T, L.p, L.R, L.Fsp, L.act);
    TP_LAUNCH_CHECK();
  }
  simt::GemmArgs g2{};
  g2.a = h; g2.a_bs = L.Fsp; g2.a_sm = P * L.Fsp; g2.a_sk = 1;
  g2.b = w2p; g2.b_bs = L.d * L.Fsp; g2.b_sm = L.Fsp; g2.b_sk = 1;
  g2.out = part; g2.o_bs = L.T * L.d; g2.o_sm = L.d; g2.o_sn = 1;
  g2.M = L.T; g2.N = L.d; g2.K = L.Fsp; g2.batch = P; g2.out_f32 = 1;
  return simt::gemm<T>(g2, s);
}

template <typename T>
tp_status simt_backward(const MlpLayout& L, const void* dy, const void* x, const void* z,
                        const void* h, const void* w1p, const void* w2p, float* dh, void* dz,
                        float* dw1p, float* dw2p, float* part, cudaStream_t s) {
  const int64_t P = L.p;
  tp_status st;
  simt::GemmArgs g{};
  // dH_i[t][c] = sum_n dY[t][n] w2p[i][n][c]
  g.a = dy; g.a_bs = 0; g.a_sm = L.d; g.a_sk = 1;
  g.b = w2p; g.b_bs = L.d * L.Fsp; g.b_sm = 1; g.b_sk = L.Fsp;
  g.out = dh; g.o_bs = L.Fsp; g.o_sm = P * L.Fsp; g.o_sn = 1;
  g.M = L.T; g.N = L.Fsp; g.K = L.d; g.batch = P; g.out_f32 = 1;
  if ((st = simt::gemm<T>(g, s)) != TP_OK) return st;
  const int64_t total = L.T * P * L.Fsp;
  {
    ProfScope prof(s, "simt_act_bwd");
    simt::act_bwd_kernel<T><<<simt::elementwise_grid(total), 256, 0, s>>>(
        dh, static_cast<const T*>(z), static_cast<T*>(dz), L.T, L.p, L.R, L.Fsp, L.act);
    TP_LAUNCH_CHECK();
  }
  // dW2_i[n][c] = sum_t dY[t][n] h[t][i*Fsp + c]
  g = simt::GemmArgs{};
  g.a = dy; g.a_bs = 0; g.a_sm = 1; g.a_sk = L.d;
  g.b = h; g.b_bs = L.Fsp; g.b_sm = 1; g.b_sk = P * L.Fsp;
  g.out = dw2p; g.o_bs = L.d * L.Fsp; g.o_sm = L.Fsp; g.o_sn = 1;
  g.M = L.d; g.N = L.Fsp; g.K = L.T; g.batch = P; g.out_f32 = 1;
  if ((st = simt::gemm<T>(g, s)) != TP_OK) return st;
  // dW1_i[r][k] = sum_t dz[t][i*R + r] x[t][k]
  g = simt::GemmArgs{};
  g.a = dz; g.a_bs = L.R; g.a_sm = 1; g.a_sk = P * L.R;
  g.b = x; g.b_bs = 0; g.b_sm = 1; g.b_sk = L.d;
  g.out = dw1p; g.o_bs = L.R * L.d; g.o_sm = L.d; g.o_sn = 1;
  g.M = L.R; g.N = L.d; g.K = L.T; g.batch = P; g.out_f32 = 1;
  if ((st = simt::gemm<T>(g, s)) != TP_OK) return st;
  // dx_i[t][k] = sum_r dz[t][i*R + r] w1p[i][r][k]
  g = simt::GemmArgs{};
  g.a = dz; g.a_bs = L.R; g.a_sm = P * L.R; g.a_sk = 1;
  g.b = w1p; g.b_bs = L.R * L.d; g.b_sm = 1; g.b_sk = L.d;
  g.out = part; g.o_bs = L.T * L.d; g.o_sm = L.d; g.o_sn = 1;
  g.M = L.T; g.N = L.d; g.K = L.R; g.batch = P; g.out_f32 = 1;
  return simt::gemm<T>(g, s);
}

pack::ColMap w1_colmap(const MlpLayout& L, const void* w1, const void* wu) {
  pack::ColMap cm{};
  cm.kind = L.act == TP_ACT_SWIGLU ? 1 : 0;
  cm.R = L.R;
  cm.F_s = L.Fs;
  cm.src[0] = w1; cm.src[1] = wu; cm.src[2] = nullptr;
  cm.ld[0] = L.F; cm.ld[1] = L.F; cm.ld[2] = 0;
  return cm;
}

// ``ld1`` is the row length of the user's W1 / Wu (their d_ff; larger than L.F when L is one
// shard's layout and w1 / wu / w2 already point at that shard's first column / row).
template <typename T>
tp_status pack_t(const MlpLayout& L, const void* w1, const void* wu, const void* w2, void* w1p,
                 void* w2p, cudaStream_t s, int64_t ld1 = 0) {
  const int64_t rows = L.p * L.R;
  dim3 blk(32, 8);
  dim3 g1(static_cast<unsigned>(ceil_div(rows, 32)), static_cast<unsigned>(ceil_div(L.d, 32)), 1);
  if (!pack::grid_ok(g1.x, g1.y, 1)) return set_error(TP_ERR_UNSUPPORTED, "pack grid too large");
  pack::ColMap cm = w1_colmap(L, w1, wu);
  if (ld1 > 0) cm.ld[0] = cm.ld[1] = ld1;
  pack::pack_cols_kernel<T><<<g1, blk, 0, s>>>(static_cast<T*>(w1p), rows, L.d, cm);
  TP_LAUNCH_CHECK();
  dim3 g2(static_cast<unsigned>(ceil_div(L.d, 32)), static_cast<unsigned>(ceil_div(L.Fsp, 32)),
          static_cast<unsigned>(L.p));
  if (!pack::grid_ok(g2.x, g2.y, g2.z)) return set_error(TP_ERR_UNSUPPORTED, "pack grid too large");
  pack::pack_rows_kernel<T><<<g2, blk, 0, s>>>(static_cast<T*>(w2p), L.p, L.d, L.Fsp, L.Fs,
                                               static_cast<const T*>(w2), L.d);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace
}  // namespace tp

using namespace tp;

extern "C" size_t tp_mlp_w1_packed_bytes(const tp_mlp_desc* desc) {
  MlpLayout L;
  return layout_of(desc, &L) == TP_OK ? L.w1p_bytes : 0;
}
extern "C" size_t tp_mlp_w2_packed_bytes(const tp_mlp_desc* desc) {
  MlpLayout L;
  return layout_of(desc, &L) == TP_OK ? L.w2p_bytes : 0;
}
extern "C" size_t tp_mlp_saved_bytes(const tp_mlp_desc* desc) {
  MlpLayout L;
  return layout_of(desc, &L) == TP_OK ? L.saved_bytes : 0;
}
extern "C" size_t tp_mlp_fwd_workspace(const tp_mlp_desc* desc) {
  MlpLayout L;
  return layout_of(desc, &L) == TP_OK ? L.fwd_ws : 0;
}
extern "C" size_t tp_mlp_bwd_workspace(const tp_mlp_desc* desc) {
  MlpLayout L;
  return layout_of(desc, &L) == TP_OK ? L.bwd_ws : 0;
}

extern "C" tp_status tp_mlp_pack(const tp_mlp_desc* desc, const void* w1, const void* w_up,
                                 const void* w2, void* w1p, void* w2p, void* stream) {
  clear_error();
  MlpLayout L;
  tp_status st = layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (!w1 || !w2 || !w1p || !w2p) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if ((L.act == TP_ACT_SWIGLU) != (w_up != nullptr))
    return set_error(TP_ERR_INVALID_ARG, "w_up must be given exactly for TP_ACT_SWIGLU");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return L.dtype == TP_BF16 ? pack_t<__nv_bfloat16>(L, w1, w_up, w2, w1p, w2p, s)
                            : pack_t<float>(L, w1, w_up, w2, w1p, w2p, s);
}

extern "C" tp_status tp_mlp_unpack_grads(const tp_mlp_desc* desc, const void* dw1p,
                                         const void* dw2p, void* dw1, void* dw_up, void* dw2,
                                         void* stream) {
  clear_error();
  MlpLayout L;
  tp_status st = layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (!dw1p || !dw2p || !dw1 || !dw2) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if ((L.act == TP_ACT_SWIGLU) != (dw_up != nullptr))
    return set_error(TP_ERR_INVALID_ARG, "dw_up must be given exactly for TP_ACT_SWIGLU");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t rows = L.p * L.R;
  dim3 blk(32, 8);
  dim3 g1(static_cast<unsigned>(ceil_div(rows, 32)), static_cast<unsigned>(ceil_div(L.d, 32)), 1);
  pack::unpack_cols_kernel<<<g1, blk, 0, s>>>(static_cast<const float*>(dw1p), rows, L.d,
                                               w1_colmap(L, dw1, dw_up), static_cast<float*>(dw1),
                                               static_cast<float*>(dw_up), nullptr);
  TP_LAUNCH_CHECK();
  dim3 g2(static_cast<unsigned>(ceil_div(L.d, 32)), static_cast<unsigned>(ceil_div(L.Fsp, 32)),
          static_cast<unsigned>(L.p));
  pack::unpack_rows_kernel<<<g2, blk, 0, s>>>(static_cast<const float*>(dw2p), L.p, L.d, L.Fsp,
                                               L.Fs, static_cast<float*>(dw2), L.d);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

namespace tp {
namespace {
// The forward on layout L.  ``count``: add the reduction to the counter (not for a shard's
// partial, whose reduction is the caller's collective).
tp_status mlp_forward(const MlpLayout& L, const tp_mlp_desc* desc, const void* x, const void* w1p,
                      const void* w2p, const void* residual, void* y, void* y_norm, void* saved,
                      void* workspace, size_t ws_bytes, cudaStream_t s, bool count) {
  tp_status st;
  if (desc->reduce_mode == TP_REDUCE_FUSED && !L.tc)
    return set_error(TP_ERR_UNSUPPORTED,
                     "TP_REDUCE_FUSED needs the tensor-core path (bf16, d a multiple of 8)");
  if (L.T == 0) {
    if (count) count_reduction();
    return TP_OK;
  }
  if (!x || !w1p || !w2p || !y) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (!workspace) return set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < L.fwd_ws) return set_error(TP_ERR_WORKSPACE, "workspace too small");
  void* z = saved ? off(saved, L.saved_z_off) : off(workspace, L.fz_off);
  void* h = saved ? off(saved, L.saved_h_off) : off(workspace, L.fh_off);
  float* part = reinterpret_cast<float*>(off(workspace, L.fpart_off));
  if (L.tc) {
    if (!tensor_cores_usable())
      return set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
    for (const void* q : {x, w1p, w2p, residual, static_cast<const void*>(y),
                          static_cast<const void*>(saved)})
      if (q && !aligned16(q))
        return set_error(TP_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    void* sk = off(workspace, L.fsk_off);
    const size_t skb = L.fpart_off - L.fsk_off;
    if (fused_decode_ok(L)) {
      if ((st = mlp_decode(L, x, w1p, w2p, h, saved ? z : nullptr, part, sk, s)) != TP_OK)
        return st;
    } else {
      if ((st = tc_up(L, x, w1p, h, saved ? z : nullptr, sk, skb, s)) != TP_OK) return st;
      if ((st = tc_down(L, h, w2p, part, residual, y, sk, skb, s)) != TP_OK) return st;
    }
    if (L.reduce_mode == TP_REDUCE_FUSED) {
      if (y_norm && (st = reduce::rmsnorm(y, L.y_dtype, L.T, L.d, L.norm_eps, y_norm, L.dtype, s)) != TP_OK)
        return st;
      if (count) count_reduction();
      return TP_OK;
    }
  } else if (L.dtype == TP_BF16) {
    if ((st = simt_forward<__nv_bfloat16>(L, x, w1p, w2p, z, h, part, s)) != TP_OK) return st;
  } else {
    if ((st = simt_forward<float>(L, x, w1p, w2p, z, h, part, s)) != TP_OK) return st;
  }
  st = y_norm ? reduce::reduce_norm(part, L.p, L.T, L.d, residual, y, L.y_dtype, y_norm, L.dtype,
                                    L.norm_eps, s)
              : reduce::launch(part, TP_F32, L.p, L.T * L.d, residual, y, L.y_dtype, s);
  if (st == TP_OK && count) count_reduction();
  return st;
}

// The backward on layout L; dx in L.dtype, or fp32 when ``dx_f32``.
tp_status mlp_backward(const MlpLayout& L, const void* dy, const void* x, const void* saved,
                       const void* w1p, const void* w2p, void* dx, void* dw1p, void* dw2p,
                       void* workspace, size_t ws_bytes, cudaStream_t s, bool dx_f32,
                       bool count) {
  tp_status st;
  if (!w1p || !w2p || !dw1p || !dw2p) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (L.T == 0) {  // no tokens: zero weight gradients, nothing else
    TP_CUDA_TRY(cudaMemsetAsync(dw1p, 0, static_cast<size_t>(L.p * L.R * L.d) * 4, s));
    TP_CUDA_TRY(cudaMemsetAsync(dw2p, 0, static_cast<size_t>(L.p * L.d * L.Fsp) * 4, s));
    if (count) count_reduction();
    return TP_OK;
  }
  if (!dy || !x || !saved || !dx) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (!workspace) return set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < L.bwd_ws) return set_error(TP_ERR_WORKSPACE, "workspace too small");
  const void* z = static_cast<const uint8_t*>(saved) + L.saved_z_off;
  const void* h = static_cast<const uint8_t*>(saved) + L.saved_h_off;
  float* dh = reinterpret_cast<float*>(off(workspace, L.bdh_off));
  void* dz = off(workspace, L.bdz_off);
  float* part = reinterpret_cast<float*>(off(workspace, L.bpart_off));
  float* g1 = static_cast<float*>(dw1p);
  float* g2 = static_cast<float*>(dw2p);
  if (L.tc) {
    if (!tensor_cores_usable())
      return set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
    for (const void* q : {dy, x, saved, w1p, w2p, static_cast<const void*>(dx)})
      if (!aligned16(q)) return set_error(TP_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    st = tc_backward(L, dy, x, z, h, w1p, w2p, dz, g1, g2, part, dx, dx_f32, s);
    if (st == TP_OK && L.reduce_mode == TP_REDUCE_FUSED) {   // dx already summed
      if (count) count_reduction();
      return TP_OK;
    }
  } else if (L.dtype == TP_BF16) {
    st = simt_backward<__nv_bfloat16>(L, dy, x, z, h, w1p, w2p, dh, dz, g1, g2, part, s);
  } else {
    st = simt_backward<float>(L, dy, x, z, h, w1p, w2p, dh, dz, g1, g2, part, s);
  }
  if (st != TP_OK) return st;
  st = reduce::launch(part, TP_F32, L.p, L.T * L.d, nullptr, dx, dx_f32 ? TP_F32 : L.dtype, s);
  if (st == TP_OK && count) count_reduction();
  return st;
}
}  // namespace
}  // namespace tp

extern "C" tp_status tp_mlp_fwd(const tp_mlp_desc* desc, const void* x, const void* w1p,
                                const void* w2p, const void* residual, void* y, void* y_norm,
                                void* saved, void* workspace, size_t ws_bytes, void* stream) {
  clear_error();
  MlpLayout L;
  tp_status st = layout_of(desc, &L);
  if (st != TP_OK) return st;
  return mlp_forward(L, desc, x, w1p, w2p, residual, y, y_norm, saved, workspace, ws_bytes,
                     static_cast<cudaStream_t>(stream), true);
}

extern "C" tp_status tp_mlp_bwd(const tp_mlp_desc* desc, const void* dy, const void* x,
                                const void* saved, const void* w1p, const void* w2p, void* dx,
                                void* dw1p, void* dw2p, void* workspace, size_t ws_bytes,
                                void* stream) {
  clear_error();
  MlpLayout L;
  tp_status st = layout_of(desc, &L);
  if (st != TP_OK) return st;
  return mlp_backward(L, dy, x, saved, w1p, w2p, dx, dw1p, dw2p, workspace, ws_bytes,
                      static_cast<cudaStream_t>(stream), false, true);
}

// ------------------------------------------------------------------------ one shard per device
// "Tensor Parallelism" (klaylearn), Notes, and "How does tensor parallelism split a transformer
// feed-forward block's two matmuls", "One collective": with one shard per GPU, device i holds
// the column slice W1_i (and Wu_i) and the row slice W2_i, computes h_i = act(x W1_i) and the
// full-shape partial y_i = h_i W2_i, and the devices' all-reduce adds the partials.  Shard i on
// its own is the block with p = 1 and d_ff / p features, whose packed layout is exactly shard i's
// slice of the p-shard packing; these calls run that problem and leave the sum to the caller's
// collective (so they add nothing to the reduction counter).
namespace tp {
namespace {
tp_status shard_desc_of(const tp_mlp_desc* desc, int32_t shard, int32_t partial_dtype,
                        tp_mlp_desc* sd, MlpLayout* LS) {
  MlpLayout L;
  tp_status st = layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (shard < 0 || shard >= L.p) return set_error(TP_ERR_INVALID_ARG, "shard must be in 0 .. p-1");
  if (partial_dtype != TP_F32 && partial_dtype != TP_BF16)
    return set_error(TP_ERR_INVALID_ARG, "partial_dtype must be TP_F32 or TP_BF16");
  if (L.dtype == TP_F32 && partial_dtype != TP_F32)
    return set_error(TP_ERR_UNSUPPORTED, "fp32 blocks give fp32 partials");
  if (desc->flags != 0)
    return set_error(TP_ERR_INVALID_ARG, "shard calls take no flags (partial_dtype sets the type)");
  *sd = *desc;
  sd->d_ff = L.Fs;
  sd->p = 1;
  sd->flags = (L.dtype == TP_BF16 && partial_dtype == TP_F32) ? TP_FLAG_F32_RESIDUAL : 0;
  sd->reduce_mode = L.tc ? TP_REDUCE_FUSED : TP_REDUCE_SEPARATE;
  return layout_of(sd, LS);
}
}  // namespace
}  // namespace tp

extern "C" tp_status tp_mlp_shard_sizes(const tp_mlp_desc* desc, int32_t partial_dtype,
                                        tp_shard_sizes* out) {
  clear_error();
  if (!out) return set_error(TP_ERR_INVALID_ARG, "out is null");
  tp_mlp_desc sd;
  MlpLayout L;
  tp_status st = shard_desc_of(desc, 0, partial_dtype, &sd, &L);
  if (st != TP_OK) return st;
  out->col_weight_bytes = L.w1p_bytes;
  out->row_weight_bytes = L.w2p_bytes;
  out->saved_bytes = L.saved_bytes;
  out->fwd_workspace = L.fwd_ws;
  out->bwd_workspace = L.bwd_ws;
  out->partial_bytes = static_cast<size_t>(L.T * L.d) * elem_bytes(partial_dtype);
  return TP_OK;
}

extern "C" tp_status tp_mlp_pack_shard(const tp_mlp_desc* desc, int32_t shard, const void* w1,
                                       const void* w_up, const void* w2, void* w1p_shard,
                                       void* w2p_shard, void* stream) {
  clear_error();
  tp_mlp_desc sd;
  MlpLayout L;
  tp_status st = shard_desc_of(desc, shard, desc ? desc->dtype : TP_F32, &sd, &L);
  if (st != TP_OK) return st;
  if (!w1 || !w2 || !w1p_shard || !w2p_shard) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if ((L.act == TP_ACT_SWIGLU) != (w_up != nullptr))
    return set_error(TP_ERR_INVALID_ARG, "w_up must be given exactly for TP_ACT_SWIGLU");
  // shard i's first column of W1 / Wu and first row of W2 in the user's full matrices
  const int64_t col0 = static_cast<int64_t>(shard) * L.Fs;
  const size_t eb = static_cast<size_t>(L.eb);
  const uint8_t* w1s = static_cast<const uint8_t*>(w1) + col0 * eb;
  const uint8_t* wus = w_up ? static_cast<const uint8_t*>(w_up) + col0 * eb : nullptr;
  const uint8_t* w2s = static_cast<const uint8_t*>(w2) + col0 * L.d * eb;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return L.dtype == TP_BF16
             ? pack_t<__nv_bfloat16>(L, w1s, wus, w2s, w1p_shard, w2p_shard, s, desc->d_ff)
             : pack_t<float>(L, w1s, wus, w2s, w1p_shard, w2p_shard, s, desc->d_ff);
}

extern "C" tp_status tp_mlp_fwd_shard(const tp_mlp_desc* desc, int32_t shard,
                                      int32_t partial_dtype, const void* x, const void* w1p_shard,
                                      const void* w2p_shard, void* partial, void* saved_shard,
                                      void* workspace, size_t ws_bytes, void* stream) {
  clear_error();
  tp_mlp_desc sd;
  MlpLayout L;
  tp_status st = shard_desc_of(desc, shard, partial_dtype, &sd, &L);
  if (st != TP_OK) return st;
  return mlp_forward(L, &sd, x, w1p_shard, w2p_shard, nullptr, partial, nullptr, saved_shard,
                     workspace, ws_bytes, static_cast<cudaStream_t>(stream), false);
}

extern "C" tp_status tp_mlp_bwd_shard(const tp_mlp_desc* desc, int32_t shard,
                                      int32_t partial_dtype, const void* dy, const void* x,
                                      const void* saved_shard, const void* w1p_shard,
                                      const void* w2p_shard, void* dx_partial, void* dw1p_shard,
                                      void* dw2p_shard, void* workspace, size_t ws_bytes,
                                      void* stream) {
  clear_error();
  tp_mlp_desc sd;
  MlpLayout L;
  tp_status st = shard_desc_of(desc, shard, partial_dtype, &sd, &L);
  if (st != TP_OK) return st;
  return mlp_backward(L, dy, x, saved_shard, w1p_shard, w2p_shard, dx_partial, dw1p_shard,
                      dw2p_shard, workspace, ws_bytes, static_cast<cudaStream_t>(stream),
                      partial_dtype == TP_F32, false);
}

// ------------------------------------------------------------------ sequence-parallel variant
// "Why tensor parallelism has to stay in scale-up" (Keysight), "Where the 320 comes from": with
// sequence parallelism the block's all-reduce becomes a reduce-scatter of the partials into the
// shards' token slices (residual add and norm then run on the slices) and an all-gather of the
// slices before the column-parallel GEMM.  Backward: the all-gather's gradient is a
// reduce-scatter (dx) and the reduce-scatter's an all-gather (dy).
namespace {
size_t act_bytes(const MlpLayout& L) { return align256(static_cast<size_t>(L.T * L.d) * L.eb); }

tp_status sp_layout(const tp_mlp_desc* desc, MlpLayout* L) {
  tp_status st = layout_of(desc, L);
  if (st != TP_OK) return st;
  if (desc->reduce_mode != TP_REDUCE_SEPARATE)
    return set_error(TP_ERR_UNSUPPORTED,
                     "the sequence-parallel calls reduce-scatter the partials: use TP_REDUCE_SEPARATE");
  if (L->p > seqpar::kMaxSlices) return set_error(TP_ERR_SHAPE, "p must be <= 64 for slices");
  if (L->T % L->p) return set_error(TP_ERR_SHAPE, "sequence parallelism needs p to divide T");
  return TP_OK;
}
}  // namespace

extern "C" size_t tp_mlp_fwd_sp_workspace(const tp_mlp_desc* desc) {
  MlpLayout L;
  if (sp_layout(desc, &L) != TP_OK) return 0;
  return act_bytes(L) + L.fwd_ws;
}

extern "C" tp_status tp_mlp_fwd_sp(const tp_mlp_desc* desc, const void* const* x_slices,
                                   const void* w1p, const void* w2p,
                                   void* const* residual_slices, void* const* y_slices,
                                   void* const* y_norm_slices, void* saved, void* workspace,
                                   size_t ws_bytes, void* stream) {
  clear_error();
  MlpLayout L;
  tp_status st = sp_layout(desc, &L);
  if (st != TP_OK) return st;
  if (L.T == 0) {
    count_reduction();
    return TP_OK;
  }
  void* const* xs = const_cast<void* const*>(x_slices);
  if ((st = seqpar::check_slices(L.p, L.T, xs, "x_slices")) != TP_OK) return st;
  if ((st = seqpar::check_slices(L.p, L.T, y_slices, "y_slices")) != TP_OK) return st;
  if (residual_slices && (st = seqpar::check_slices(L.p, L.T, residual_slices, "residual_slices")) != TP_OK)
    return st;
  if (y_norm_slices && (st = seqpar::check_slices(L.p, L.T, y_norm_slices, "y_norm_slices")) != TP_OK)
    return st;
  if (!w1p || !w2p) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (!workspace) return set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < act_bytes(L) + L.fwd_ws) return set_error(TP_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* x = workspace;                        // the gathered [T][d] input
  void* ws = off(workspace, act_bytes(L));    // the forward's own workspace
  void* z = saved ? off(saved, L.saved_z_off) : off(ws, L.fz_off);
  void* h = saved ? off(saved, L.saved_h_off) : off(ws, L.fh_off);
  float* part = reinterpret_cast<float*>(off(ws, L.fpart_off));
  if ((st = seqpar::all_gather(x_slices, L.p, (L.T / L.p) * L.d * L.eb, x, s)) != TP_OK) return st;
  if (L.tc) {
    if (!tensor_cores_usable())
      return set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
    for (const void* q : {w1p, w2p, static_cast<const void*>(saved)})
      if (q && !aligned16(q)) return set_error(TP_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    void* sk = off(ws, L.fsk_off);
    const size_t skb = L.fpart_off - L.fsk_off;
    if (fused_decode_ok(L)) {
      if ((st = mlp_decode(L, x, w1p, w2p, h, saved ? z : nullptr, part, sk, s)) != TP_OK)
        return st;
    } else {
      if ((st = tc_up(L, x, w1p, h, saved ? z : nullptr, sk, skb, s)) != TP_OK) return st;
      if ((st = tc_down(L, h, w2p, part, nullptr, nullptr, sk, skb, s)) != TP_OK) return st;
    }
  } else if (L.dtype == TP_BF16) {
    if ((st = simt_forward<__nv_bfloat16>(L, x, w1p, w2p, z, h, part, s)) != TP_OK) return st;
  } else {
    if ((st = simt_forward<float>(L, x, w1p, w2p, z, h, part, s)) != TP_OK) return st;
  }
  st = seqpar::reduce_scatter(part, L.p, L.T, L.d, residual_slices, y_slices, L.y_dtype,
                              y_norm_slices, L.dtype, L.norm_eps, s);
  if (st == TP_OK) count_reduction();
  return st;
}

extern "C" size_t tp_mlp_bwd_sp_workspace(const tp_mlp_desc* desc) {
  MlpLayout L;
  if (sp_layout(desc, &L) != TP_OK) return 0;
  return 2 * act_bytes(L) + L.bwd_ws;
}

extern "C" tp_status tp_mlp_bwd_sp(const tp_mlp_desc* desc, const void* const* dy_slices,
                                   const void* const* x_slices, const void* saved,
                                   const void* w1p, const void* w2p, void* const* dx_slices,
                                   void* dw1p, void* dw2p, void* workspace, size_t ws_bytes,
                                   void* stream) {
  clear_error();
  MlpLayout L;
  tp_status st = sp_layout(desc, &L);
  if (st != TP_OK) return st;
  if (!w1p || !w2p || !dw1p || !dw2p) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L.T == 0) {
    TP_CUDA_TRY(cudaMemsetAsync(dw1p, 0, static_cast<size_t>(L.p * L.R * L.d) * 4, s));
    TP_CUDA_TRY(cudaMemsetAsync(dw2p, 0, static_cast<size_t>(L.p * L.d * L.Fsp) * 4, s));
    count_reduction();
    return TP_OK;
  }
  if ((st = seqpar::check_slices(L.p, L.T, const_cast<void* const*>(dy_slices), "dy_slices")) != TP_OK ||
      (st = seqpar::check_slices(L.p, L.T, const_cast<void* const*>(x_slices), "x_slices")) != TP_OK ||
      (st = seqpar::check_slices(L.p, L.T, dx_slices, "dx_slices")) != TP_OK)
    return st;
  if (!saved) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (!workspace) return set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < 2 * act_bytes(L) + L.bwd_ws) return set_error(TP_ERR_WORKSPACE, "workspace too small");
  void* dy = workspace;
  void* x = off(workspace, act_bytes(L));
  void* ws = off(workspace, 2 * act_bytes(L));
  const int64_t slice_bytes = (L.T / L.p) * L.d * L.eb;
  if ((st = seqpar::all_gather(dy_slices, L.p, slice_bytes, dy, s)) != TP_OK) return st;
  if ((st = seqpar::all_gather(x_slices, L.p, slice_bytes, x, s)) != TP_OK) return st;
  const void* z = static_cast<const uint8_t*>(saved) + L.saved_z_off;
  const void* h = static_cast<const uint8_t*>(saved) + L.saved_h_off;
  float* dh = reinterpret_cast<float*>(off(ws, L.bdh_off));
  void* dz = off(ws, L.bdz_off);
  float* part = reinterpret_cast<float*>(off(ws, L.bpart_off));
  float* g1 = static_cast<float*>(dw1p);
  float* g2 = static_cast<float*>(dw2p);
  if (L.tc) {
    if (!tensor_cores_usable())
      return set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
    for (const void* q : {saved, w1p, w2p})
      if (!aligned16(q)) return set_error(TP_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    st = tc_backward(L, dy, x, z, h, w1p, w2p, dz, g1, g2, part, nullptr, false, s);
  } else if (L.dtype == TP_BF16) {
    st = simt_backward<__nv_bfloat16>(L, dy, x, z, h, w1p, w2p, dh, dz, g1, g2, part, s);
  } else {
    st = simt_backward<float>(L, dy, x, z, h, w1p, w2p, dh, dz, g1, g2, part, s);
  }
  if (st != TP_OK) return st;
  st = seqpar::reduce_scatter(part, L.p, L.T, L.d, nullptr, dx_slices, L.dtype, nullptr, L.dtype,
                              L.norm_eps, s);
  if (st == TP_OK) count_reduction();
  return st;
}

// ------------------------------------------------------------------ mixture of experts
// "Tensor-parallel all-reduce count per transformer layer in MLX shard_linear" (llms-explorer),
// facts on MoE layers: replicated router, routed and shared experts sharded in place, one
// block-level sum, bias once after the sum.  Every expert is a SwiGLU block packed exactly like
// the dense MLP (tp_mlp_pack's layout for d, d_ff, p); the E experts' packings lie back to back.
namespace {
struct MoeLayout {
  int64_t T, d, F, Fsh, n_rows;
  int E, k, p;
  MlpLayout ex;       // one routed expert as an MLP block (T = routed rows)
  MlpLayout sh;       // the shared expert over the T tokens (valid when Fsh > 0)
  size_t logits_off, idx_off, w_off, cnt_off, off_off, mbp_off, perm_off, inv_off, xs_off,
      hs_off, part_off, shared_off, shared_y_off, bytes;
};

tp_status moe_layout(const tp_moe_desc* desc, MoeLayout* M) {
  if (!desc) return set_error(TP_ERR_INVALID_ARG, "desc is null");
  if (desc->dtype != TP_BF16) return set_error(TP_ERR_UNSUPPORTED, "the MoE block is bf16");
  if (desc->flags != 0) return set_error(TP_ERR_INVALID_ARG, "unknown flags");
  if (desc->T < 0 || desc->d < 8 || desc->d % 8) return set_error(TP_ERR_SHAPE, "T >= 0, d a multiple of 8");
  if (desc->n_experts < 1 || desc->n_experts % 8 || (desc->n_experts % 64 && desc->n_experts > 256))
    return set_error(TP_ERR_SHAPE, "n_experts: a multiple of 8, and of 64 above 256");
  if (desc->top_k < 1 || desc->top_k > moe::kMaxTopK || desc->top_k > desc->n_experts)
    return set_error(TP_ERR_SHAPE, "top_k must be 1..8 and <= n_experts");
  if (desc->d_ff_shared < 0) return set_error(TP_ERR_SHAPE, "d_ff_shared must be >= 0");
  M->T = desc->T; M->d = desc->d; M->F = desc->d_ff; M->Fsh = desc->d_ff_shared;
  M->E = desc->n_experts; M->k = desc->top_k; M->p = desc->p;
  M->n_rows = M->T * M->k;
  if (M->n_rows > INT32_MAX) return set_error(TP_ERR_UNSUPPORTED, "too many routed rows");
  tp_mlp_desc me{M->n_rows, M->d, M->F, M->p, TP_ACT_SWIGLU, TP_BF16, TP_REDUCE_SEPARATE, 0, 0.f};
  tp_status st = layout_of(&me, &M->ex);
  if (st != TP_OK) return st;
  if (M->Fsh > 0) {
    // the shared expert's shard sum is fused into its down GEMM, written as fp32
    tp_mlp_desc ms{M->T, M->d, M->Fsh, M->p, TP_ACT_SWIGLU, TP_BF16, TP_REDUCE_FUSED,
                   TP_FLAG_F32_RESIDUAL, 0.f};
    if ((st = layout_of(&ms, &M->sh)) != TP_OK) return st;
  }
  size_t o = 0;
  auto take = [&](size_t& field, size_t bytes) {
    field = o;
    o += align256(bytes);
  };
  const size_t R = static_cast<size_t>(M->n_rows);
  take(M->logits_off, static_cast<size_t>(M->T) * M->E * 4);
  take(M->idx_off, R * 4);
  take(M->w_off, R * 4);
  take(M->cnt_off, static_cast<size_t>(M->E) * 4);
  take(M->off_off, static_cast<size_t>(M->E) * 4);
  take(M->mbp_off, static_cast<size_t>(M->E + 1) * 4);
  take(M->perm_off, R * 4);
  take(M->inv_off, R * 4);
  take(M->xs_off, R * M->d * 2);
  take(M->hs_off, R * M->p * M->ex.Fsp * 2);
  take(M->part_off, R * M->d * 4);            // routed rows, the shards already summed
  take(M->shared_off, M->Fsh > 0 ? M->sh.fwd_ws : 0);
  take(M->shared_y_off, M->Fsh > 0 ? static_cast<size_t>(M->T) * M->d * 4 : 0);
  M->bytes = o;
  return TP_OK;
}
}  // namespace

extern "C" size_t tp_moe_expert_w1_bytes(const tp_moe_desc* desc) {
  MoeLayout M;
  return moe_layout(desc, &M) == TP_OK ? M.ex.w1p_bytes : 0;
}
extern "C" size_t tp_moe_expert_w2_bytes(const tp_moe_desc* desc) {
  MoeLayout M;
  return moe_layout(desc, &M) == TP_OK ? M.ex.w2p_bytes : 0;
}
extern "C" size_t tp_moe_shared_w1_bytes(const tp_moe_desc* desc) {
  MoeLayout M;
  return moe_layout(desc, &M) == TP_OK && M.Fsh > 0 ? M.sh.w1p_bytes : 0;
}
extern "C" size_t tp_moe_shared_w2_bytes(const tp_moe_desc* desc) {
  MoeLayout M;
  return moe_layout(desc, &M) == TP_OK && M.Fsh > 0 ? M.sh.w2p_bytes : 0;
}
extern "C" size_t tp_moe_fwd_workspace(const tp_moe_desc* desc) {
  MoeLayout M;
  return moe_layout(desc, &M) == TP_OK ? M.bytes : 0;
}

extern "C" tp_status tp_moe_pack(const tp_moe_desc* desc, const void* const* wg,
                                 const void* const* wu, const void* const* w2, const void* wg_s,
                                 const void* wu_s, const void* w2_s, void* w1p, void* w2p,
                                 void* w1p_s, void* w2p_s, void* stream) {
  clear_error();
  MoeLayout M;
  tp_status st = moe_layout(desc, &M);
  if (st != TP_OK) return st;
  if (!wg || !wu || !w2 || !w1p || !w2p) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int e = 0; e < M.E; ++e) {
    if (!wg[e] || !wu[e] || !w2[e]) return set_error(TP_ERR_INVALID_ARG, "null expert weight");
    if ((st = pack_t<__nv_bfloat16>(M.ex, wg[e], wu[e], w2[e], off(w1p, e * M.ex.w1p_bytes),
                                    off(w2p, e * M.ex.w2p_bytes), s)) != TP_OK)
      return st;
  }
  if (M.Fsh > 0) {
    if (!wg_s || !wu_s || !w2_s || !w1p_s || !w2p_s)
      return set_error(TP_ERR_INVALID_ARG, "the shared expert's weights are null");
    return pack_t<__nv_bfloat16>(M.sh, wg_s, wu_s, w2_s, w1p_s, w2p_s, s);
  }
  return TP_OK;
}

// Steps (1)-(6) of the forward: router logits, top-k routing, dispatch (counts, stable
// positions, gather) and the two grouped expert GEMMs, in M's workspace regions; the routing goes
// to idx / wts, the routed rows' outputs (shards summed) to the part region, and with ``zs`` the
// routed rows' gate/up pre-activations ([row][p R], as the dense MLP saves them) to zs.
tp_status moe_routed(const MoeLayout& M, const void* x, const void* wr, const void* w1p,
                     const void* w2p, void* workspace, int32_t* idx, float* wts, void* zs,
                     cudaStream_t s) {
  tp_status st;
  float* logits = reinterpret_cast<float*>(off(workspace, M.logits_off));
  int32_t* cnt = reinterpret_cast<int32_t*>(off(workspace, M.cnt_off));
  int32_t* offs = reinterpret_cast<int32_t*>(off(workspace, M.off_off));
  int32_t* mbp = reinterpret_cast<int32_t*>(off(workspace, M.mbp_off));
  int32_t* perm = reinterpret_cast<int32_t*>(off(workspace, M.perm_off));
  int32_t* inv = reinterpret_cast<int32_t*>(off(workspace, M.inv_off));
  auto* xs = reinterpret_cast<__nv_bfloat16*>(off(workspace, M.xs_off));
  auto* hs = reinterpret_cast<__nv_bfloat16*>(off(workspace, M.hs_off));
  float* part = reinterpret_cast<float*>(off(workspace, M.part_off));
  const MlpLayout& L = M.ex;
  // (1) router logits = x Wr (Wr [d][E] read MN-major), fp32: on the tensor cores when Wr's rows
  // are whole 16-byte units (E a multiple of 8; the 64-wide loads past E read zeros and the
  // epilogue writes the E valid columns), else one block per token on the SIMT core
  if (M.E % 8) {
    ProfScope prof(s, "moe_router");
    const int threads = (256 / M.E) * M.E;
    TP_LAUNCH_PDL(moe::router_simt_kernel, dim3(static_cast<unsigned>(M.T)), dim3(threads), 0, s,
                  static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(wr),
                  M.d, M.E, logits);
  } else {
    const Operand xo{x, false, M.T, M.d, 1, M.d, 0};
    const Operand ro{wr, true, M.E, M.d, 1, M.E, 0};
    tc::EpiStoreF32::Params ep;
    ep.out = logits;
    ep.ld = M.E;
    ep.batch_stride = 0;
    ep.rows_valid = static_cast<int32_t>(M.T);
    ep.cols_valid = M.E;
    ep.swap = 0;
    st = M.E <= 64 ? tc::run_gemm<TileCfg<64, 1, false, true, stages_for(64, 1)>, tc::EpiStoreF32>(
                         xo, ro, M.T, M.E, M.d, 1, ep, s, "moe_router")
                   : tc::run_gemm<TileCfg<128, 1, false, true, stages_for(128, 1)>, tc::EpiStoreF32>(
                         xo, ro, M.T, M.E, M.d, 1, ep, s, "moe_router");
    if (st != TP_OK) return st;
  }
  // (2) top-k and weights; (3) per-expert counts, offsets and stable positions; (4) gather
  {
    ProfScope prof(s, "moe_route");
    TP_LAUNCH_PDL(moe::topk_kernel, dim3(static_cast<unsigned>(ceil_div(M.T, 8))), dim3(256), 0,
                  s, logits, M.T, M.E, M.k, idx, wts);
    TP_LAUNCH_PDL(moe::count_kernel, dim3(static_cast<unsigned>(M.E)), dim3(1024), 0, s,
                  static_cast<const int32_t*>(idx), M.n_rows, cnt);
    TP_LAUNCH_PDL(moe::position_kernel, dim3(static_cast<unsigned>(M.E)), dim3(1024), 0, s,
                  static_cast<const int32_t*>(idx), M.n_rows, static_cast<const int32_t*>(cnt), 128,
                  offs, mbp, perm, inv);
    TP_LAUNCH_PDL(moe::gather_kernel,
                  dim3(static_cast<unsigned>(ceil_div(M.n_rows, moe::kGatherRowsPerBlock))),
                  dim3(32 * moe::kGatherRowsPerBlock), 0, s, static_cast<const __nv_bfloat16*>(x),
                  static_cast<const int32_t*>(perm), M.k, M.d, M.n_rows, xs);
  }
  // (5) grouped up GEMM + SwiGLU over all experts: rows of expert e are xs[off[e] .. +cnt[e]).
  // Swapped: each tile is 256 packed rows of one expert's W1 (128 gate + 128 up features) times
  // up to 128 of its routed rows, the MMA width cut to that block's rows rounded up to 16, so an
  // expert's last block costs its rows rather than a full tile.
  {
    const int64_t rows = L.p * L.R;
    tc::EpiHiddenParams ep;
    ep.h = hs;
    ep.z = static_cast<__nv_bfloat16*>(zs);
    ep.ld_h = L.p * L.Fsp;
    ep.ld_z = zs ? rows : 0;
    ep.tokens = static_cast<int32_t>(M.n_rows);
    ep.rows = static_cast<int32_t>(rows);
    ep.act = TP_ACT_SWIGLU;
    ep.swap = 1;
    const Operand wo{w1p, false, rows, M.d, M.E, M.d, rows * M.d};
    const Operand xo{xs, false, M.n_rows, M.d, 1, M.d, 0};
    tc::GemmOpts opt;
    opt.grp_cnt = cnt;
    opt.grp_off = offs;
    opt.grp_mbp = mbp;
    opt.grp_n = M.E;
    opt.grp_div = 1;
    opt.grp_swap = true;
    st = tc::run_gemm<TileCfg<128, 2, false, false, stages_for(128, 2)>, tc::EpiHiddenSwap>(
        wo, xo, rows, M.T, M.d, M.E, ep, s, "moe_up_gemm", opt);
    if (st != TP_OK) return st;
  }
  // (6) grouped down GEMM: problem e * p + i = expert e, shard i; each tile runs shard 0..p-1's
  // k-blocks into one accumulator, so the routed rows leave with their shards summed: [row][d].
  // Swapped like the up GEMM: 256 rows of W2 (output features, two 128-row MMAs) times up to 128
  // routed rows.
  {
    const Operand ho{hs, false, M.n_rows, L.Fsp, L.p, L.p * L.Fsp, L.Fsp};
    const Operand wo{w2p, false, M.d, L.Fsp, static_cast<int64_t>(M.E) * L.p, L.Fsp, M.d * L.Fsp};
    tc::EpiStoreF32::Params ep;
    ep.out = part;
    ep.ld = M.d;
    ep.batch_stride = 0;
    ep.rows_valid = static_cast<int32_t>(M.n_rows);
    ep.cols_valid = static_cast<int32_t>(M.d);
    ep.swap = 1;
    tc::GemmOpts opt;
    opt.grp_cnt = cnt;
    opt.grp_off = offs;
    opt.grp_mbp = mbp;
    opt.grp_n = M.E;
    opt.grp_div = L.p;
    opt.grp_sum = true;
    opt.grp_swap = true;
    st = tc::run_gemm<TileCfg<128, 2, false, false, stages_for(128, 2)>, tc::EpiStoreF32>(
        wo, ho, M.d, M.T, L.Fsp, static_cast<int64_t>(M.E) * L.p, ep, s, "moe_down_gemm", opt);
    if (st != TP_OK) return st;
  }
  return TP_OK;
}

extern "C" tp_status tp_moe_fwd(const tp_moe_desc* desc, const void* x, const void* wr,
                                const void* w1p, const void* w2p, const void* w1p_s,
                                const void* w2p_s, const void* bias, const void* residual,
                                void* y, void* route_idx, void* route_w, void* workspace,
                                size_t ws_bytes, void* stream) {
  clear_error();
  MoeLayout M;
  tp_status st = moe_layout(desc, &M);
  if (st != TP_OK) return st;
  if (M.T == 0) {
    count_reduction();
    return TP_OK;
  }
  if (!x || !wr || !w1p || !w2p || !y) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (M.Fsh > 0 && (!w1p_s || !w2p_s))
    return set_error(TP_ERR_INVALID_ARG, "the shared expert's packed weights are null");
  for (const void* q : {x, wr, w1p, w2p, w1p_s, w2p_s, bias, residual, static_cast<const void*>(y)})
    if (q && !aligned16(q)) return set_error(TP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!workspace) return set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < M.bytes) return set_error(TP_ERR_WORKSPACE, "workspace too small");
  if (!tensor_cores_usable())
    return set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* idx = route_idx ? static_cast<int32_t*>(route_idx)
                           : reinterpret_cast<int32_t*>(off(workspace, M.idx_off));
  float* wts = route_w ? static_cast<float*>(route_w) : reinterpret_cast<float*>(off(workspace, M.w_off));
  if ((st = moe_routed(M, x, wr, w1p, w2p, workspace, idx, wts, nullptr, s)) != TP_OK) return st;
  int32_t* inv = reinterpret_cast<int32_t*>(off(workspace, M.inv_off));
  float* part = reinterpret_cast<float*>(off(workspace, M.part_off));
  // (7) the shared expert over all tokens, its p shards summed in its down GEMM: [T][d] fp32
  const float* shared_sum = nullptr;
  if (M.Fsh > 0) {
    void* ws = off(workspace, M.shared_off);
    void* h = off(ws, M.sh.fh_off);
    float* sy = reinterpret_cast<float*>(off(workspace, M.shared_y_off));
    void* sk = off(ws, M.sh.fsk_off);
    const size_t skb = M.sh.fpart_off - M.sh.fsk_off;
    if ((st = tc_up(M.sh, x, w1p_s, h, nullptr, sk, skb, s)) != TP_OK) return st;
    if ((st = tc_down(M.sh, h, w2p_s, nullptr, nullptr, sy, sk, skb, s)) != TP_OK) return st;
    shared_sum = sy;
  }
  // (8) the block's sum: shared expert + the weighted routed rows (choices in order), bias
  // once, residual
  {
    ProfScope prof(s, "moe_combine");
    const int64_t nv = M.T * (M.d / 8);
    const int64_t blocks = std::min<int64_t>(ceil_div(nv, 256), static_cast<int64_t>(num_sms()) * 8);
    TP_LAUNCH_PDL(moe::combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                  static_cast<const float*>(part), shared_sum, static_cast<const int32_t*>(inv),
                  static_cast<const float*>(wts), M.k, M.T, M.d,
                  static_cast<const __nv_bfloat16*>(bias),
                  static_cast<const __nv_bfloat16*>(residual), static_cast<__nv_bfloat16*>(y));
  }
  count_reduction();
  return TP_OK;
}

// ------------------------------------------------------------------ MoE backward
namespace {
// Streams on which the routed experts' backward GEMMs run side by side (created once per
// device, non-blocking; forked from and joined back to the caller's stream with events).
constexpr int kMoeStreams = 8;
tp_status moe_streams(cudaStream_t (&out)[kMoeStreams]) {
  static cudaStream_t pool[64][kMoeStreams] = {};
  int dev = 0;
  TP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 64) return set_error(TP_ERR_UNSUPPORTED, "device index above 63");
  for (int j = 0; j < kMoeStreams; ++j) {
    if (!pool[dev][j]) TP_CUDA_TRY(cudaStreamCreateWithFlags(&pool[dev][j], cudaStreamNonBlocking));
    out[j] = pool[dev][j];
  }
  return TP_OK;
}

// Backward workspace: the forward's regions, then the backward's own.
struct MoeBwdLayout {
  size_t zs_off, dw_off, dl_off, dxr_off, gs_off, dz_off, dxs_off, zsh_off, hsh_off, dzs_off,
      dxsh_off, bytes;
};
MoeBwdLayout moe_bwd_layout(const MoeLayout& M) {
  MoeBwdLayout B;
  size_t o = M.bytes;
  auto take = [&](size_t& field, size_t bytes) {
    field = o;
    o += align256(bytes);
  };
  const size_t R = static_cast<size_t>(M.n_rows), T = static_cast<size_t>(M.T);
  const size_t d = static_cast<size_t>(M.d);
  const size_t zrow = static_cast<size_t>(M.ex.p * M.ex.R);
  take(B.zs_off, R * zrow * 2);       // routed rows' gate/up pre-activations
  take(B.dw_off, R * 4);              // routing-weight gradients [T][k]
  take(B.dl_off, T * M.E * 2);        // router-logit gradients [T][E] bf16
  take(B.dxr_off, T * d * 4);         // dx through the router
  take(B.gs_off, R * d * 2);          // w * dy per routed row, expert order
  take(B.dz_off, R * zrow * 2);       // dz of the expert being differentiated
  take(B.dxs_off, R * d * 4);         // routed rows' input gradients
  const size_t zsh = M.Fsh > 0 ? T * static_cast<size_t>(M.sh.p * M.sh.R) * 2 : 0;
  take(B.zsh_off, zsh);               // the shared expert's z, h and dz
  take(B.hsh_off, M.Fsh > 0 ? T * static_cast<size_t>(M.sh.p * M.sh.Fsp) * 2 : 0);
  take(B.dzs_off, zsh);
  take(B.dxsh_off, M.Fsh > 0 ? T * d * 4 : 0);
  B.bytes = o;
  return B;
}
}  // namespace

extern "C" size_t tp_moe_bwd_workspace(const tp_moe_desc* desc) {
  MoeLayout M;
  return moe_layout(desc, &M) == TP_OK ? moe_bwd_layout(M).bytes : 0;
}

extern "C" tp_status tp_moe_bwd(const tp_moe_desc* desc, const void* x, const void* wr,
                                const void* w1p, const void* w2p, const void* w1p_s,
                                const void* w2p_s, const void* dy, void* dx, float* dwr,
                                float* dw1p, float* dw2p, float* dw1p_s, float* dw2p_s,
                                void* workspace, size_t ws_bytes, void* stream) {
  clear_error();
  MoeLayout M;
  tp_status st = moe_layout(desc, &M);
  if (st != TP_OK) return st;
  const MoeBwdLayout B = moe_bwd_layout(M);
  const MlpLayout& L = M.ex;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!dwr || !dw1p || !dw2p || (M.Fsh > 0 && (!dw1p_s || !dw2p_s)))
    return set_error(TP_ERR_INVALID_ARG, "null gradient pointer");
  if (M.T == 0) {   // no tokens: every gradient is zero
    TP_CUDA_TRY(cudaMemsetAsync(dwr, 0, static_cast<size_t>(M.d) * M.E * 4, s));
    TP_CUDA_TRY(cudaMemsetAsync(dw1p, 0, static_cast<size_t>(M.E) * L.w1p_bytes * 2, s));
    TP_CUDA_TRY(cudaMemsetAsync(dw2p, 0, static_cast<size_t>(M.E) * L.w2p_bytes * 2, s));
    if (M.Fsh > 0) {
      TP_CUDA_TRY(cudaMemsetAsync(dw1p_s, 0, M.sh.w1p_bytes * 2, s));
      TP_CUDA_TRY(cudaMemsetAsync(dw2p_s, 0, M.sh.w2p_bytes * 2, s));
    }
    return TP_OK;
  }
  if (!x || !wr || !w1p || !w2p || !dy || !dx) return set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (M.Fsh > 0 && (!w1p_s || !w2p_s))
    return set_error(TP_ERR_INVALID_ARG, "the shared expert's packed weights are null");
  for (const void* q : {x, wr, w1p, w2p, w1p_s, w2p_s, dy, static_cast<const void*>(dx),
                        static_cast<const void*>(dw1p), static_cast<const void*>(dw2p),
                        static_cast<const void*>(dw1p_s), static_cast<const void*>(dw2p_s)})
    if (q && !aligned16(q)) return set_error(TP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!workspace) return set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < B.bytes) return set_error(TP_ERR_WORKSPACE, "workspace too small");
  if (!tensor_cores_usable())
    return set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
  using BF = __nv_bfloat16;
  int32_t* idx = reinterpret_cast<int32_t*>(off(workspace, M.idx_off));
  float* wts = reinterpret_cast<float*>(off(workspace, M.w_off));
  const int32_t* cnt = reinterpret_cast<const int32_t*>(off(workspace, M.cnt_off));
  const int32_t* offs = reinterpret_cast<const int32_t*>(off(workspace, M.off_off));
  const int32_t* perm = reinterpret_cast<const int32_t*>(off(workspace, M.perm_off));
  const int32_t* inv = reinterpret_cast<const int32_t*>(off(workspace, M.inv_off));
  BF* xs = reinterpret_cast<BF*>(off(workspace, M.xs_off));
  BF* hs = reinterpret_cast<BF*>(off(workspace, M.hs_off));
  float* o = reinterpret_cast<float*>(off(workspace, M.part_off));
  BF* zs = reinterpret_cast<BF*>(off(workspace, B.zs_off));
  float* dwk = reinterpret_cast<float*>(off(workspace, B.dw_off));
  BF* dl = reinterpret_cast<BF*>(off(workspace, B.dl_off));
  float* dxr = reinterpret_cast<float*>(off(workspace, B.dxr_off));
  BF* gs = reinterpret_cast<BF*>(off(workspace, B.gs_off));
  BF* dz = reinterpret_cast<BF*>(off(workspace, B.dz_off));
  float* dxs = reinterpret_cast<float*>(off(workspace, B.dxs_off));
  // (1) the forward's routing, dispatch and expert activations again, keeping z
  if ((st = moe_routed(M, x, wr, w1p, w2p, workspace, idx, wts, zs, s)) != TP_OK) return st;
  // (2) routing-weight gradients, then the router logits' through the softmax over the chosen k
  {
    ProfScope prof(s, "moe_bwd_route");
    const int64_t warps = M.n_rows;
    TP_LAUNCH_PDL(moe::route_weight_grad_kernel, dim3(static_cast<unsigned>(ceil_div(warps * 32, 256))),
                  dim3(256), 0, s, static_cast<const BF*>(dy), static_cast<const float*>(o), inv,
                  M.k, M.T, M.d, dwk);
    const int64_t n = M.T * M.E;
    TP_LAUNCH_PDL(moe::router_logit_grad_kernel, dim3(static_cast<unsigned>(ceil_div(n, 256))),
                  dim3(256), 0, s, static_cast<const int32_t*>(idx), static_cast<const float*>(wts),
                  static_cast<const float*>(dwk), M.k, M.T, M.E, dl);
    // w * dy of every routed row, in expert order
    TP_LAUNCH_PDL(moe::gather_scaled_kernel,
                  dim3(static_cast<unsigned>(ceil_div(M.n_rows, moe::kGatherRowsPerBlock))),
                  dim3(32 * moe::kGatherRowsPerBlock), 0, s, static_cast<const BF*>(dy), perm,
                  static_cast<const float*>(wts), M.k, M.d, M.n_rows, gs);
  }
  // (3) dWr = x^T dl [d][E] (x and dl read MN-major) and dx through the router dl Wr^T [T][d]
  // (dl and Wr read K-major), fp32, on the tensor cores
  {
    const Operand xa{x, true, M.d, M.T, 1, M.d, 0};
    const Operand lb{dl, true, M.E, M.T, 1, M.E, 0};
    tc::EpiStoreF32::Params ep;
    ep.out = dwr;
    ep.ld = M.E;
    ep.batch_stride = 0;
    ep.rows_valid = static_cast<int32_t>(M.d);
    ep.cols_valid = M.E;
    ep.swap = 0;
    st = tc::run_gemm<TileCfg<128, 1, true, true, stages_for(128, 1)>, tc::EpiStoreF32>(
        xa, lb, M.d, M.E, M.T, 1, ep, s, "moe_bwd_dwr_gemm");
    if (st != TP_OK) return st;
    const Operand la{dl, false, M.T, M.E, 1, M.E, 0};
    const Operand wb{wr, false, M.d, M.E, 1, M.E, 0};
    ep.out = dxr;
    ep.ld = M.d;
    ep.rows_valid = static_cast<int32_t>(M.T);
    ep.cols_valid = static_cast<int32_t>(M.d);
    st = tc::run_gemm<TileCfg<128, 1, false, false, stages_for(128, 1)>, tc::EpiStoreF32>(
        la, wb, M.T, M.d, M.E, 1, ep, s, "moe_bwd_dxr_gemm");
    if (st != TP_OK) return st;
  }
  // (4) every chosen expert's MLP backward on its routed rows (their gradient w * dy): dW1, dW2
  // into its slice of dw1p / dw2p, dx of the rows (shards summed in the accumulator) into dxs.
  // The per-expert row counts come back to the host once.  Each expert works on its own rows of
  // every buffer (dz included), so the experts run side by side on kMoeStreams streams.
  {
    std::vector<int32_t> hcnt(static_cast<size_t>(M.E)), hoff(static_cast<size_t>(M.E));
    TP_CUDA_TRY(cudaMemcpyAsync(hcnt.data(), cnt, hcnt.size() * 4, cudaMemcpyDeviceToHost, s));
    TP_CUDA_TRY(cudaMemcpyAsync(hoff.data(), offs, hoff.size() * 4, cudaMemcpyDeviceToHost, s));
    TP_CUDA_TRY(cudaStreamSynchronize(s));
    cudaStream_t pool[kMoeStreams];
    if ((st = moe_streams(pool)) != TP_OK) return st;
    cudaEvent_t ev[kMoeStreams + 1];
    for (auto& e : ev) TP_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    TP_CUDA_TRY(cudaEventRecord(ev[kMoeStreams], s));
    for (int j = 0; j < kMoeStreams; ++j) TP_CUDA_TRY(cudaStreamWaitEvent(pool[j], ev[kMoeStreams], 0));
    const int64_t zrow = L.p * L.R, hrow = L.p * L.Fsp;
    int next = 0;
    for (int e = 0; e < M.E && st == TP_OK; ++e) {
      const int64_t n = hcnt[static_cast<size_t>(e)], r0 = hoff[static_cast<size_t>(e)];
      cudaStream_t se = pool[next];
      next = next + 1 == kMoeStreams ? 0 : next + 1;
      if (n == 0) {   // an expert no token chose: zero gradients
        if (cudaMemsetAsync(dw1p + e * (L.w1p_bytes / 2), 0, L.w1p_bytes * 2, se) != cudaSuccess ||
            cudaMemsetAsync(dw2p + e * (L.w2p_bytes / 2), 0, L.w2p_bytes * 2, se) != cudaSuccess)
          st = set_error(TP_ERR_CUDA, "cudaMemsetAsync of an unchosen expert's gradients");
        continue;
      }
      tp_mlp_desc me{n, M.d, M.F, M.p, TP_ACT_SWIGLU, TP_BF16, TP_REDUCE_FUSED, 0, 0.f};
      MlpLayout Le;
      if ((st = layout_of(&me, &Le)) != TP_OK) break;
      st = tc_backward(Le, gs + r0 * M.d, xs + r0 * M.d, zs + r0 * zrow, hs + r0 * hrow,
                       off(const_cast<void*>(w1p), e * L.w1p_bytes),
                       off(const_cast<void*>(w2p), e * L.w2p_bytes), dz + r0 * zrow,
                       dw1p + e * (L.w1p_bytes / 2), dw2p + e * (L.w2p_bytes / 2), nullptr,
                       dxs + r0 * M.d, true, se);
    }
    // join: the caller's stream waits for every expert's work (also on an error, so that nothing
    // of this call is left running unordered behind it)
    for (int j = 0; j < kMoeStreams; ++j) {
      if (cudaEventRecord(ev[j], pool[j]) == cudaSuccess) (void)cudaStreamWaitEvent(s, ev[j], 0);
    }
    for (auto& e : ev) (void)cudaEventDestroy(e);
    if (st != TP_OK) return st;
  }
  // (5) the shared expert: its forward again (keeping z and h), then its MLP backward with dy
  const float* dxsh = nullptr;
  if (M.Fsh > 0) {
    void* ws = off(workspace, M.shared_off);
    void* h = off(workspace, B.hsh_off);
    void* z = off(workspace, B.zsh_off);
    void* sk = off(ws, M.sh.fsk_off);
    const size_t skb = M.sh.fpart_off - M.sh.fsk_off;
    float* dxs_sh = reinterpret_cast<float*>(off(workspace, B.dxsh_off));
    if ((st = tc_up(M.sh, x, w1p_s, h, z, sk, skb, s)) != TP_OK) return st;
    if ((st = tc_backward(M.sh, dy, x, z, h, w1p_s, w2p_s, off(workspace, B.dzs_off), dw1p_s,
                          dw2p_s, nullptr, dxs_sh, true, s)) != TP_OK)
      return st;
    dxsh = dxs_sh;
  }
  // (6) dx = sum over the choices of the routed rows' input gradients + the router's + the
  // shared expert's
  {
    ProfScope prof(s, "moe_bwd_combine");
    const int64_t nv = M.T * (M.d / 8);
    const int64_t blocks = std::min<int64_t>(ceil_div(nv, 256), static_cast<int64_t>(num_sms()) * 8);
    TP_LAUNCH_PDL(moe::dx_combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                  static_cast<const float*>(dxs), static_cast<const float*>(dxr), dxsh, inv, M.k,
                  M.T, M.d, static_cast<BF*>(dx));
  }
  return TP_OK;
}
