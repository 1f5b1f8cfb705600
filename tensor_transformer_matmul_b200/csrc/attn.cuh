// Attention block internals: layout, packing, QKV projection, local GQA attention per shard,
// KV-cache append, row-parallel output projection and the partial-sum reduce.
#pragma once

#include <algorithm>
#include <tuple>

#include "flash_attn.cuh"
#include "gemm_launch.cuh"
#include "gemm_pair.cuh"
#include "pack.cuh"
#include "reduce.cuh"
#include "seqpar.cuh"
#include "simt.cuh"
#include "tp_common.cuh"

namespace tp {

struct AttnLayout {
  int64_t b, s, h, tokens, kv_len, kv_cap;
  int n_q, n_kv, hd, p, qh, kh, causal, dtype, eb, y_dtype;
  float norm_eps;
  int64_t R_a;          // packed QKV rows per shard
  size_t wqkv_bytes, wo_bytes;
  size_t qkv_off, o_off, part_off, ml_off, sk_off, ws_bytes;
  int kv_splits;        // decode: key chunks per (sequence, KV head)
  int kv_chunk;         // decode: keys per chunk
  size_t cnt_off;       // decode: arrival counters [b][n_kv]
  int reduce_mode;
  bool tc;              // bf16 with 16-byte rows: tensor-core projections
};

namespace attn_tc {
using tc::Operand;
template <int BN, int ASUB>
using KK = tc::TileCfg<BN, ASUB, false, false,
                       std::min(8, (200 * 1024) / (128 * ASUB * 64 * 2 + BN * 64 * 2))>;
template <class C> struct Tag { using type = C; };
// 256 x 256 tiles on SM pairs (cta_group::2): the prefill and backward projections
template <bool A_MN, bool B_MN>
using PP = tc::PairCfg<A_MN, B_MN, 6>;
constexpr int64_t kSwapMaxT = 128;
template <class F>
auto by_tokens(int64_t T, F&& f) {
  if (T <= 16) return f(Tag<KK<16, 1>>{});
  if (T <= 64) return f(Tag<KK<64, 1>>{});
  return f(Tag<KK<128, 1>>{});
}
}  // namespace attn_tc

inline int64_t qkv_tiles(const AttnLayout& L) { return ceil_div(L.p * L.R_a, 128); }
inline int64_t out_tiles(const AttnLayout& L) { return L.p * ceil_div(L.h, 128); }

// stream-K bytes of the QKV projection and of the output projection (0 when not stream-K)
inline size_t attn_sk_bytes(const AttnLayout& L) {
  using namespace attn_tc;
  if (!L.tc || L.tokens == 0) return 0;
  const int64_t rows = L.p * L.R_a, K = static_cast<int64_t>(L.qh) * L.hd;
  const bool fused = L.reduce_mode == TP_REDUCE_FUSED;
  size_t a = 0, b = 0;
  if (L.tokens <= kSwapMaxT) {
    if (decode_stream_k(qkv_tiles(L), L.tokens, ceil_div(L.h, 64))) a = by_tokens(L.tokens, [&](auto t) {
      return tc::plan_stream_k<typename decltype(t)::type>(rows, L.tokens, L.h, 1, false, num_sms()).bytes();
    });
    if (decode_stream_k(out_tiles(L), L.tokens, ceil_div(static_cast<int64_t>(L.qh) * L.hd, 64)) || fused) b = by_tokens(L.tokens, [&](auto t) {
      return tc::plan_stream_k<typename decltype(t)::type>(L.h, L.tokens, K, L.p, fused, num_sms()).bytes();
    });
  }
  return std::max(a, b);
}


// Decode shapes the MMA decode kernel takes (the rest use the SIMT split kernel).
// Most splits of one KV head merged through distributed shared memory (a non-portable cluster
// size on sm_100; the launch checks that such clusters fit and otherwise merges through memory).
constexpr int64_t kDecodeClusterMax = 16;

inline bool decode_mma_eligible(const AttnLayout& L, const tp_attn_desc* d) {
  const int group = d->n_q / d->n_kv;
  return d->dtype == TP_BF16 && (L.hd == 64 || L.hd == 128) &&
         (group == 1 || group == 2 || group == 4 || group == 8);
}

inline tp_status attn_layout_of(const tp_attn_desc* d, AttnLayout* L) {
  if (!d) return set_error(TP_ERR_INVALID_ARG, "desc is null");
  if (d->b < 0 || d->s < 0) return set_error(TP_ERR_SHAPE, "b and s must be >= 0");
  if (d->h < 1 || d->n_q < 1 || d->n_kv < 1 || d->p < 1)
    return set_error(TP_ERR_SHAPE, "h, n_q, n_kv and p must be >= 1");
  if (d->n_q % d->n_kv) return set_error(TP_ERR_SHAPE, "n_kv must divide n_q");
  if (d->n_q % d->p || d->n_kv % d->p)
    return set_error(TP_ERR_SHAPE, "p must divide n_q and n_kv (heads are never split)");
  if (d->head_dim < 8 || d->head_dim > 256 || d->head_dim % 8)
    return set_error(TP_ERR_SHAPE, "head_dim must be a multiple of 8 in [8, 256]");
  if (d->dtype != TP_F32 && d->dtype != TP_BF16) return set_error(TP_ERR_INVALID_ARG, "dtype");
  if (d->reduce_mode != TP_REDUCE_SEPARATE && d->reduce_mode != TP_REDUCE_FUSED)
    return set_error(TP_ERR_INVALID_ARG, "unknown reduce_mode");
  if (d->flags & ~TP_FLAG_F32_RESIDUAL) return set_error(TP_ERR_INVALID_ARG, "unknown flags");
  if (d->kv_len < 0) return set_error(TP_ERR_SHAPE, "kv_len must be >= 0");
  if (d->kv_len > 0 && d->s != 1) return set_error(TP_ERR_SHAPE, "decode (kv_len > 0) needs s == 1");
  L->b = d->b; L->s = d->s; L->h = d->h; L->tokens = d->b * d->s;
  L->n_q = d->n_q; L->n_kv = d->n_kv; L->hd = d->head_dim; L->p = d->p;
  L->qh = d->n_q / d->p; L->kh = d->n_kv / d->p;
  L->causal = d->causal ? 1 : 0; L->dtype = d->dtype; L->eb = elem_bytes(d->dtype);
  L->y_dtype = (d->flags & TP_FLAG_F32_RESIDUAL) ? TP_F32 : d->dtype;
  L->norm_eps = d->norm_eps > 0.f ? d->norm_eps : 1e-5f;
  L->kv_len = d->kv_len;
  L->kv_cap = d->kv_cap > 0 ? d->kv_cap : d->kv_len + 1;
  if (L->kv_len > 0 && L->kv_cap < L->kv_len + 1)
    return set_error(TP_ERR_SHAPE, "kv_cap must be >= kv_len + 1");
  L->R_a = static_cast<int64_t>(L->qh + 2 * L->kh) * L->hd;
  const int64_t P = L->p;
  L->wqkv_bytes = static_cast<size_t>(P * L->R_a * L->h) * L->eb;
  L->wo_bytes = static_cast<size_t>(P * L->h * L->qh * L->hd) * L->eb;
  if (L->kv_len > 0) {
    // blocks over (split, KV head, sequence); chunks a multiple of 16 keys
    const int64_t n_keys = L->kv_len + 1;
    // at most one wave: splits * n_kv * b <= SMs when possible; a split's K and V rows must fit
    // in shared memory (staged by bulk copies)
    int64_t max_chunk = std::min<int64_t>(
        512, (200 * 1024) / (2 * static_cast<int64_t>(L->hd) * L->eb + 4 * (L->n_q / L->n_kv)) / 16 * 16);
    // the MMA decode kernel (bf16, head_dim 64/128, <= 8 query heads per KV head) stages at most
    // 384 (head_dim 128) or 768 (head_dim 64) keys per split, and merges the splits of a KV head
    // inside a cluster when there are at most kDecodeClusterMax of them
    int64_t want = std::max<int64_t>(1, num_sms() / std::max<int64_t>(1, L->b * L->n_kv));
    if (decode_mma_eligible(*L, d)) {
      max_chunk = std::min<int64_t>(max_chunk, L->hd == 128 ? 384 : 768);
      want = std::min<int64_t>(want, kDecodeClusterMax);
    }
    int64_t splits = std::min<int64_t>(std::min<int64_t>(want, 64), ceil_div(n_keys, 16));
    splits = std::max<int64_t>(splits, ceil_div(n_keys, max_chunk));
    L->kv_chunk = static_cast<int>(round_up(ceil_div(n_keys, splits), 16));
    L->kv_splits = static_cast<int>(ceil_div(n_keys, L->kv_chunk));
    if (L->kv_chunk > max_chunk || L->kv_splits > 64)
      return set_error(TP_ERR_UNSUPPORTED, "decode KV length too long for the split-KV kernel");
  } else {
    L->kv_chunk = 0;
    L->kv_splits = 0;
  }
  const size_t qkvb = static_cast<size_t>(L->tokens * P * L->R_a) * L->eb;
  const size_t ob = static_cast<size_t>(L->tokens * L->n_q * L->hd) * L->eb;
  const size_t partb = static_cast<size_t>(P * L->tokens * L->h) * 4;
  // decode split-KV scratch: per (sequence, q head, split) an (m, l) pair and hd outputs
  const size_t mlb = static_cast<size_t>(L->b * L->n_q * L->kv_splits) * (L->hd + 4) * 4;
  L->reduce_mode = d->reduce_mode;
  L->tc = d->dtype == TP_BF16 && d->h % 8 == 0;
  L->qkv_off = 0;
  L->o_off = align256(qkvb);
  L->part_off = L->o_off + align256(ob);
  const size_t pb = (L->tc && L->reduce_mode == TP_REDUCE_FUSED) ? 0 : partb;
  L->ml_off = L->part_off + align256(pb);
  L->cnt_off = L->ml_off + align256(mlb);
  const size_t cntb = L->kv_len > 0 ? static_cast<size_t>(L->b * L->n_kv) * sizeof(int32_t) : 0;
  L->sk_off = L->cnt_off + align256(cntb);
  L->ws_bytes = L->sk_off + align256(attn_sk_bytes(*L));
  return TP_OK;
}

// ``ldq`` / ``ldkv``: row lengths of the user's Wq and Wk / Wv when they exceed this layout's
// (L is one shard's layout and the pointers sit at that shard's first column).
template <typename T>
inline tp_status attn_pack_t(const AttnLayout& L, const void* wq, const void* wk, const void* wv,
                             const void* wo, void* wqkv_p, void* wo_p, cudaStream_t s,
                             int64_t ldq = 0, int64_t ldkv = 0) {
  pack::ColMap cm{};
  cm.kind = 2;
  cm.R = L.R_a;
  cm.q_rows = static_cast<int64_t>(L.qh) * L.hd;
  cm.k_rows = static_cast<int64_t>(L.kh) * L.hd;
  cm.src[0] = wq; cm.src[1] = wk; cm.src[2] = wv;
  cm.ld[0] = ldq > 0 ? ldq : static_cast<int64_t>(L.n_q) * L.hd;
  cm.ld[1] = cm.ld[2] = ldkv > 0 ? ldkv : static_cast<int64_t>(L.n_kv) * L.hd;
  const int64_t rows = L.p * L.R_a;
  dim3 blk(32, 8);
  dim3 g1(static_cast<unsigned>(ceil_div(rows, 32)), static_cast<unsigned>(ceil_div(L.h, 32)), 1);
  if (!pack::grid_ok(g1.x, g1.y, 1)) return set_error(TP_ERR_UNSUPPORTED, "pack grid too large");
  pack::pack_cols_kernel<T><<<g1, blk, 0, s>>>(static_cast<T*>(wqkv_p), rows, L.h, cm);
  TP_LAUNCH_CHECK();
  const int64_t K = static_cast<int64_t>(L.qh) * L.hd;
  dim3 g2(static_cast<unsigned>(ceil_div(L.h, 32)), static_cast<unsigned>(ceil_div(K, 32)),
          static_cast<unsigned>(L.p));
  if (!pack::grid_ok(g2.x, g2.y, g2.z)) return set_error(TP_ERR_UNSUPPORTED, "pack grid too large");
  pack::pack_rows_kernel<T><<<g2, blk, 0, s>>>(static_cast<T*>(wo_p), L.p, L.h, K, K,
                                               static_cast<const T*>(wo), L.h);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

inline tp_status attn_pack(const AttnLayout& L, const void* wq, const void* wk, const void* wv,
                           const void* wo, void* wqkv_p, void* wo_p, cudaStream_t s,
                           int64_t ldq = 0, int64_t ldkv = 0) {
  return L.dtype == TP_BF16
             ? attn_pack_t<__nv_bfloat16>(L, wq, wk, wv, wo, wqkv_p, wo_p, s, ldq, ldkv)
             : attn_pack_t<float>(L, wq, wk, wv, wo, wqkv_p, wo_p, s, ldq, ldkv);
}

namespace attn {

// Index helpers into the packed qkv activations [tokens][p * R_a].
struct QkvIdx {
  int64_t ld;     // p * R_a
  int64_t R_a;
  int qh, kh, hd, group;   // group = n_q / n_kv
  __device__ __forceinline__ int64_t q(int64_t t, int j) const {   // global q head j
    const int i = j / qh, jj = j - i * qh;
    return t * ld + i * R_a + static_cast<int64_t>(jj) * hd;
  }
  __device__ __forceinline__ int64_t k(int64_t t, int g) const {   // global kv head g
    const int i = g / kh, gg = g - i * kh;
    return t * ld + i * R_a + static_cast<int64_t>(qh + gg) * hd;
  }
  __device__ __forceinline__ int64_t v(int64_t t, int g) const {
    const int i = g / kh, gg = g - i * kh;
    return t * ld + i * R_a + static_cast<int64_t>(qh + kh + gg) * hd;
  }
};

// Prefill attention, one warp per (token, query head), online softmax over the visible keys.
// o[t][j*hd + e]; lane l holds dims l, l+32, ... of q and of the running output.
template <typename T>
__global__ void __launch_bounds__(128) prefill_simt_kernel(const T* qkv, T* o, QkvIdx ix,
                                                           int64_t b, int64_t s, int n_q,
                                                           int causal, float scale, float* lse) {
  constexpr int kMaxPerLane = 8;  // head_dim <= 256
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= b * s * n_q) return;
  const int j = static_cast<int>(wid % n_q);
  const int64_t t = wid / n_q;          // global token
  const int64_t bi = t / s, pos = t - bi * s;
  const int g = j / ix.group;
  const int per = (ix.hd + 31) / 32;
  float q[kMaxPerLane], acc[kMaxPerLane];
#pragma unroll
  for (int r = 0; r < kMaxPerLane; ++r) {
    const int e = lane + 32 * r;
    q[r] = (r < per && e < ix.hd) ? to_f(qkv[ix.q(t, j) + e]) * scale : 0.f;
    acc[r] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int64_t last = causal ? pos : s - 1;
  for (int64_t kp = 0; kp <= last; ++kp) {
    const int64_t tk = bi * s + kp;
    const int64_t kb = ix.k(tk, g), vb = ix.v(tk, g);
    float dot = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxPerLane; ++r) {
      const int e = lane + 32 * r;
      if (r < per && e < ix.hd) dot = fmaf(q[r], to_f(qkv[kb + e]), dot);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float mn = fmaxf(m, dot);
    const float corr = expf(m - mn), pw = expf(dot - mn);
    l = l * corr + pw;
#pragma unroll
    for (int r = 0; r < kMaxPerLane; ++r) {
      const int e = lane + 32 * r;
      if (r < per && e < ix.hd) acc[r] = acc[r] * corr + pw * to_f(qkv[vb + e]);
    }
    m = mn;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int r = 0; r < kMaxPerLane; ++r) {
    const int e = lane + 32 * r;
    if (r < per && e < ix.hd) o[t * static_cast<int64_t>(n_q) * ix.hd + j * ix.hd + e] = from_f<T>(acc[r] * inv);
  }
  // log2 of the softmax denominator in units of the log2-scaled scores (backward pass)
  if (lse && lane == 0) lse[t * n_q + j] = (m + logf(l)) * 1.4426950408889634f;
}

// Decode attention, split over keys.  Block = (split c, KV head g, sequence bi), 256 threads.
// The split's K and V rows (contiguous in the cache) are staged into shared memory by two bulk
// async copies, then three phases run over the staged keys (all query heads of the KV group
// together, so each K and V row is read from HBM once):
//   1. scores: a group of HD/8 lanes per key, each lane holding 8 consecutive dims;
//      s[key][a] = (q_a . k) * log2(e)/sqrt(hd)
//   2. softmax statistics: one warp per query head, m_a = max s, p = exp2(s - m_a), l_a = sum p
//   3. o_a[d] = sum_key p[key][a] v[key][d]: each thread owns one dim d and GROUP*HD/256 heads
// The new token (position kv_len) takes its key and value from the projection; the split that
// holds it patches them into its staged rows and stores them into cache slot kv_len.
// Output per (bi, q head, split): a record of hd + 4 floats, o[hd] then m (log2 units) and l
// (16-byte aligned records, so the merge reads o with vector loads).
// The last block of a (sequence, KV head) to finish merges all splits of its query heads, in
// split order: o = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c, from the per-split records
// (o[HD], m in log2 units, l) in ``ml``.  No block waits for another: a counter per (sequence,
// KV head) tells each block whether it is the last, and the last one resets it.
template <typename T, int GROUP, int HD>
__device__ __forceinline__ void merge_splits_if_last(const float* ml, int* counters, T* o,
                                                     int64_t bi, int g, int n_q, int n_kv) {
  constexpr int kWarps = 8;
  constexpr int kRec = HD + 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int* cnt = counters + bi * n_kv + g;
    const int last = atomicAdd(cnt, 1) == static_cast<int>(gridDim.x) - 1;
    if (last) *cnt = 0;
    s_last = last;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // weights w[a][c] = exp(m_c - M_a) / L_a of every split: all (m, l) pairs are loaded at once,
  // then one warp per query head reduces over the splits with shuffles; then independent loads
  // of the o_c
  constexpr int kMaxSplits = 64;
  __shared__ float s_w[GROUP][kMaxSplits], s_lc[GROUP][kMaxSplits];
  const int splits = gridDim.x;   // <= kMaxSplits (host)
  const float* recs = ml + (bi * n_q + static_cast<int64_t>(g) * GROUP) * splits * kRec;
  for (int idx = threadIdx.x; idx < GROUP * splits; idx += blockDim.x) {
    const int a = idx / splits, sp = idx - a * splits;
    const float* r = recs + (static_cast<int64_t>(a) * splits + sp) * kRec;
    s_w[a][sp] = __ldcg(r + HD);        // m (log2 units)
    s_lc[a][sp] = __ldcg(r + HD + 1);   // l
  }
  __syncthreads();
  for (int a = warp; a < GROUP; a += kWarps) {
    // splits <= 64: lane handles splits lane and lane + 32
    const float m0 = lane < splits ? s_w[a][lane] : -INFINITY;
    const float m1 = lane + 32 < splits ? s_w[a][lane + 32] : -INFINITY;
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M);
    const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
    float Ls = (lane < splits ? s_lc[a][lane] * f0 : 0.f) +
               (lane + 32 < splits ? s_lc[a][lane + 32] * f1 : 0.f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
    const float inv = 1.f / Ls;
    if (lane < splits) s_w[a][lane] = f0 * inv;
    if (lane + 32 < splits) s_w[a][lane + 32] = f1 * inv;
  }
  __syncthreads();
  // o: four consecutive dims per thread, every split's 16-byte load issued before the adds,
  // which run in split order
  constexpr int V4 = HD / 4;
  for (int idx = threadIdx.x; idx < GROUP * V4; idx += blockDim.x) {
    const int a = idx / V4, e4 = idx - a * V4;
    const float4* r = reinterpret_cast<const float4*>(recs + static_cast<int64_t>(a) * splits * kRec) + e4;
    float4 acc2 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 16
    for (int sp = 0; sp < splits; ++sp) {
      const float4 v = __ldcg(r + static_cast<int64_t>(sp) * (kRec / 4));
      const float w = s_w[a][sp];
      acc2.x += w * v.x;
      acc2.y += w * v.y;
      acc2.z += w * v.z;
      acc2.w += w * v.w;
    }
    T* op = o + bi * static_cast<int64_t>(n_q) * HD + (g * GROUP + a) * HD + 4 * e4;
    op[0] = from_f<T>(acc2.x);
    op[1] = from_f<T>(acc2.y);
    op[2] = from_f<T>(acc2.z);
    op[3] = from_f<T>(acc2.w);
  }
}

template <int HD, int GROUP, typename T>
struct DecodeSmem {
  static size_t bytes(int chunk) {
    return static_cast<size_t>(chunk) * HD * sizeof(T) * 2 + static_cast<size_t>(chunk) * GROUP * 4 +
           64;
  }
};

template <typename T, int GROUP, int HD>
__global__ void __launch_bounds__(256) decode_split_kernel(const T* qkv, QkvIdx ix, T* kc, T* vc,
                                                           int64_t kv_cap, int64_t kv_len,
                                                           int chunk, int n_q, int n_kv,
                                                           float scale, float* ml, int* counters,
                                                           T* o, uint32_t* err) {
  constexpr int kWarps = 8;
  constexpr int LPK = HD / 8;            // lanes per key
  constexpr int KPW = 32 / LPK;          // keys per warp pass
  constexpr int APT = (GROUP * HD + 255) / 256;   // heads per thread in phase 3
  constexpr int kRec = HD + 4;                    // floats per split record: o[HD], m, l, pad
  extern __shared__ __align__(16) uint8_t dsm[];
  T* sK = reinterpret_cast<T*>(dsm);
  T* sV = sK + static_cast<size_t>(chunk) * HD;
  float* s_p = reinterpret_cast<float*>(sV + static_cast<size_t>(chunk) * HD);   // [chunk][GROUP]
  __shared__ float s_m[GROUP], s_l[GROUP];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_ok;
  const int c = blockIdx.x, g = blockIdx.y;
  const int64_t bi = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_keys = kv_len + 1;       // the cached positions plus the new token
  const int64_t k0 = static_cast<int64_t>(c) * chunk;
  const int nk = static_cast<int>(min(n_keys, k0 + chunk) - k0);
  T* kbase = kc + (bi * n_kv + g) * kv_cap * HD;
  T* vbase = vc + (bi * n_kv + g) * kv_cap * HD;
  const T* knew = qkv + ix.k(bi, g);
  const T* vnew = qkv + ix.v(bi, g);
  const float sl2 = scale * 1.4426950408889634f;
  pdl_wait();   // global memory only from here on (programmatic dependent launch)
  pdl_trigger();

  // ---- stage the split's K and V rows
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  const uint32_t rows_bytes = static_cast<uint32_t>(nk) * HD * sizeof(T);
  if (threadIdx.x == 0) {
    sm100::mbar_arrive_expect_tx(&bar, 2 * rows_bytes);
    sm100::bulk_load(sK, kbase + k0 * HD, rows_bytes, &bar);
    sm100::bulk_load(sV, vbase + k0 * HD, rows_bytes, &bar);
  }
  {
    // every thread waits (bounded); on a timeout the copies must still land before the block
    // leaves, so wait again without the abort shortcut (also bounded)
    int dummy_abort = 0;
    bool ok = sm100::mbar_wait(&bar, 0, &dummy_abort, err, DEVERR_WAIT_FULL);
    if (!ok) {
      const uint64_t t0 = globaltimer_ns();
      while (!sm100::mbar_try_wait(&bar, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
    if (threadIdx.x == 0) s_ok = 1;
    __syncthreads();
    if (!ok) s_ok = 0;
    __syncthreads();
    if (!s_ok) return;
  }
  // the new token: patch its staged rows from the projection and append it to the cache
  if (kv_len >= k0 && kv_len < k0 + nk) {
    const int r = static_cast<int>(kv_len - k0);
    for (int e = threadIdx.x; e < HD; e += blockDim.x) {
      const T kvv = knew[e], vvv = vnew[e];
      sK[static_cast<size_t>(r) * HD + e] = kvv;
      sV[static_cast<size_t>(r) * HD + e] = vvv;
      kbase[kv_len * HD + e] = kvv;
      vbase[kv_len * HD + e] = vvv;
    }
  }
  __syncthreads();

  // ---- phase 1: scores
  {
    // the group's query vectors, scaled, staged once per block in shared memory
    __shared__ __align__(16) float s_q[GROUP][HD];
    for (int idx = threadIdx.x; idx < GROUP * HD; idx += blockDim.x) {
      const int a = idx / HD, e = idx - a * HD;
      s_q[a][e] = to_f(qkv[ix.q(bi, g * GROUP + a) + e]) * sl2;
    }
    __syncthreads();
    const int kslot = lane / LPK;
    const int d0 = (lane % LPK) * 8;
    float q[GROUP][8];
#pragma unroll
    for (int a = 0; a < GROUP; ++a) {
      const float4 q0 = *reinterpret_cast<const float4*>(&s_q[a][d0]);
      const float4 q1 = *reinterpret_cast<const float4*>(&s_q[a][d0 + 4]);
      q[a][0] = q0.x; q[a][1] = q0.y; q[a][2] = q0.z; q[a][3] = q0.w;
      q[a][4] = q1.x; q[a][5] = q1.y; q[a][6] = q1.z; q[a][7] = q1.w;
    }
    const int stride = kWarps * KPW;
    for (int wb = warp * KPW; wb < nk; wb += stride) {   // warp-uniform trip count
      const int i = wb + kslot;
      const bool ok = i < nk;
      float kv[8];
      const int ii = ok ? i : 0;
      if constexpr (sizeof(T) == 2) {
        const uint4 w = *reinterpret_cast<const uint4*>(sK + static_cast<size_t>(ii) * HD + d0);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2) {
          kv[2 * h2] = bf16lo(ww[h2]);
          kv[2 * h2 + 1] = bf16hi(ww[h2]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) kv[e] = to_f(sK[static_cast<size_t>(ii) * HD + d0 + e]);
      }
#pragma unroll
      for (int a = 0; a < GROUP; ++a) {
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) dot = fmaf(q[a][e], kv[e], dot);
#pragma unroll
        for (int off = LPK / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (ok && (lane % LPK) == 0) s_p[i * GROUP + a] = dot;
      }
    }
  }
  __syncthreads();
  // ---- phase 2: per query head, max and exp over the chunk (one warp per head)
  for (int a = warp; a < GROUP; a += kWarps) {
    float mx = -INFINITY;
    for (int i = lane; i < nk; i += 32) mx = fmaxf(mx, s_p[i * GROUP + a]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sum = 0.f;
    for (int i = lane; i < nk; i += 32) {
      const float pv = exp2f(s_p[i * GROUP + a] - mx);
      s_p[i * GROUP + a] = pv;
      sum += pv;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane == 0) {
      s_m[a] = mx;
      s_l[a] = sum;
    }
  }
  __syncthreads();
  // ---- phase 3: o_a[d] = sum_key p[key][a] v[key][d]
  {
    const int d = threadIdx.x % HD;
    const int a0 = (threadIdx.x / HD) * APT;
    float acc[APT];
#pragma unroll
    for (int t = 0; t < APT; ++t) acc[t] = 0.f;
    if (a0 < GROUP) {
#pragma unroll 8
      for (int i = 0; i < nk; ++i) {
        const float v = to_f(sV[static_cast<size_t>(i) * HD + d]);
#pragma unroll
        for (int t = 0; t < APT; ++t)
          if (a0 + t < GROUP) acc[t] = fmaf(s_p[i * GROUP + a0 + t], v, acc[t]);
      }
#pragma unroll
      for (int t = 0; t < APT; ++t) {
        const int a = a0 + t;
        if (a < GROUP) {
          const int j = g * GROUP + a;
          float* rec = ml + ((bi * n_q + j) * gridDim.x + c) * kRec;
          if (d == 0) {
            rec[HD] = s_m[a];   // in log2 units (the scores carry log2(e))
            rec[HD + 1] = s_l[a];
          }
          rec[d] = acc[t];
        }
      }
    }
  }
  merge_splits_if_last<T, GROUP, HD>(ml, counters, o, bi, g, n_q, n_kv);
}


// ---------------------------------------------------------------------------------------------
// Decode attention for bf16 with head_dim 64 or 128 and up to 8 query heads per KV head.
//
// The same (split, KV head, sequence) blocks and split records as decode_split_kernel, with the
// split's K and V rows streamed instead of staged whole:
//   * the split is cut into sub-chunks of 32 keys; each sub-chunk's K and V arrive as 128B-swizzled
//     TMA tiles [32 keys][64 dims] (the cache seen as [b*n_kv][kv_len][hd]; rows past the cached
//     positions are out of bounds and arrive as zeros) on an mbarrier of their own, all issued
//     at the start, so computing starts as soon as the first tiles land;
//   * warp w takes the 16-key blocks w, w + 8, ...: per block, S = Q K^T for the group's query
//     heads (rows of a 16-row MMA, the unused rows zero) and then O += P V with warp-level bf16
//     MMAs (m16n8k16, fp32 accumulate); the fragments come from the swizzled tiles through
//     ldmatrix, so neither product meets a shared-memory bank conflict;
//   * each warp keeps an online softmax (running max in log2 units, running sum, rescaled O);
//     the 8 warps' states are then combined in shared memory into the split's record;
//   * the block holding the new token (position kv_len) patches its K and V rows into the staged
//     tiles from the projection and stores them into cache slot kv_len.
// The per-block contraction is tiny (at most 8 heads share a K/V row), so the MMAs only take the
// arithmetic off the path of the HBM stream.
template <int HD>
struct DecodeMmaCfg {
  static constexpr int kSub = 32;                       // keys per TMA tile / barrier
  static constexpr int kHalves = HD / 64;               // 64-dim tiles per row
  static constexpr int kTileBytes = kSub * 128;         // one [32][64] bf16 tile
  static constexpr int kSubBytes = 2 * kHalves * kTileBytes;   // K and V of one sub-chunk
  static constexpr int kMaxSub = HD == 128 ? 12 : 24;   // at most 384 (128) or 768 (64) keys
  static constexpr int kMaxChunk = kMaxSub * kSub;
  static constexpr size_t kSmem = static_cast<size_t>(kMaxSub) * kSubBytes + 1024;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8, fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int GROUP, int HD, bool CLUSTER>
__global__ void __launch_bounds__(256) decode_mma_kernel(
    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
    const __nv_bfloat16* qkv, QkvIdx ix, __nv_bfloat16* kc, __nv_bfloat16* vc, int64_t kv_cap,
    int64_t kv_len, int chunk, int n_q, int n_kv, float scale, float* ml, int* counters,
    __nv_bfloat16* o, uint32_t* err) {
  using C = DecodeMmaCfg<HD>;
  constexpr int kWarps = 8;
  constexpr int kRec = HD + 4;
  constexpr int KS = HD / 16;          // k-steps of S = Q K^T
  static_assert(GROUP >= 1 && GROUP <= 8, "at most 8 query heads per KV head");
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[C::kMaxSub];
  __shared__ int s_abort;
  // this split's merged result (cluster merge): o[GROUP][HD], m (log2 units) and l per head
  __shared__ __align__(16) float s_res_o[CLUSTER ? GROUP : 1][CLUSTER ? HD : 4];
  __shared__ float s_res_m[GROUP], s_res_l[GROUP];
  const int c = blockIdx.x, g = blockIdx.y;
  const int64_t bi = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qr = lane >> 2, qc = lane & 3;    // MMA fragment row (query head) and column pair
  const int64_t n_keys = kv_len + 1;
  const int64_t k0 = static_cast<int64_t>(c) * chunk;
  const int nk = static_cast<int>(min(n_keys, k0 + chunk) - k0);
  const int nsub = (nk + C::kSub - 1) / C::kSub;
  const int nblk = (nk + 15) / 16;
  const float sl2 = scale * 1.4426950408889634f;
  // tile (sub, kind 0 = K / 1 = V, half) of the staging area
  auto tile = [&](int sub, int kind, int half) -> uint8_t* {
    return dsm + static_cast<size_t>(sub) * C::kSubBytes + (kind * C::kHalves + half) * C::kTileBytes;
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < nsub; ++i) sm100::mbar_init(&bars[i], 1);
    s_abort = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  // The cached rows 0 .. kv_len-1 are written only by earlier decode steps' calls of this kernel,
  // never by the kernels just before it on the stream (the projection writes q, k, v of the new
  // token; this kernel itself writes slot kv_len, which the tensor maps leave out), so their
  // streaming starts before the programmatic-launch wait and overlaps the previous kernel's tail.
  if (threadIdx.x == 0) {
    const int32_t z = static_cast<int32_t>(bi * n_kv + g);
    for (int i = 0; i < nsub; ++i) {
      sm100::mbar_arrive_expect_tx(&bars[i], C::kSubBytes);
      const int32_t y = static_cast<int32_t>(k0 + i * C::kSub);
      for (int hf = 0; hf < C::kHalves; ++hf) {
        sm100::tma_load_3d(&kmap, &bars[i], tile(i, 0, hf), hf * 64, y, z);
        sm100::tma_load_3d(&vmap, &bars[i], tile(i, 1, hf), hf * 64, y, z);
      }
    }
  }
  pdl_wait();   // everything else in global memory only from here on
  pdl_trigger();

  // the group's query rows as MMA A fragments (rows >= GROUP and rows 8..15 are zero)
  uint32_t qa[KS][2];
  {
    const __nv_bfloat16* qrow = qkv + ix.q(bi, g * GROUP + (qr < GROUP ? qr : 0));
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const uint32_t lo = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * qc);
      const uint32_t hi = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * qc + 8);
      qa[kk][0] = qr < GROUP ? lo : 0u;
      qa[kk][1] = qr < GROUP ? hi : 0u;
    }
  }
  float oacc[HD / 8][4];
#pragma unroll
  for (int nt = 0; nt < HD / 8; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const bool owns_new = kv_len >= k0 && kv_len < k0 + nk;
  const int r_new = static_cast<int>(kv_len - k0);
  int abort_local = 0;

  for (int kb = warp; kb < nblk; kb += kWarps) {
    const int sub = kb >> 1, ro = (kb & 1) * 16;
    if (!sm100::mbar_wait(&bars[sub], 0, &s_abort, err, DEVERR_WAIT_FULL)) {
      abort_local = 1;
      break;
    }
    if (owns_new && (r_new >> 4) == kb) {
      // the new token's key and value: from the projection into the staged tiles and the cache
      const __nv_bfloat16* knew = qkv + ix.k(bi, g);
      const __nv_bfloat16* vnew = qkv + ix.v(bi, g);
      __nv_bfloat16* kdst = kc + ((bi * n_kv + g) * kv_cap + kv_len) * HD;
      __nv_bfloat16* vdst = vc + ((bi * n_kv + g) * kv_cap + kv_len) * HD;
      const int r = r_new & 31;
      for (int e = lane * 4; e < HD; e += 128) {
        const uint2 kv4 = *reinterpret_cast<const uint2*>(knew + e);
        const uint2 vv4 = *reinterpret_cast<const uint2*>(vnew + e);
        const int half = e >> 6, ch = (e & 63) >> 3;
        const size_t off = static_cast<size_t>(r) * 128 + ((ch ^ (r & 7)) << 4) + (e & 7) * 2;
        *reinterpret_cast<uint2*>(tile(sub, 0, half) + off) = kv4;
        *reinterpret_cast<uint2*>(tile(sub, 1, half) + off) = vv4;
        *reinterpret_cast<uint2*>(kdst + e) = kv4;
        *reinterpret_cast<uint2*>(vdst + e) = vv4;
      }
      __syncwarp();
    }
    // ---- S = Q K^T for keys kb*16 .. kb*16+15: two n-tiles of 8 keys
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int mi = lane >> 3, rr = lane & 7;
      const int r = ro + (mi >> 1) * 8 + rr;       // staged row (key) this lane addresses
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        const int half = kk >> 2, ch = ((kk & 3) << 1) + (mi & 1);
        const uint32_t addr = sm100::smem_addr(tile(sub, 0, half)) + r * 128 + ((ch ^ (r & 7)) << 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(addr, b0, b1, b2, b3);
        mma_16816(sacc[0], qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
        mma_16816(sacc[1], qa[kk][0], 0u, qa[kk][1], 0u, b2, b3);
      }
    }
    // ---- online softmax for query head qr over these 16 keys (log2 units)
    float sv[2][2];
    float mblk = -INFINITY;
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int key = kb * 16 + n * 8 + 2 * qc + j;
        sv[n][j] = key < nk ? sacc[n][j] * sl2 : -INFINITY;
        mblk = fmaxf(mblk, sv[n][j]);
      }
    mblk = fmaxf(mblk, __shfl_xor_sync(0xffffffffu, mblk, 1));
    mblk = fmaxf(mblk, __shfl_xor_sync(0xffffffffu, mblk, 2));
    const float m_new = fmaxf(m_run, mblk);       // finite: the block's first key is valid
    const float corr = exp2f(m_run - m_new);      // 0 on the first block (m_run = -inf)
    float p[2][2];
    float psum = 0.f;
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        p[n][j] = exp2f(sv[n][j] - m_new);
        psum += p[n][j];
      }
    l_run = l_run * corr + psum;
    m_run = m_new;
#pragma unroll
    for (int nt = 0; nt < HD / 8; ++nt) {
      oacc[nt][0] *= corr;
      oacc[nt][1] *= corr;
    }
    // ---- O += P V: P (head rows, 16 keys) as the A fragment straight from the S layout
    const uint32_t pa0 = pack_bf16x2(p[0][0], p[0][1]);
    const uint32_t pa2 = pack_bf16x2(p[1][0], p[1][1]);
    {
      const int mi = lane >> 3, rr = lane & 7;
      const int r = ro + (mi & 1) * 8 + rr;
#pragma unroll
      for (int np = 0; np < HD / 16; ++np) {
        const int half = np >> 2, ch = ((np & 3) << 1) + (mi >> 1);
        const uint32_t addr = sm100::smem_addr(tile(sub, 1, half)) + r * 128 + ((ch ^ (r & 7)) << 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma_16816(oacc[2 * np], pa0, 0u, pa2, 0u, b0, b1);
        mma_16816(oacc[2 * np + 1], pa0, 0u, pa2, 0u, b2, b3);
      }
    }
  }
  // the row sum over the quad's lanes
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

  // ---- abort path: every tile must land before the block leaves (bounded), then return (in a
  // cluster, only after the two cluster barriers every CTA of the cluster takes)
  if (abort_local) s_abort = 1;
  __syncthreads();
  if (s_abort) {
    if (threadIdx.x < nsub) {
      const uint64_t t0 = globaltimer_ns();
      while (!sm100::mbar_try_wait(&bars[threadIdx.x], 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
    __syncthreads();
    if constexpr (CLUSTER) {
      sm100::cluster_sync();
      sm100::cluster_sync();
    }
    return;
  }

  // ---- combine the 8 warps' states (the staging area is free now)
  float* wo = reinterpret_cast<float*>(dsm);                       // [warp][GROUP][HD]
  float* wm = wo + kWarps * GROUP * HD;                             // [warp][GROUP]
  float* wl = wm + kWarps * GROUP;
  if (qr < GROUP) {
#pragma unroll
    for (int nt = 0; nt < HD / 8; ++nt)
      *reinterpret_cast<float2*>(&wo[(warp * GROUP + qr) * HD + nt * 8 + 2 * qc]) =
          make_float2(oacc[nt][0], oacc[nt][1]);
    if (qc == 0) {
      wm[warp * GROUP + qr] = m_run;
      wl[warp * GROUP + qr] = l_run;
    }
  }
  __syncthreads();
  constexpr int V4 = HD / 4;
  for (int idx = threadIdx.x; idx < GROUP * V4; idx += blockDim.x) {
    const int a = idx / V4, e4 = idx - a * V4;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w * GROUP + a]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = wm[w * GROUP + a];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
      const float4 v = *reinterpret_cast<const float4*>(&wo[(w * GROUP + a) * HD + 4 * e4]);
      acc.x += f * v.x;
      acc.y += f * v.y;
      acc.z += f * v.z;
      acc.w += f * v.w;
      L += f * wl[w * GROUP + a];
    }
    if constexpr (CLUSTER) {
      *reinterpret_cast<float4*>(&s_res_o[a][4 * e4]) = acc;
      if (e4 == 0) {
        s_res_m[a] = M;
        s_res_l[a] = L;
      }
    } else {
      const int j = g * GROUP + a;
      float* rec = ml + ((bi * n_q + j) * gridDim.x + c) * kRec;
      *reinterpret_cast<float4*>(rec + 4 * e4) = acc;
      if (e4 == 0) {
        rec[HD] = M;
        rec[HD + 1] = L;
      }
    }
  }
  if constexpr (CLUSTER) {
    // The splits of this KV head are the cluster's CTAs (rank = split).  After the barrier, CTA r
    // merges its share of the GROUP x HD outputs from every split's shared memory, in split
    // order: o = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
    sm100::cluster_sync();
    const int splits = static_cast<int>(gridDim.x);
    const int rank = static_cast<int>(sm100::cluster_rank());
    constexpr int kOut = GROUP * HD;
    const int per = (kOut + splits - 1) / splits;
    const int i0 = rank * per;
    const int i1 = i0 + per < kOut ? i0 + per : kOut;
    for (int idx = i0 + threadIdx.x; idx < i1; idx += blockDim.x) {
      const int a = idx / HD, e = idx - a * HD;
      const uint32_t am = sm100::smem_addr(&s_res_m[a]);
      const uint32_t al = sm100::smem_addr(&s_res_l[a]);
      const uint32_t ao = sm100::smem_addr(&s_res_o[a][e]);
      float mc[kDecodeClusterMax], lc[kDecodeClusterMax], oc[kDecodeClusterMax];
#pragma unroll
      for (int cc = 0; cc < kDecodeClusterMax; ++cc) {
        if (cc < splits) {
          mc[cc] = sm100::ld_shared_cluster_f32(sm100::map_to_rank(am, cc));
          lc[cc] = sm100::ld_shared_cluster_f32(sm100::map_to_rank(al, cc));
          oc[cc] = sm100::ld_shared_cluster_f32(sm100::map_to_rank(ao, cc));
        }
      }
      float Mx = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < kDecodeClusterMax; ++cc)
        if (cc < splits) Mx = fmaxf(Mx, mc[cc]);
      float Ls = 0.f, acc = 0.f;
#pragma unroll
      for (int cc = 0; cc < kDecodeClusterMax; ++cc) {
        if (cc < splits) {
          const float f = mc[cc] == -INFINITY ? 0.f : exp2f(mc[cc] - Mx);
          Ls += f * lc[cc];
          acc += f * oc[cc];
        }
      }
      o[bi * static_cast<int64_t>(n_q) * HD + (g * GROUP + a) * HD + e] = from_f<__nv_bfloat16>(acc / Ls);
    }
    sm100::cluster_sync();   // no CTA leaves while a peer may still read its shared memory
  } else {
    merge_splits_if_last<__nv_bfloat16, GROUP, HD>(ml, counters, o, bi, g, n_q, n_kv);
  }
}

}  // namespace attn

// Decode attention with the splits of each KV head merged inside a cluster (one CTA per split).
// Tries the layout's split count, then fewer splits (longer chunks, up to the kernel's limit),
// and launches with the largest count whose clusters all fit on the device at once (one per
// sequence and KV head); *done tells the caller whether it launched.
template <int MAX_CHUNK, class Kern, class Args>
inline tp_status launch_decode_cluster(Kern kern, dim3 grid, size_t smem, const AttnLayout& L,
                                       cudaStream_t s, Args args, bool* done) {
  *done = false;
  if (L.kv_splits < 2) return TP_OK;
  static int fits[64][kDecodeClusterMax + 1];   // per device and cluster size; 0 = not queried
  int dev = 0;
  TP_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 64) return TP_OK;
  TP_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem)));
  TP_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  const int64_t n_keys = L.kv_len + 1;
  for (int64_t c = std::min<int64_t>(L.kv_splits, kDecodeClusterMax); c >= 2; --c) {
    const int64_t chunk = round_up(ceil_div(n_keys, c), 16);
    if (chunk > MAX_CHUNK) break;              // fewer splits only make the chunks longer
    if (ceil_div(n_keys, chunk) != c) continue;   // c splits of this chunk leave one empty
    int& fit = fits[dev][c];
    if (fit == 0) {
      cfg.gridDim = dim3(static_cast<unsigned>(c), grid.y, grid.z);
      attr[0].val.clusterDim.x = static_cast<unsigned>(c);
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
      }
      fit = n > 0 ? n : -1;
    }
    if (fit < L.b * L.n_kv) continue;
    cfg.gridDim = dim3(static_cast<unsigned>(c), grid.y, grid.z);
    attr[0].val.clusterDim.x = static_cast<unsigned>(c);
    cfg.numAttrs = 2;
    std::get<8>(args) = static_cast<int>(chunk);   // the kernel's chunk argument
    ProfScope prof(s, "attn_decode");
    const cudaError_t e = std::apply(
        [&](auto... a) { return cudaLaunchKernelEx(&cfg, kern, a...); }, args);
    if (e != cudaSuccess)
      return set_error(TP_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
    count_launch();
    *done = true;
    return TP_OK;
  }
  return TP_OK;
}

template <typename T>
inline tp_status attn_core(const AttnLayout& L, const void* qkv_v, void* o_v, void* kc, void* vc,
                           float* ml, int* counters, cudaStream_t s, float* lse = nullptr,
                           bool counters_zeroed = false) {
  const T* qkv = static_cast<const T*>(qkv_v);
  T* o = static_cast<T*>(o_v);
  attn::QkvIdx ix{L.p * L.R_a, L.R_a, L.qh, L.kh, L.hd, L.n_q / L.n_kv};
  const float scale = 1.0f / sqrtf(static_cast<float>(L.hd));
  if (L.kv_len == 0) {
    const bool tc = sizeof(T) == 2 && tensor_cores_usable() && (L.hd == 64 || L.hd == 128) &&
                    L.s <= INT32_MAX && L.b <= 65535 && ceil_div(L.s, fa::kRows) <= 65535;
    if (tc) {
      const int group = L.n_q / L.n_kv;
      if (L.hd == 128)
        return fa::launch<128>(qkv, L.b, L.s, L.n_q, L.qh, L.kh, group, L.R_a, L.p, L.causal, o, s,
                               lse);
      return fa::launch<64>(qkv, L.b, L.s, L.n_q, L.qh, L.kh, group, L.R_a, L.p, L.causal, o, s,
                            lse);
    }
    const int64_t warps = L.tokens * L.n_q;
    const int64_t blocks = ceil_div(warps * 32, 128);
    if (blocks > INT32_MAX) return set_error(TP_ERR_UNSUPPORTED, "attention grid too large");
    ProfScope prof(s, "attn_prefill");
    attn::prefill_simt_kernel<T><<<static_cast<unsigned>(blocks), 128, 0, s>>>(
        qkv, o, ix, L.b, L.s, L.n_q, L.causal, scale, lse);
    TP_LAUNCH_CHECK();
    return TP_OK;
  }
  // decode: split-KV attention that also appends the new key/value and merges its splits
  const int group = L.n_q / L.n_kv;
  dim3 grid(static_cast<unsigned>(L.kv_splits), static_cast<unsigned>(L.n_kv),
            static_cast<unsigned>(L.b));
  if (L.b > 65535) return set_error(TP_ERR_UNSUPPORTED, "decode batch above 65535");
  if (!counters_zeroed) {   // else the projection's launch cleared them
    const int64_t words = L.b * L.n_kv;
    TP_LAUNCH_PDL(zero_words_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(words, 256), 64))),
                  dim3(256), 0, s, reinterpret_cast<uint32_t*>(counters), words);
  }
  if constexpr (sizeof(T) == 2) {
    const bool mma = tensor_cores_usable() && (L.hd == 64 || L.hd == 128) &&
                     (group == 1 || group == 2 || group == 4 || group == 8) &&
                     L.kv_chunk <= (L.hd == 128 ? attn::DecodeMmaCfg<128>::kMaxChunk
                                                : attn::DecodeMmaCfg<64>::kMaxChunk) &&
                     L.kv_len <= INT32_MAX - 512 && L.b * L.n_kv <= INT32_MAX;
    if (mma) {
      // the caches as [b*n_kv][kv_len][hd]: the new token's slot and any slot past it read as zeros
      CUtensorMap km, vm;
      const uint64_t hd = static_cast<uint64_t>(L.hd);
      tp_status r = encode_tmap_bf16_3d(&km, kc, hd, static_cast<uint64_t>(L.kv_len),
                                        static_cast<uint64_t>(L.b * L.n_kv), hd * 2,
                                        static_cast<uint64_t>(L.kv_cap) * hd * 2, 64,
                                        attn::DecodeMmaCfg<128>::kSub);
      if (r != TP_OK) return r;
      r = encode_tmap_bf16_3d(&vm, vc, hd, static_cast<uint64_t>(L.kv_len),
                              static_cast<uint64_t>(L.b * L.n_kv), hd * 2,
                              static_cast<uint64_t>(L.kv_cap) * hd * 2, 64,
                              attn::DecodeMmaCfg<128>::kSub);
      if (r != TP_OK) return r;
#define TP_DECODE_MMA_CASE(G, H)                                                              \
      if (group == G && L.hd == H) {                                                          \
        const size_t smem = attn::DecodeMmaCfg<H>::kSmem;                                     \
        auto args = std::make_tuple(km, vm, reinterpret_cast<const __nv_bfloat16*>(qkv), ix,  \
                                    static_cast<__nv_bfloat16*>(kc),                          \
                                    static_cast<__nv_bfloat16*>(vc), L.kv_cap, L.kv_len,      \
                                    L.kv_chunk, L.n_q, L.n_kv, scale, ml, counters,           \
                                    reinterpret_cast<__nv_bfloat16*>(o), device_error_word()); \
        bool done = false;                                                                    \
        tp_status cst = launch_decode_cluster<attn::DecodeMmaCfg<H>::kMaxChunk>(                \
            attn::decode_mma_kernel<G, H, true>, grid, smem, L, s, args, &done);               \
        if (cst != TP_OK) return cst;                                                         \
        if (done) return TP_OK;                                                               \
        auto* kern = attn::decode_mma_kernel<G, H, false>;                                    \
        TP_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                                         static_cast<int>(smem)));                            \
        ProfScope prof(s, "attn_decode");                                                     \
        TP_LAUNCH_PDL(kern, grid, dim3(256), smem, s, km, vm,                                 \
                      reinterpret_cast<const __nv_bfloat16*>(qkv), ix,                        \
                      static_cast<__nv_bfloat16*>(kc), static_cast<__nv_bfloat16*>(vc),       \
                      L.kv_cap, L.kv_len, L.kv_chunk, L.n_q, L.n_kv, scale, ml, counters,     \
                      reinterpret_cast<__nv_bfloat16*>(o), device_error_word());             \
        return TP_OK;                                                                         \
      }
      TP_DECODE_MMA_CASE(8, 128) TP_DECODE_MMA_CASE(4, 128) TP_DECODE_MMA_CASE(2, 128)
      TP_DECODE_MMA_CASE(1, 128) TP_DECODE_MMA_CASE(8, 64) TP_DECODE_MMA_CASE(4, 64)
      TP_DECODE_MMA_CASE(2, 64) TP_DECODE_MMA_CASE(1, 64)
#undef TP_DECODE_MMA_CASE
    }
  }
#define TP_DECODE_CASE(G, H)                                                                  \
  if (group == G && L.hd == H) {                                                              \
    const size_t smem = attn::DecodeSmem<H, G, T>::bytes(L.kv_chunk);                         \
    TP_CUDA_TRY(cudaFuncSetAttribute(attn::decode_split_kernel<T, G, H>,                      \
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,             \
                                     static_cast<int>(smem)));                                \
    ProfScope prof(s, "attn_decode");                                                         \
    auto* kern = attn::decode_split_kernel<T, G, H>;                                          \
    TP_LAUNCH_PDL(kern, grid, dim3(256), smem, s, qkv, ix, static_cast<T*>(kc),               \
                  static_cast<T*>(vc), L.kv_cap, L.kv_len, L.kv_chunk, L.n_q, L.n_kv, scale,  \
                  ml, counters, o, device_error_word());                                      \
  } else
  TP_DECODE_CASE(8, 128) TP_DECODE_CASE(4, 128) TP_DECODE_CASE(2, 128) TP_DECODE_CASE(1, 128)
  TP_DECODE_CASE(8, 64) TP_DECODE_CASE(4, 64) TP_DECODE_CASE(2, 64) TP_DECODE_CASE(1, 64)
  TP_DECODE_CASE(1, 32) TP_DECODE_CASE(2, 32) TP_DECODE_CASE(4, 32) TP_DECODE_CASE(8, 32)
  {
    return set_error(TP_ERR_UNSUPPORTED,
                     "decode supports head_dim in {32, 64, 128} and n_q/n_kv in {1, 2, 4, 8}");
  }
#undef TP_DECODE_CASE
  return TP_OK;
}

namespace attn_tc {

inline tp_status qkv_proj(const AttnLayout& L, const void* x, const void* wqkv, void* qkv,
                          void* sk_ws, size_t sk_bytes, cudaStream_t s,
                          int* zero_also = nullptr, int64_t zero_also_words = 0) {
  const int64_t rows = L.p * L.R_a;
  tc::EpiHidden::Params ep;
  ep.h = static_cast<__nv_bfloat16*>(qkv);
  ep.z = nullptr;
  ep.ld_h = rows;
  ep.ld_z = 0;
  ep.tokens = static_cast<int32_t>(L.tokens);
  ep.rows = static_cast<int32_t>(rows);
  ep.act = TP_ACT_IDENTITY;
  const Operand xo{x, false, L.tokens, L.h, 1, L.h, 0};
  const Operand wo{wqkv, false, rows, L.h, 1, L.h, 0};
  if (L.tokens <= kSwapMaxT) {
    ep.swap = 1;
    const tc::StreamKArgs sk{false, sk_ws, sk_bytes};
    tc::GemmOpts opt;
    opt.sk = decode_stream_k(qkv_tiles(L), L.tokens, ceil_div(L.h, 64)) ? &sk : nullptr;
    opt.rotate_k = true;
    opt.zero_also = reinterpret_cast<uint32_t*>(zero_also);
    opt.zero_also_words = zero_also ? zero_also_words : 0;
    return by_tokens(L.tokens, [&](auto t) {
      return tc::run_gemm<typename decltype(t)::type, tc::EpiHiddenSwap>(wo, xo, rows, L.tokens, L.h, 1,
                                                                     ep, s, "attn_qkv_gemm", opt);
    });
  }
  if (zero_also && zero_also_words > 0)
    TP_LAUNCH_PDL(zero_words_kernel,
                  dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(zero_also_words, 256), 64))),
                  dim3(256), 0, s, reinterpret_cast<uint32_t*>(zero_also), zero_also_words);
  ep.swap = 0;
  return tc::run_gemm_pair<PP<false, false>, tc::EpiHidden>(xo, wo, L.tokens, rows, L.h, 1, ep, s,
                                                            "attn_qkv_gemm");
}

// Row-parallel output projection: fp32 partials [p][tokens][h] (separate reduce), or the fused
// in-order sum plus residual written straight to y.
inline tp_status out_proj(const AttnLayout& L, const void* o, const void* wo_p, float* part,
                          const void* residual, void* y, void* sk_ws, size_t sk_bytes,
                          cudaStream_t s) {
  const int64_t K = static_cast<int64_t>(L.qh) * L.hd;
  const Operand ao{o, false, L.tokens, K, L.p, static_cast<int64_t>(L.n_q) * L.hd, K};
  const Operand wo{wo_p, false, L.h, K, L.p, K, L.h * K};
  const bool swap = L.tokens <= kSwapMaxT;
  if (L.reduce_mode == TP_REDUCE_FUSED) {
    tc::EpiReduceOut::Params ep;
    ep.out = y;
    ep.residual = residual;
    ep.ld = L.h;
    ep.rows_valid = static_cast<int32_t>(L.tokens);
    ep.cols_valid = static_cast<int32_t>(L.h);
    ep.out_bf16 = L.y_dtype == TP_BF16 ? 1 : 0;
    ep.swap = swap ? 1 : 0;
    const tc::StreamKArgs sk{true, sk_ws, sk_bytes};
    tc::GemmOpts opt;
    opt.sk = &sk;
    opt.rotate_k = swap;
    if (swap)
      return by_tokens(L.tokens, [&](auto t) {
        return tc::run_gemm<typename decltype(t)::type, tc::EpiReduceOut>(
            wo, ao, L.h, L.tokens, K, L.p, ep, s, "attn_out_gemm", opt);
      });
    // prefill: each 256 x 256 tile runs the k-blocks of shard 0, 1, ..., p-1 into one
    // accumulator, so the shard sum never leaves TMEM
    return tc::run_gemm_pair<PP<false, false>, tc::EpiReduceOut>(ao, wo, L.tokens, L.h, K, L.p, ep,
                                                                 s, "attn_out_gemm", -1, true);
  }
  tc::EpiStoreF32::Params ep;
  ep.out = part;
  ep.ld = L.h;
  ep.batch_stride = L.tokens * L.h;
  ep.rows_valid = static_cast<int32_t>(L.tokens);
  ep.cols_valid = static_cast<int32_t>(L.h);
  if (swap) {
    ep.swap = 1;
    const tc::StreamKArgs sk{false, sk_ws, sk_bytes};
    tc::GemmOpts opt;
    opt.sk = decode_stream_k(out_tiles(L), L.tokens, ceil_div(static_cast<int64_t>(L.qh) * L.hd, 64)) ? &sk : nullptr;
    opt.rotate_k = true;
    return by_tokens(L.tokens, [&](auto t) {
      return tc::run_gemm<typename decltype(t)::type, tc::EpiStoreF32>(wo, ao, L.h, L.tokens, K, L.p,
                                                                       ep, s, "attn_out_gemm", opt);
    });
  }
  ep.swap = 0;
  return tc::run_gemm_pair<PP<false, false>, tc::EpiStoreF32>(ao, wo, L.tokens, L.h, K, L.p, ep, s,
                                                              "attn_out_gemm");
}
}  // namespace attn_tc

template <typename T>
inline tp_status attn_simt_proj(const AttnLayout& L, const void* x, const void* wqkv, void* qkv,
                                const void* o, const void* wo_p, float* part, cudaStream_t s,
                                bool first) {
  const int64_t P = L.p;
  simt::GemmArgs g{};
  if (first) {
    g.a = x; g.a_bs = 0; g.a_sm = L.h; g.a_sk = 1;
    g.b = wqkv; g.b_bs = 0; g.b_sm = L.h; g.b_sk = 1;
    g.out = qkv; g.o_bs = 0; g.o_sm = P * L.R_a; g.o_sn = 1;
    g.M = L.tokens; g.N = P * L.R_a; g.K = L.h; g.batch = 1; g.out_f32 = 0;
    return simt::gemm<T>(g, s);
  }
  const int64_t K = static_cast<int64_t>(L.qh) * L.hd;
  g.a = o; g.a_bs = K; g.a_sm = static_cast<int64_t>(L.n_q) * L.hd; g.a_sk = 1;
  g.b = wo_p; g.b_bs = L.h * K; g.b_sm = K; g.b_sk = 1;
  g.out = part; g.o_bs = L.tokens * L.h; g.o_sm = L.h; g.o_sn = 1;
  g.M = L.tokens; g.N = L.h; g.K = K; g.batch = P; g.out_f32 = 1;
  return simt::gemm<T>(g, s);
}

// With ``sp`` (sequence parallelism) the partials are reduce-scattered into the shards' token
// slices instead of summed into y (which, like residual and y_norm, is then unused).
inline tp_status attn_forward(const AttnLayout& L, const void* x, const void* wqkv,
                              const void* wo_p, void* kc, void* vc, const void* residual,
                              void* y, void* y_norm, void* ws, cudaStream_t s,
                              const seqpar::SpOut* sp = nullptr) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  void* qkv = w + L.qkv_off;
  void* o = w + L.o_off;
  float* part = reinterpret_cast<float*>(w + L.part_off);
  float* ml = reinterpret_cast<float*>(w + L.ml_off);
  int* counters = reinterpret_cast<int*>(w + L.cnt_off);
  tp_status st;
  if (L.tc) {
    if (!tensor_cores_usable())
      return set_error(TP_ERR_UNSUPPORTED, "bf16 tensor-core path needs an sm_100 device");
    for (const void* q : {x, wqkv, wo_p, residual, static_cast<const void*>(y)})
      if (q && (reinterpret_cast<uintptr_t>(q) & 15))
        return set_error(TP_ERR_INVALID_ARG, "bf16 pointers must be 16-byte aligned");
    void* sk = w + L.sk_off;
    const size_t skb = L.ws_bytes - L.sk_off;
    // decode: the projection's launch also clears the split-merge counters of the attention
    const bool dec = L.kv_len > 0;
    if ((st = attn_tc::qkv_proj(L, x, wqkv, qkv, sk, skb, s, dec ? counters : nullptr,
                                dec ? L.b * L.n_kv : 0)) != TP_OK)
      return st;
    if ((st = attn_core<__nv_bfloat16>(L, qkv, o, kc, vc, ml, counters, s, nullptr, dec)) != TP_OK)
      return st;
    if ((st = attn_tc::out_proj(L, o, wo_p, part, residual, y, sk, skb, s)) != TP_OK) return st;
    if (L.reduce_mode == TP_REDUCE_FUSED)
      return y_norm ? reduce::rmsnorm(y, L.y_dtype, L.tokens, L.h, L.norm_eps, y_norm, L.dtype, s)
                    : TP_OK;
  } else if (L.dtype == TP_BF16) {
    if ((st = attn_simt_proj<__nv_bfloat16>(L, x, wqkv, qkv, o, wo_p, part, s, true)) != TP_OK) return st;
    if ((st = attn_core<__nv_bfloat16>(L, qkv, o, kc, vc, ml, counters, s)) != TP_OK) return st;
    if ((st = attn_simt_proj<__nv_bfloat16>(L, x, wqkv, qkv, o, wo_p, part, s, false)) != TP_OK) return st;
  } else {
    if ((st = attn_simt_proj<float>(L, x, wqkv, qkv, o, wo_p, part, s, true)) != TP_OK) return st;
    if ((st = attn_core<float>(L, qkv, o, kc, vc, ml, counters, s)) != TP_OK) return st;
    if ((st = attn_simt_proj<float>(L, x, wqkv, qkv, o, wo_p, part, s, false)) != TP_OK) return st;
  }
  if (sp)
    return seqpar::reduce_scatter(part, L.p, L.tokens, L.h, sp->res, sp->y, L.y_dtype, sp->norm,
                                  L.dtype, L.norm_eps, s);
  if (y_norm)
    return reduce::reduce_norm(part, L.p, L.tokens, L.h, residual, y, L.y_dtype, y_norm, L.dtype,
                               L.norm_eps, s);
  return reduce::launch(part, TP_F32, L.p, L.tokens * L.h, residual, y, L.y_dtype, s);
}

}  // namespace tp
