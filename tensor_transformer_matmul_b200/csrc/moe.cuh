// Kernels of the tensor-parallel mixture-of-experts block (routing, dispatch, combine).
//
// "Tensor-parallel all-reduce count per transformer layer in MLX shard_linear" (llms-explorer),
// facts on MoE layers: the router stays replicated, the routed experts and the shared expert are
// sharded in place, and the block makes one sum of the shards' outputs (the shared expert's slice
// folded in); a sharded-to-all linear adds its bias once, after the sum.
//
// Per call, on the device:
//   logits = x Wr (tcgen05 GEMM, fp32)  ->  top-k per token, weights = softmax of the k chosen
//   logits  ->  per expert, its (token, choice) entries in token order (counts, offsets, a stable
//   position for every entry)  ->  gather of the routed token rows into expert order  ->  grouped
//   up / down GEMMs over all experts (gemm_tc.cuh, grouped mode; the down GEMM runs the p shards'
//   k-blocks of a row tile into one accumulator, so the shard sum -- the block's one reduction --
//   happens there, as it does in the shared expert's fused down GEMM)  ->  one combine: shared
//   expert + weighted routed rows (choices in order) + bias, then the residual.
#pragma once

#include "reduce.cuh"
#include "tp_common.cuh"

namespace tp {
namespace moe {

constexpr int kMaxTopK = 8;

// Router logits for few experts (E not a multiple of 64): block t, thread q*E + e sums
// x[t][k] Wr[k][e] over k = q, q + Q, ... (Q = blockDim / E; consecutive threads read
// consecutive Wr elements), then thread e adds the Q partial sums in order.  fp32.
__global__ void __launch_bounds__(256) router_simt_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const __nv_bfloat16* __restrict__ wr,
                                                          int64_t d, int E,
                                                          float* __restrict__ logits) {
  pdl_wait();
  pdl_trigger();
  __shared__ float part[256];
  const int64_t t = blockIdx.x;
  const int Q = static_cast<int>(blockDim.x) / E;
  const int e = threadIdx.x % E, q = threadIdx.x / E;
  float acc = 0.f;
  if (q < Q)
    for (int64_t k = q; k < d; k += Q)
      acc = fmaf(__bfloat162float(x[t * d + k]), __bfloat162float(wr[k * E + e]), acc);
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < E) {
    float v = 0.f;
    for (int j = 0; j < Q; ++j) v += part[j * E + threadIdx.x];
    logits[t * E + threadIdx.x] = v;
  }
}

// One warp per token: the k largest logits (descending; among equal logits the lower expert
// index first) and their softmax.  Lane L reads logits L, L + 32, ... (coalesced across the warp)
// and keeps its own k largest in that order; then k rounds of a warp-wide maximum (ties: the
// lower index) take the next entry from the lane that holds it.  The result, and the softmax
// computed from it by lane 0 in choice order, are those of a sequential scan over all E logits.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int64_t T,
                                                   int E, int k, int32_t* __restrict__ idx,
                                                   float* __restrict__ w) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;   // warp-uniform
  const float* l = logits + t * E;
  float best[kMaxTopK];
  int bi[kMaxTopK];
  int nkept = 0;
  for (int e = lane; e < E; e += 32) {
    const float v = l[e];
    if (nkept == k && !(v > best[k - 1])) continue;   // not above this lane's k-th
    // insertion after every kept entry with a logit >= v (this lane's indices ascend)
    int pos = nkept < k ? nkept : k - 1;
    while (pos > 0 && best[pos - 1] < v) {
      best[pos] = best[pos - 1];
      bi[pos] = bi[pos - 1];
      --pos;
    }
    best[pos] = v;
    bi[pos] = e;
    if (nkept < k) ++nkept;
  }
  int head = 0;
  float ch_v[kMaxTopK];
  int ch_i[kMaxTopK];
  for (int j = 0; j < k; ++j) {
    float v = head < nkept ? best[head] : -INFINITY;
    int i = head < nkept ? bi[head] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, v, o);
      const int oi = __shfl_xor_sync(0xffffffffu, i, o);
      if (ov > v || (ov == v && oi < i)) {
        v = ov;
        i = oi;
      }
    }
    ch_v[j] = v;
    ch_i[j] = i;
    if (head < nkept && bi[head] == i) ++head;   // the lane that held it moves on
  }
  if (lane == 0) {
    float s = 0.f, ex[kMaxTopK];
    for (int j = 0; j < k; ++j) {
      ex[j] = expf(ch_v[j] - ch_v[0]);
      s += ex[j];
    }
    for (int j = 0; j < k; ++j) {
      idx[t * k + j] = ch_i[j];
      w[t * k + j] = ex[j] / s;
    }
  }
}

__device__ __forceinline__ int block_sum_int(int v, int* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  int tot = 0;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) tot += red[i];
  __syncthreads();
  return tot;
}

// Block e: cnt[e] = number of entries routed to expert e.
__global__ void __launch_bounds__(1024) count_kernel(const int32_t* __restrict__ idx,
                                                     int64_t n_entries, int32_t* __restrict__ cnt) {
  pdl_wait();
  pdl_trigger();
  __shared__ int red[32];
  const int e = blockIdx.x;
  int c = 0;
  for (int64_t i = threadIdx.x; i < n_entries; i += blockDim.x) c += idx[i] == e ? 1 : 0;
  c = block_sum_int(c, red);
  if (threadIdx.x == 0) cnt[e] = c;
}

// Exclusive prefix sum of v over the block (threads in index order); red holds 32 ints.
__device__ __forceinline__ int block_exclusive_scan_int(int v, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int nw = static_cast<int>(blockDim.x >> 5);
    int w = lane < nw ? red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    if (lane < nw) red[lane] = w;   // inclusive totals of warps 0..lane
  }
  __syncthreads();
  const int before = (warp > 0 ? red[warp - 1] : 0) + inc - v;
  __syncthreads();   // red is reused by the caller
  return before;
}

// Block e: off[e] = sum of the counts of experts < e and mbp[e] = sum of their block_rows-row
// blocks (the last block also writes mbp[E], the total); then every entry routed to e gets the
// next position in entry order: perm[off + pos] = entry, inv[entry] = off + pos (a stable order,
// so the dispatch is deterministic).  Thread t owns a contiguous range of the entries: it counts
// its hits, an exclusive scan over the block gives its first position, and a second pass over
// the same range writes them.
__global__ void __launch_bounds__(1024) position_kernel(const int32_t* __restrict__ idx,
                                                        int64_t n_entries,
                                                        const int32_t* __restrict__ cnt,
                                                        int block_rows,
                                                        int32_t* __restrict__ off,
                                                        int32_t* __restrict__ mbp,
                                                        int32_t* __restrict__ perm,
                                                        int32_t* __restrict__ inv) {
  pdl_wait();
  pdl_trigger();
  __shared__ int red[32];
  const int e = blockIdx.x;
  int o = 0, nb = 0;
  for (int i = threadIdx.x; i < e; i += blockDim.x) {
    o += cnt[i];
    nb += (cnt[i] + block_rows - 1) / block_rows;
  }
  const int base0 = block_sum_int(o, red);
  const int blocks0 = block_sum_int(nb, red);
  if (threadIdx.x == 0) {
    off[e] = base0;
    mbp[e] = blocks0;
    if (e == static_cast<int>(gridDim.x) - 1) mbp[e + 1] = blocks0 + (cnt[e] + block_rows - 1) / block_rows;
  }
  const int64_t per = (n_entries + blockDim.x - 1) / blockDim.x;
  const int64_t i0 = static_cast<int64_t>(threadIdx.x) * per;
  const int64_t i1 = i0 + per < n_entries ? i0 + per : n_entries;
  int c = 0;
  for (int64_t i = i0; i < i1; ++i) c += idx[i] == e ? 1 : 0;
  int slot = base0 + block_exclusive_scan_int(c, red);
  if (c > 0)
    for (int64_t i = i0; i < i1; ++i)
      if (idx[i] == e) {
        perm[slot] = static_cast<int32_t>(i);
        inv[i] = slot;
        ++slot;
      }
}

// xs[r] = x[perm[r] / k] for the n_rows routed rows: one warp per row, 16-byte words
// (d % 8 == 0).
constexpr int kGatherRowsPerBlock = 8;
__global__ void __launch_bounds__(32 * kGatherRowsPerBlock) gather_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ perm, int k, int64_t d,
    int64_t n_rows, __nv_bfloat16* __restrict__ xs) {
  pdl_wait();
  pdl_trigger();
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kGatherRowsPerBlock + (threadIdx.x >> 5);
  if (r >= n_rows) return;
  const int64_t t = perm[r] / k;
  const uint4* src = reinterpret_cast<const uint4*>(x + t * d);
  uint4* dst = reinterpret_cast<uint4*>(xs + r * d);
  for (int64_t j = threadIdx.x & 31; j < d / 8; j += 32) dst[j] = src[j];
}

// y[t] = residual[t] + ((shared[t] + sum_{j<k} w[t][j] * routed[inv[t k + j]]) + bias): the
// routed rows and the shared expert arrive with their p shards already summed (in order, inside
// their GEMMs' accumulators); the choices are added in order, all in fp32 with one rounding.
// 8 consecutive columns per thread (d % 8 == 0).
__global__ void __launch_bounds__(256) combine_kernel(
    const float* __restrict__ routed, const float* __restrict__ shared,
    const int32_t* __restrict__ inv, const float* __restrict__ w, int k, int64_t T, int64_t d,
    const __nv_bfloat16* __restrict__ bias, const __nv_bfloat16* residual, __nv_bfloat16* y) {
  pdl_wait();
  pdl_trigger();
  const int64_t nv = T * (d / 8);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < nv; q += stride) {
    const int64_t t = q / (d / 8);
    const int64_t c = (q - t * (d / 8)) * 8;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (shared) {
      const float4* s4 = reinterpret_cast<const float4*>(shared + t * d + c);
      const float4 a = s4[0], b = s4[1];
      acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
      acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
    }
    // all choices' indices and weights first, then all their rows, so that the loads of the
    // k rows are in flight together; the sum still runs over the choices in order
    float wt[kMaxTopK];
    int64_t rr[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      wt[j] = j < k ? w[t * k + j] : 0.f;
      rr[j] = j < k ? inv[t * k + j] : 0;
    }
    float4 ra[kMaxTopK], rb[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k) {
        const float4* r4 = reinterpret_cast<const float4*>(routed + rr[j] * d + c);
        ra[j] = r4[0];
        rb[j] = r4[1];
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k) {
        const float v[8] = {ra[j].x, ra[j].y, ra[j].z, ra[j].w, rb[j].x, rb[j].y, rb[j].z, rb[j].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(wt[j], v[e], acc[e]);
      }
    }
    if (bias) {
      const uint4 bw = *reinterpret_cast<const uint4*>(bias + c);
      const float bv[8] = {bf16lo(bw.x), bf16hi(bw.x), bf16lo(bw.y), bf16hi(bw.y),
                           bf16lo(bw.z), bf16hi(bw.z), bf16lo(bw.w), bf16hi(bw.w)};
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += bv[e];
    }
    if (residual) {
      const uint4 rw = *reinterpret_cast<const uint4*>(residual + t * d + c);
      const float rv[8] = {bf16lo(rw.x), bf16hi(rw.x), bf16lo(rw.y), bf16hi(rw.y),
                           bf16lo(rw.z), bf16hi(rw.z), bf16lo(rw.w), bf16hi(rw.w)};
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = rv[e] + acc[e];
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(y + t * d + c) = o;
  }
}

// ------------------------------------------------------------------------------ backward
// dw[t k + j] = <dy_t, o[inv[t k + j]]>: the gradient of routing weight w_tj (o: the routed
// rows' outputs, fp32 [row][d]).  One warp per (token, choice); fp32 sum.
__global__ void __launch_bounds__(256) route_weight_grad_kernel(
    const __nv_bfloat16* __restrict__ dy, const float* __restrict__ o,
    const int32_t* __restrict__ inv, int k, int64_t T, int64_t d, float* __restrict__ dw) {
  pdl_wait();
  pdl_trigger();
  const int64_t q = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (q >= T * k) return;
  const int64_t t = q / k;
  const __nv_bfloat16* g = dy + t * d;
  const float* r = o + static_cast<int64_t>(inv[q]) * d;
  float acc = 0.f;
  for (int64_t c = 8 * lane; c < d; c += 256) {
    float gv[8], rv[8];
    reduce::Vec8<__nv_bfloat16>::load(g + c, gv);
    reduce::Vec8<float>::load(r + c, rv);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc = fmaf(gv[e], rv[e], acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dw[q] = acc;
}

// dl[t][e] = w_tj (dw_tj - sum_i w_ti dw_ti) when e = idx[t][j], else 0: the gradient of the
// router logits through the softmax over each token's k chosen logits (bf16 [T][E]).
__global__ void __launch_bounds__(256) router_logit_grad_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ w, const float* __restrict__ dw,
    int k, int64_t T, int E, __nv_bfloat16* __restrict__ dl) {
  pdl_wait();
  pdl_trigger();
  const int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (q >= T * E) return;
  const int64_t t = q / E;
  const int e = static_cast<int>(q - t * E);
  float s = 0.f, v = 0.f;
  for (int j = 0; j < k; ++j) s = fmaf(w[t * k + j], dw[t * k + j], s);
  for (int j = 0; j < k; ++j)
    if (idx[t * k + j] == e) v = w[t * k + j] * (dw[t * k + j] - s);
  dl[q] = __float2bfloat16_rn(v);
}

// gs[r] = w[perm[r]] * dy[perm[r] / k] (bf16), the routed rows' output gradients in expert
// order: one warp per row, 8 columns per lane and step (d % 8 == 0).
__global__ void __launch_bounds__(32 * kGatherRowsPerBlock) gather_scaled_kernel(
    const __nv_bfloat16* __restrict__ dy, const int32_t* __restrict__ perm,
    const float* __restrict__ w, int k, int64_t d, int64_t n_rows,
    __nv_bfloat16* __restrict__ gs) {
  pdl_wait();
  pdl_trigger();
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kGatherRowsPerBlock + (threadIdx.x >> 5);
  if (r >= n_rows) return;
  const int32_t entry = perm[r];
  const float sc = w[entry];
  const __nv_bfloat16* src = dy + static_cast<int64_t>(entry / k) * d;
  __nv_bfloat16* dst = gs + r * d;
  for (int64_t c = 8 * (threadIdx.x & 31); c < d; c += 256) {
    float v[8];
    reduce::Vec8<__nv_bfloat16>::load(src + c, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] *= sc;
    reduce::Vec8<__nv_bfloat16>::store(dst + c, v);
  }
}

// dx[t] = (sum_{j<k} dxs[inv[t k + j]] + dxr[t]) + dxsh[t]: the routed rows' input gradients
// (choices in order), the router's and the shared expert's (optional), fp32, one rounding.
__global__ void __launch_bounds__(256) dx_combine_kernel(
    const float* __restrict__ dxs, const float* __restrict__ dxr, const float* __restrict__ dxsh,
    const int32_t* __restrict__ inv, int k, int64_t T, int64_t d, __nv_bfloat16* __restrict__ dx) {
  pdl_wait();
  pdl_trigger();
  const int64_t nv = T * (d / 8);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < nv; q += stride) {
    const int64_t t = q / (d / 8);
    const int64_t c = (q - t * (d / 8)) * 8;
    // every choice's row is loaded before the in-order sum, so the k loads are in flight together
    float vr[kMaxTopK][8];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) reduce::Vec8<float>::load(dxs + static_cast<int64_t>(inv[t * k + j]) * d + c, vr[j]);
    float acc[8], v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = vr[0][e];
#pragma unroll
    for (int j = 1; j < kMaxTopK; ++j) {
      if (j < k) {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += vr[j][e];
      }
    }
    reduce::Vec8<float>::load(dxr + t * d + c, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += v[e];
    if (dxsh) {
      reduce::Vec8<float>::load(dxsh + t * d + c, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += v[e];
    }
    reduce::Vec8<__nv_bfloat16>::store(dx + t * d + c, acc);
  }
}

}  // namespace moe
}  // namespace tp
