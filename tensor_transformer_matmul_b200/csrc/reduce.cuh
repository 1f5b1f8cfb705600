// Partial-sum reduce and RMSNorm kernels (HBM-bound, vectorised, coalesced).
#pragma once

#include "sm100.cuh"
#include "tp_common.cuh"

namespace tp {
namespace reduce {

template <typename T> struct Vec8;
template <> struct Vec8<float> {
  __device__ __forceinline__ static void load(const float* p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  __device__ __forceinline__ static void store(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};
template <> struct Vec8<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    v[0] = bf16lo(w.x); v[1] = bf16hi(w.x); v[2] = bf16lo(w.y); v[3] = bf16hi(w.y);
    v[4] = bf16lo(w.z); v[5] = bf16hi(w.z); v[6] = bf16lo(w.w); v[7] = bf16hi(w.w);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]); w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]); w.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = w;
  }
};

// out[j] = res[j] + sum_{s=0}^{p-1} part[s*n + j]   (fp32, in order, one rounding)
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) reduce_vec8_kernel(const Tin* __restrict__ part, int p,
                                                          int64_t n, const Tout* res,
                                                          Tout* out) {
  pdl_wait();   // programmatic dependent launch: global memory only from here on
  pdl_trigger();
  const int64_t nv = n >> 3;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nv;
       i += stride) {
    float acc[8];
    Vec8<Tin>::load(part + 8 * i, acc);
    for (int s = 1; s < p; ++s) {
      float v[8];
      Vec8<Tin>::load(part + static_cast<int64_t>(s) * n + 8 * i, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += v[e];
    }
    if (res) {
      float r[8];
      Vec8<Tout>::load(res + 8 * i, r);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = r[e] + acc[e];
    }
    Vec8<Tout>::store(out + 8 * i, acc);
  }
}

// Same sum for p <= PMAX: all p loads are issued before the first add (more bytes in flight);
// the additions still run in the order 0..p-1.
template <typename Tin, typename Tout, int PMAX>
__global__ void __launch_bounds__(256) reduce_vec8_small_kernel(const Tin* __restrict__ part,
                                                                int p, int64_t n,
                                                                const Tout* res, Tout* out) {
  pdl_wait();   // programmatic dependent launch: global memory only from here on
  pdl_trigger();
  const int64_t nv = n >> 3;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nv;
       i += stride) {
    float v[PMAX][8];
#pragma unroll
    for (int s = 0; s < PMAX; ++s)
      if (s < p) Vec8<Tin>::load(part + static_cast<int64_t>(s) * n + 8 * i, v[s]);
    float r[8];
    if (res) Vec8<Tout>::load(res + 8 * i, r);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = v[0][e];
#pragma unroll
    for (int s = 1; s < PMAX; ++s)
      if (s < p) {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += v[s][e];
      }
    if (res) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = r[e] + acc[e];
    }
    Vec8<Tout>::store(out + 8 * i, acc);
  }
}

template <typename Tin, typename Tout>
__global__ void reduce_scalar_kernel(const Tin* part, int p, int64_t n, const Tout* res,
                                     Tout* out) {
  pdl_wait();   // programmatic dependent launch: global memory only from here on
  pdl_trigger();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < n; j += stride) {
    float acc = to_f(part[j]);
    for (int s = 1; s < p; ++s) acc += to_f(part[static_cast<int64_t>(s) * n + j]);
    if (res) acc = to_f(res[j]) + acc;
    out[j] = from_f<Tout>(acc);
  }
}

template <typename Tin, typename Tout>
inline tp_status launch_t(const void* part, int p, int64_t n, const void* res, void* out,
                          cudaStream_t s) {
  if (n == 0) return TP_OK;
  const bool vec = (n % 8 == 0) && (reinterpret_cast<uintptr_t>(part) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(out) % 16 == 0) &&
                   (!res || reinterpret_cast<uintptr_t>(res) % 16 == 0);
  const int64_t work = vec ? n / 8 : n;
  int64_t blocks = ceil_div(work, 256);
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  ProfScope prof(s, "reduce_partials");
  if (vec && p <= 8)
    (void)launch_pdl(reduce_vec8_small_kernel<Tin, Tout, 8>, dim3(static_cast<unsigned>(blocks)),
                     dim3(256), 0, s, static_cast<const Tin*>(part), p, n,
                     static_cast<const Tout*>(res), static_cast<Tout*>(out));
  else if (vec)
    (void)launch_pdl(reduce_vec8_kernel<Tin, Tout>, dim3(static_cast<unsigned>(blocks)), dim3(256),
                     0, s, static_cast<const Tin*>(part), p, n, static_cast<const Tout*>(res),
                     static_cast<Tout*>(out));
  else
    (void)launch_pdl(reduce_scalar_kernel<Tin, Tout>, dim3(static_cast<unsigned>(blocks)),
                     dim3(256), 0, s, static_cast<const Tin*>(part), p, n,
                     static_cast<const Tout*>(res), static_cast<Tout*>(out));
  TP_LAUNCH_CHECK();
  return TP_OK;
}

inline tp_status launch(const void* part, int in_dtype, int p, int64_t n, const void* res,
                        void* out, int out_dtype, cudaStream_t s) {
  if (in_dtype == TP_F32 && out_dtype == TP_F32) return launch_t<float, float>(part, p, n, res, out, s);
  if (in_dtype == TP_F32 && out_dtype == TP_BF16)
    return launch_t<float, __nv_bfloat16>(part, p, n, res, out, s);
  if (in_dtype == TP_BF16 && out_dtype == TP_F32)
    return launch_t<__nv_bfloat16, float>(part, p, n, res, out, s);
  return launch_t<__nv_bfloat16, __nv_bfloat16>(part, p, n, res, out, s);
}

// One row of "reduce, then normalise": out = res + sum_s part[s] (fp32, shards in order, one
// rounding), then norm = out / sqrt(mean(out^2) + eps) of the stored (rounded) out values.  The
// block's threads split the row; ``prow`` is the row in partial 0 (partial s at + s*n).
// VEC (d % 8 == 0, 16-byte aligned rows): 8 consecutive elements per thread and access; the
// partials are loaded four at a time, every load of a group issued before its adds, which run in
// the order 0..p-1.  Used by the plain and the sequence-parallel reduce-and-norm kernels,
// so that both give the same bits for the same row.
constexpr int kRowThreads = 256;
template <typename Tin, typename Tout, typename Tn, bool VEC>
__device__ __forceinline__ void reduce_norm_row(const Tin* __restrict__ prow, int p, int64_t n,
                                                int64_t d, const Tout* rrow, Tout* orow,
                                                Tn* nrow, float eps, float* red) {
  float ss = 0.f;
  if (VEC) {
    for (int64_t j = 8 * static_cast<int64_t>(threadIdx.x); j < d; j += 8 * blockDim.x) {
      float acc[8];
      for (int g = 0; g < p; g += 4) {
        float v[4][8];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (g + q < p) Vec8<Tin>::load(prow + static_cast<int64_t>(g + q) * n + j, v[q]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (g + q >= p) break;
          if (g + q == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = v[0][e];
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += v[q][e];
          }
        }
      }
      if (rrow) {
        float r[8];
        Vec8<Tout>::load(rrow + j, r);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = r[e] + acc[e];
      }
      Vec8<Tout>::store(orow + j, acc);
#pragma unroll
      for (int e = 0; e < 8; ++e) {   // the stored, rounded value
        const float y = to_f(from_f<Tout>(acc[e]));
        ss = fmaf(y, y, ss);
      }
    }
  } else {
    for (int64_t j = threadIdx.x; j < d; j += blockDim.x) {
      float acc = to_f(prow[j]);
      for (int q = 1; q < p; ++q) acc += to_f(prow[static_cast<int64_t>(q) * n + j]);
      if (rrow) acc = to_f(rrow[j]) + acc;
      const Tout y = from_f<Tout>(acc);
      orow[j] = y;
      const float yv = to_f(y);
      ss = fmaf(yv, yv, ss);
    }
  }
  if (!nrow) return;   // block-uniform
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float scale = rsqrtf(red[0] / static_cast<float>(d) + eps);
  if (VEC) {
    // the same elements this thread stored: its own writes, read back in order
    for (int64_t j = 8 * static_cast<int64_t>(threadIdx.x); j < d; j += 8 * blockDim.x) {
      float y[8];
      Vec8<Tout>::load(orow + j, y);
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] *= scale;
      Vec8<Tn>::store(nrow + j, y);
    }
  } else {
    for (int64_t j = threadIdx.x; j < d; j += blockDim.x)
      nrow[j] = from_f<Tn>(to_f(orow[j]) * scale);
  }
}

// One row per block: reduce_norm_row over rows of [rows][d].
template <typename Tin, typename Tout, typename Tn, bool VEC>
__global__ void __launch_bounds__(kRowThreads, 3) reduce_norm_rows_kernel(
    const Tin* __restrict__ part, int p, int64_t rows, int64_t d, const Tout* res, Tout* out,
    Tn* norm, float eps) {
  pdl_wait();   // programmatic dependent launch: global memory only from here on
  pdl_trigger();
  __shared__ float red[kRowThreads / 32];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * d;
  reduce_norm_row<Tin, Tout, Tn, VEC>(part + base, p, rows * d, d, res ? res + base : nullptr,
                                      out + base, norm + base, eps, red);
}

template <typename Tin, typename Tout, typename Tn>
inline void reduce_norm_launch(const void* part, int p, int64_t rows, int64_t d, const void* res,
                               void* out, void* norm, float eps, cudaStream_t s) {
  const bool vec = p <= 8 && d % 8 == 0 && (reinterpret_cast<uintptr_t>(part) & 31) == 0 &&
                   (reinterpret_cast<uintptr_t>(out) & 15) == 0 &&
                   (!res || (reinterpret_cast<uintptr_t>(res) & 15) == 0);
  if (vec)
    (void)launch_pdl(reduce_norm_rows_kernel<Tin, Tout, Tn, true>, dim3(static_cast<unsigned>(rows)),
                     dim3(kRowThreads), 0, s, static_cast<const Tin*>(part), p, rows, d,
                     static_cast<const Tout*>(res), static_cast<Tout*>(out),
                     static_cast<Tn*>(norm), eps);
  else
    (void)launch_pdl(reduce_norm_rows_kernel<Tin, Tout, Tn, false>,
                     dim3(static_cast<unsigned>(rows)), dim3(kRowThreads), 0, s,
                     static_cast<const Tin*>(part), p, rows, d, static_cast<const Tout*>(res),
                     static_cast<Tout*>(out), static_cast<Tn*>(norm), eps);
}

// Few rows: "reduce, then normalise" with one cluster of kNormCluster CTAs per row.  CTA c of
// the cluster takes columns [c*w, (c+1)*w) of the row: it adds the partials in shard order and then
// the residual (fp32, one rounding), stores y, and sums the squares of its stored values.  The CTAs
// exchange these sums through distributed shared memory; each adds all of them in rank order, so
// every CTA gets the same scale, and normalises its own columns from registers.  One kernel
// replaces the sum over all rows*d elements followed by the row-split RMSNorm.
constexpr int kNormCluster = 8;
constexpr int kNormThreads = 128;
constexpr int kNormVecs = 2;   // 8-element vectors per thread: d <= 8 * 128 * 8 * 2 = 16384
template <typename Tout, typename Tn>
__global__ void __launch_bounds__(kNormThreads) reduce_norm_cluster_kernel(
    const float* __restrict__ part, int p, int64_t n, int64_t d, int w, const Tout* res, Tout* out,
    Tn* norm, float eps) {
  pdl_wait();   // programmatic dependent launch: global memory only from here on
  pdl_trigger();
  __shared__ float red[kNormThreads / 32];
  __shared__ float s_part;
  __shared__ float s_all[kNormCluster];
  const uint32_t rank = sm100::cluster_rank();
  const int64_t base = static_cast<int64_t>(blockIdx.y) * d;
  const int64_t c0 = static_cast<int64_t>(rank) * w;
  const int64_t c1 = c0 + w < d ? c0 + w : d;
  float y[kNormVecs][8];
  float ss = 0.f;
#pragma unroll
  for (int v = 0; v < kNormVecs; ++v) {
    const int64_t j = c0 + 8 * (static_cast<int64_t>(threadIdx.x) + v * kNormThreads);
    if (j >= c1) continue;
    float acc[8];
    for (int g = 0; g < p; g += 8) {   // up to 8 partials in flight, added in order 0..p-1
      float pv[8][8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (g + q < p) Vec8<float>::load(part + static_cast<int64_t>(g + q) * n + base + j, pv[q]);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (g + q >= p) break;
        if (g + q == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = pv[0][e];
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] += pv[q][e];
        }
      }
    }
    if (res) {
      float r[8];
      Vec8<Tout>::load(res + base + j, r);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = r[e] + acc[e];
    }
    Vec8<Tout>::store(out + base + j, acc);
#pragma unroll
    for (int e = 0; e < 8; ++e) {   // the stored, rounded value
      y[v][e] = to_f(from_f<Tout>(acc[e]));
      ss = fmaf(y[v][e], y[v][e], ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < kNormThreads / 32; ++i) t += red[i];
    s_part = t;
  }
  sm100::cluster_sync();   // every CTA's s_part is written and visible to the cluster
  if (threadIdx.x < kNormCluster)
    s_all[threadIdx.x] =
        sm100::ld_shared_cluster_f32(sm100::map_to_rank(sm100::smem_addr(&s_part), threadIdx.x));
  sm100::cluster_sync();   // every peer has read this CTA's s_part (it may exit after this)
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kNormCluster; ++i) tot += s_all[i];
  const float scale = rsqrtf(tot / static_cast<float>(d) + eps);
#pragma unroll
  for (int v = 0; v < kNormVecs; ++v) {
    const int64_t j = c0 + 8 * (static_cast<int64_t>(threadIdx.x) + v * kNormThreads);
    if (j >= c1) continue;
#pragma unroll
    for (int e = 0; e < 8; ++e) y[v][e] *= scale;
    Vec8<Tn>::store(norm + base + j, y[v]);
  }
}

inline bool reduce_norm_cluster_ok(const void* part, int64_t rows, int64_t d, const void* res,
                                   const void* out, const void* norm) {
  return rows > 0 && rows < num_sms() && rows <= 65535 && d % 8 == 0 &&
         d <= static_cast<int64_t>(kNormCluster) * kNormThreads * 8 * kNormVecs &&
         ((reinterpret_cast<uintptr_t>(part) | reinterpret_cast<uintptr_t>(res) |
           reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(norm)) & 15) == 0;
}

template <typename Tout, typename Tn>
inline cudaError_t reduce_norm_cluster_launch(const float* part, int p, int64_t rows, int64_t d,
                                              const void* res, void* out, void* norm, float eps,
                                              cudaStream_t s) {
  const int w = static_cast<int>(round_up(ceil_div(d, kNormCluster), 8));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kNormCluster, static_cast<unsigned>(rows));
  cfg.blockDim = dim3(kNormThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kNormCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, reduce_norm_cluster_kernel<Tout, Tn>, part, p, rows * d, d, w,
                            static_cast<const Tout*>(res), static_cast<Tout*>(out),
                            static_cast<Tn*>(norm), eps);
}

inline tp_status rmsnorm(const void* x, int in_dtype, int64_t rows, int64_t d, float eps,
                         void* out, int out_dtype, cudaStream_t s);
inline bool rmsnorm_split_ok(const void* x, int64_t rows, int64_t d, const void* out);

// y = res + sum of fp32 partials [p][rows][d]; norm = RMSNorm(y) in norm_dtype
inline tp_status reduce_norm(const float* part, int p, int64_t rows, int64_t d, const void* res,
                             void* out, int out_dtype, void* norm, int norm_dtype, float eps,
                             cudaStream_t s) {
  if (rows == 0) return TP_OK;
  if (rows > INT32_MAX) return set_error(TP_ERR_UNSUPPORTED, "too many rows");
  if (reduce_norm_cluster_ok(part, rows, d, res, out, norm)) {
    // few rows: one row per block would leave most SMs idle, so each row is spread over a
    // cluster of CTAs that share the row's sum of squares
    ProfScope prof(s, "reduce_partials");
    const bool ob = out_dtype == TP_BF16, nb = norm_dtype == TP_BF16;
    cudaError_t e;
    if (ob && nb) e = reduce_norm_cluster_launch<__nv_bfloat16, __nv_bfloat16>(part, p, rows, d, res, out, norm, eps, s);
    else if (ob) e = reduce_norm_cluster_launch<__nv_bfloat16, float>(part, p, rows, d, res, out, norm, eps, s);
    else if (nb) e = reduce_norm_cluster_launch<float, __nv_bfloat16>(part, p, rows, d, res, out, norm, eps, s);
    else e = reduce_norm_cluster_launch<float, float>(part, p, rows, d, res, out, norm, eps, s);
    if (e != cudaSuccess)
      return set_error(TP_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
    count_launch();
    return TP_OK;
  }
  if (rmsnorm_split_ok(out, rows, d, norm)) {
    // few rows with a shape the cluster kernel does not take: the plain vectorised reduce over
    // all rows*d elements, then the row-split norm (both read the stored, rounded y, as the
    // one-kernel path does)
    tp_status st = launch(part, TP_F32, p, rows * d, res, out, out_dtype, s);
    if (st != TP_OK) return st;
    return rmsnorm(out, out_dtype, rows, d, eps, norm, norm_dtype, s);
  }
  ProfScope prof(s, "reduce_partials");
  const bool ob = out_dtype == TP_BF16, nb = norm_dtype == TP_BF16;
  if (ob && nb) reduce_norm_launch<float, __nv_bfloat16, __nv_bfloat16>(part, p, rows, d, res, out, norm, eps, s);
  else if (ob) reduce_norm_launch<float, __nv_bfloat16, float>(part, p, rows, d, res, out, norm, eps, s);
  else if (nb) reduce_norm_launch<float, float, __nv_bfloat16>(part, p, rows, d, res, out, norm, eps, s);
  else reduce_norm_launch<float, float, float>(part, p, rows, d, res, out, norm, eps, s);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

// out[r] = x[r] / sqrt(mean(x[r]^2) + eps), one block per row.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const Tin* x, int64_t d, float eps,
                                                      Tout* out) {
  pdl_wait();   // programmatic dependent launch: global memory only from here on
  pdl_trigger();
  __shared__ float red[8];
  const Tin* xr = x + blockIdx.x * d;
  Tout* orow = out + blockIdx.x * d;
  float ss = 0.f;
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) {
    const float v = to_f(xr[j]);
    ss = fmaf(v, v, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float scale = rsqrtf(red[0] / static_cast<float>(d) + eps);
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) orow[j] = from_f<Tout>(to_f(xr[j]) * scale);
}

template <typename Tin, typename Tout>
inline void rmsnorm_launch(const void* x, int64_t rows, int64_t d, float eps, void* out,
                           cudaStream_t s) {
  (void)launch_pdl(rmsnorm_kernel<Tin, Tout>, dim3(static_cast<unsigned>(rows)), dim3(256), 0, s,
                   static_cast<const Tin*>(x), d, eps, static_cast<Tout*>(out));
}

// RMSNorm for few rows (fewer than SMs): block (c, r) recomputes the sum of squares of the whole
// row r, vectorised and in a fixed order (so every block of a row gets the same scale), and
// normalises columns [c*W, (c+1)*W) of it.  Needs d % 8 == 0 and 16-byte aligned rows.
constexpr int kSplitW = 512;
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) rmsnorm_split_kernel(const Tin* __restrict__ x, int64_t d,
                                                            float eps, Tout* __restrict__ out) {
  pdl_wait();   // programmatic dependent launch: global memory only from here on
  pdl_trigger();
  __shared__ float red[8];
  const Tin* xr = x + static_cast<int64_t>(blockIdx.y) * d;
  Tout* orow = out + static_cast<int64_t>(blockIdx.y) * d;
  float ss = 0.f;
  for (int64_t j = 8 * static_cast<int64_t>(threadIdx.x); j < d; j += 8 * blockDim.x) {
    float v[8];
    Vec8<Tin>::load(xr + j, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float scale = rsqrtf(red[0] / static_cast<float>(d) + eps);
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kSplitW;
  const int64_t c1 = c0 + kSplitW < d ? c0 + kSplitW : d;
  for (int64_t j = c0 + 8 * static_cast<int64_t>(threadIdx.x); j < c1; j += 8 * blockDim.x) {
    float v[8];
    Vec8<Tin>::load(xr + j, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] *= scale;
    Vec8<Tout>::store(orow + j, v);
  }
}

template <typename Tin, typename Tout>
inline void rmsnorm_split_launch(const void* x, int64_t rows, int64_t d, float eps, void* out,
                                 cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(ceil_div(d, kSplitW)), static_cast<unsigned>(rows));
  (void)launch_pdl(rmsnorm_split_kernel<Tin, Tout>, grid, dim3(256), 0, s,
                   static_cast<const Tin*>(x), d, eps, static_cast<Tout*>(out));
}

inline bool rmsnorm_split_ok(const void* x, int64_t rows, int64_t d, const void* out) {
  return rows > 0 && rows < num_sms() && d % 8 == 0 && rows <= 65535 &&
         ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15) == 0;
}

inline tp_status rmsnorm(const void* x, int in_dtype, int64_t rows, int64_t d, float eps,
                         void* out, int out_dtype, cudaStream_t s) {
  if (rows == 0) return TP_OK;
  if (rows > INT32_MAX) return set_error(TP_ERR_UNSUPPORTED, "too many rows");
  ProfScope prof(s, "rmsnorm");
  const bool ib = in_dtype == TP_BF16, ob = out_dtype == TP_BF16;
  if (rmsnorm_split_ok(x, rows, d, out)) {   // few rows: spread each row over many blocks
    if (ib && ob) rmsnorm_split_launch<__nv_bfloat16, __nv_bfloat16>(x, rows, d, eps, out, s);
    else if (ib) rmsnorm_split_launch<__nv_bfloat16, float>(x, rows, d, eps, out, s);
    else if (ob) rmsnorm_split_launch<float, __nv_bfloat16>(x, rows, d, eps, out, s);
    else rmsnorm_split_launch<float, float>(x, rows, d, eps, out, s);
  } else if (ib && ob) rmsnorm_launch<__nv_bfloat16, __nv_bfloat16>(x, rows, d, eps, out, s);
  else if (ib) rmsnorm_launch<__nv_bfloat16, float>(x, rows, d, eps, out, s);
  else if (ob) rmsnorm_launch<float, __nv_bfloat16>(x, rows, d, eps, out, s);
  else rmsnorm_launch<float, float>(x, rows, d, eps, out, s);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace reduce
}  // namespace tp
