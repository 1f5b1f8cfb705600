// Sequence-parallel collectives on one GPU.
//
// "Why tensor parallelism has to stay in scale-up" (Keysight), section "Where the 320 comes
// from": with sequence parallelism each all-reduce of the block becomes a reduce-scatter followed
// (before the next column-parallel matmul) by an all-gather; the bytes moved stay the same.
// Shard i owns token rows i*R .. i*R + R - 1 (R = T / p) of every [T][d] activation between the
// row-parallel output of one block and the column-parallel input of the next; the residual add
// and the normalisation run on those slices.
//
// With all shards on this GPU a slice is a separate [R][d] buffer (one per shard, anywhere in
// device memory), so the two collectives are:
//   reduce-scatter: slice_i = residual_i + sum_s part[s][i*R + r]   (fp32, shards in order 0..p-1,
//                   one rounding), optionally norm_i = RMSNorm(slice_i) row by row;
//   all-gather:     full[i*R + r] = slice_i[r].
#pragma once

#include <algorithm>
#include <string>

#include "reduce.cuh"
#include "tp_common.cuh"

namespace tp {
namespace seqpar {

constexpr int kMaxSlices = 64;

// device pointers of the p slices, passed by value
struct Slices {
  void* p[kMaxSlices];
};

// One block per token row, written into its shard's slice: reduce::reduce_norm_row (the plain
// reduce-and-norm kernel's row routine), so a slice equals the plain call's rows bit for bit.
constexpr int kRsThreads = reduce::kRowThreads;
template <typename Tout, typename Tn, bool VEC>
__global__ void __launch_bounds__(kRsThreads, 3) reduce_scatter_rows_kernel(
    const float* __restrict__ part, int p, int64_t rows, int64_t d, int64_t R, Slices res,
    int has_res, Slices out, Slices norm, int has_norm, float eps) {
  pdl_wait();   // programmatic dependent launch: global memory only from here on
  pdl_trigger();
  __shared__ float red[kRsThreads / 32];
  const int64_t r = blockIdx.x;
  const int sl = static_cast<int>(r / R);
  const int64_t lr = r - static_cast<int64_t>(sl) * R;
  Tout* orow = static_cast<Tout*>(out.p[sl]) + lr * d;
  const Tout* rrow = has_res ? static_cast<const Tout*>(res.p[sl]) + lr * d : nullptr;
  Tn* nrow = has_norm ? static_cast<Tn*>(norm.p[sl]) + lr * d : nullptr;
  reduce::reduce_norm_row<float, Tout, Tn, VEC>(part + r * d, p, rows * d, d, rrow, orow, nrow,
                                                eps, red);
}

// full[i*R + r] = slice_i[r]: block (x, i) copies 16-byte words of slice i (W: the slice's size
// in words), grid-stride over x.
static __global__ void __launch_bounds__(256) all_gather_words_kernel(Slices src, int64_t words,
                                                                uint4* __restrict__ full) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.y;
  const uint4* s = static_cast<const uint4*>(src.p[i]);
  uint4* d = full + static_cast<int64_t>(i) * words;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < words; w += stride)
    d[w] = s[w];
}
// the same, element by element (sizes or addresses not multiples of 16 bytes)
static __global__ void __launch_bounds__(256) all_gather_bytes_kernel(Slices src, int64_t bytes,
                                                                uint8_t* __restrict__ full) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.y;
  const uint8_t* s = static_cast<const uint8_t*>(src.p[i]);
  uint8_t* d = full + static_cast<int64_t>(i) * bytes;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < bytes; w += stride)
    d[w] = s[w];
}

inline bool all_aligned16(const Slices& s, int p) {
  for (int i = 0; i < p; ++i)
    if (reinterpret_cast<uintptr_t>(s.p[i]) & 15) return false;
  return true;
}

// Checks shared by the entry points: p slices, T divisible by p, non-null pointers.
inline tp_status check_slices(int p, int64_t T, void* const* ptrs, const char* what) {
  if (p < 1 || p > kMaxSlices) return set_error(TP_ERR_SHAPE, "p must be 1..64 for slices");
  if (T % p) return set_error(TP_ERR_SHAPE, "sequence parallelism needs p to divide the tokens");
  if (!ptrs) return set_error(TP_ERR_INVALID_ARG, std::string(what) + " is null");
  for (int i = 0; i < p; ++i)
    if (!ptrs[i]) return set_error(TP_ERR_INVALID_ARG, std::string(what) + " has a null slice");
  return TP_OK;
}

// What a block entry point writes instead of the full output when it runs sequence-parallel:
// per shard slice, the residual to add (or null), the output and its RMSNorm (or null).
struct SpOut {
  void* const* res;
  void* const* y;
  void* const* norm;
};

inline Slices to_slices(void* const* ptrs, int p) {
  Slices s{};
  for (int i = 0; i < p && ptrs; ++i) s.p[i] = ptrs[i];
  return s;
}

template <typename Tout, typename Tn>
inline void rs_launch(const float* part, int p, int64_t T, int64_t d, const Slices& res,
                      bool has_res, const Slices& out, const Slices& norm, bool has_norm,
                      float eps, bool vec, cudaStream_t s) {
  const int64_t R = T / p;
  if (vec)
    (void)launch_pdl(reduce_scatter_rows_kernel<Tout, Tn, true>, dim3(static_cast<unsigned>(T)),
                     dim3(kRsThreads), 0, s, part, p, T, d, R, res, has_res ? 1 : 0, out, norm,
                     has_norm ? 1 : 0, eps);
  else
    (void)launch_pdl(reduce_scatter_rows_kernel<Tout, Tn, false>, dim3(static_cast<unsigned>(T)),
                     dim3(kRsThreads), 0, s, part, p, T, d, R, res, has_res ? 1 : 0, out, norm,
                     has_norm ? 1 : 0, eps);
}

// Reduce-scatter of the fp32 partials [p][T][d] of p shards into the p shards' token slices.
inline tp_status reduce_scatter(const float* part, int p, int64_t T, int64_t d,
                                void* const* res, void* const* out, int out_dtype,
                                void* const* norm, int norm_dtype, float eps, cudaStream_t s) {
  if (T == 0 || d == 0) return TP_OK;
  if (T > INT32_MAX) return set_error(TP_ERR_UNSUPPORTED, "too many rows");
  const Slices so = to_slices(out, p), sr = to_slices(res, p), sn = to_slices(norm, p);
  const bool vec = d % 8 == 0 && (reinterpret_cast<uintptr_t>(part) & 15) == 0 &&
                   all_aligned16(so, p) && (!res || all_aligned16(sr, p));
  ProfScope prof(s, "reduce_scatter");
  const bool ob = out_dtype == TP_BF16, nb = norm_dtype == TP_BF16;
  const bool hr = res != nullptr, hn = norm != nullptr;
  if (ob && nb) rs_launch<__nv_bfloat16, __nv_bfloat16>(part, p, T, d, sr, hr, so, sn, hn, eps, vec, s);
  else if (ob) rs_launch<__nv_bfloat16, float>(part, p, T, d, sr, hr, so, sn, hn, eps, vec, s);
  else if (nb) rs_launch<float, __nv_bfloat16>(part, p, T, d, sr, hr, so, sn, hn, eps, vec, s);
  else rs_launch<float, float>(part, p, T, d, sr, hr, so, sn, hn, eps, vec, s);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

// All-gather of p slices of ``slice_bytes`` each into the contiguous ``full``.
inline tp_status all_gather(const void* const* slices, int p, int64_t slice_bytes, void* full,
                            cudaStream_t s) {
  if (slice_bytes == 0) return TP_OK;
  if (p > 65535) return set_error(TP_ERR_UNSUPPORTED, "too many slices");
  const Slices src = to_slices(const_cast<void* const*>(slices), p);
  const bool vec = slice_bytes % 16 == 0 && all_aligned16(src, p) &&
                   (reinterpret_cast<uintptr_t>(full) & 15) == 0;
  const int64_t work = vec ? slice_bytes / 16 : slice_bytes;
  int64_t bx = ceil_div(work, 256);
  const int64_t cap = std::max<int64_t>(1, static_cast<int64_t>(num_sms()) * 8 / p);
  if (bx > cap) bx = cap;
  ProfScope prof(s, "all_gather");
  const dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(p));
  if (vec)
    (void)launch_pdl(all_gather_words_kernel, grid, dim3(256), 0, s, src, work,
                     static_cast<uint4*>(full));
  else
    (void)launch_pdl(all_gather_bytes_kernel, grid, dim3(256), 0, s, src, work,
                     static_cast<uint8_t*>(full));
  TP_LAUNCH_CHECK();
  return TP_OK;
}

}  // namespace seqpar
}  // namespace tp
