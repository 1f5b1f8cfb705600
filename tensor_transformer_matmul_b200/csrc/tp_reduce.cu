// The all-reduce's arithmetic on one GPU -- the in-order sum of p partials, with the optional
// residual add -- and the replicated RMSNorm that follows it.
//   "How does tensor parallelism split a transformer feed-forward block's two matmuls",
//   "One collective"; "Tensor Parallelism" (klaylearn), Notes: Y = sum_i Z_i.
#include "reduce.cuh"
#include "seqpar.cuh"

extern "C" tp_status tp_reduce_partials(const void* partials, int32_t p, int64_t n,
                                        int32_t in_dtype, const void* residual, void* out,
                                        int32_t out_dtype, void* stream) {
  tp::clear_error();
  if (p < 1) return tp::set_error(TP_ERR_SHAPE, "p must be >= 1");
  if (n < 0) return tp::set_error(TP_ERR_INVALID_ARG, "n must be >= 0");
  if ((in_dtype != TP_F32 && in_dtype != TP_BF16) || (out_dtype != TP_F32 && out_dtype != TP_BF16))
    return tp::set_error(TP_ERR_INVALID_ARG, "dtype must be TP_F32 or TP_BF16");
  if (n > 0 && (!partials || !out)) return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  tp_status st = tp::reduce::launch(partials, in_dtype, p, n, residual, out, out_dtype,
                                    static_cast<cudaStream_t>(stream));
  if (st == TP_OK) tp::count_reduction();
  return st;
}

extern "C" tp_status tp_rmsnorm(const void* x, int32_t x_dtype, int64_t rows, int64_t d,
                                float eps, void* out, int32_t out_dtype, void* stream) {
  tp::clear_error();
  if (rows < 0 || d < 1) return tp::set_error(TP_ERR_SHAPE, "rows >= 0 and d >= 1 required");
  if ((x_dtype != TP_F32 && x_dtype != TP_BF16) || (out_dtype != TP_F32 && out_dtype != TP_BF16))
    return tp::set_error(TP_ERR_INVALID_ARG, "dtype");
  if (!(eps >= 0.f)) return tp::set_error(TP_ERR_INVALID_ARG, "eps must be >= 0");
  if (rows > 0 && (!x || !out)) return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  return tp::reduce::rmsnorm(x, x_dtype, rows, d, eps, out, out_dtype,
                             static_cast<cudaStream_t>(stream));
}

// Sequence-parallel collectives: "Why tensor parallelism has to stay in scale-up" (Keysight),
// "Where the 320 comes from" -- each all-reduce becomes a reduce-scatter plus an all-gather.
extern "C" tp_status tp_reduce_scatter_partials(const void* partials, int32_t p, int64_t T,
                                                int64_t d, void* const* residual_slices,
                                                void* const* out_slices, int32_t out_dtype,
                                                void* const* norm_slices, int32_t norm_dtype,
                                                float eps, void* stream) {
  tp::clear_error();
  if (T < 0 || d < 1) return tp::set_error(TP_ERR_SHAPE, "T >= 0 and d >= 1 required");
  tp_status st = tp::seqpar::check_slices(p, T, out_slices, "out_slices");
  if (st != TP_OK) return st;
  if (residual_slices && (st = tp::seqpar::check_slices(p, T, residual_slices, "residual_slices")) != TP_OK)
    return st;
  if (norm_slices && (st = tp::seqpar::check_slices(p, T, norm_slices, "norm_slices")) != TP_OK)
    return st;
  if ((out_dtype != TP_F32 && out_dtype != TP_BF16) || (norm_dtype != TP_F32 && norm_dtype != TP_BF16))
    return tp::set_error(TP_ERR_INVALID_ARG, "dtype must be TP_F32 or TP_BF16");
  if (!(eps >= 0.f)) return tp::set_error(TP_ERR_INVALID_ARG, "eps must be >= 0");
  if (T > 0 && !partials) return tp::set_error(TP_ERR_INVALID_ARG, "partials is null");
  st = tp::seqpar::reduce_scatter(static_cast<const float*>(partials), p, T, d, residual_slices,
                                  out_slices, out_dtype, norm_slices, norm_dtype, eps,
                                  static_cast<cudaStream_t>(stream));
  if (st == TP_OK) tp::count_reduction();
  return st;
}

extern "C" tp_status tp_all_gather_slices(const void* const* slices, int32_t p,
                                          int64_t rows_per_slice, int64_t d, int32_t dtype,
                                          void* out, void* stream) {
  tp::clear_error();
  if (rows_per_slice < 0 || d < 1) return tp::set_error(TP_ERR_SHAPE, "rows >= 0 and d >= 1 required");
  if (dtype != TP_F32 && dtype != TP_BF16) return tp::set_error(TP_ERR_INVALID_ARG, "dtype");
  tp_status st = tp::seqpar::check_slices(p, static_cast<int64_t>(p) * rows_per_slice,
                                          const_cast<void* const*>(slices), "slices");
  if (st != TP_OK) return st;
  if (rows_per_slice > 0 && !out) return tp::set_error(TP_ERR_INVALID_ARG, "out is null");
  return tp::seqpar::all_gather(slices, p, rows_per_slice * d * tp::elem_bytes(dtype), out,
                                static_cast<cudaStream_t>(stream));
}
