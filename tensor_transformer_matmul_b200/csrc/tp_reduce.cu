// The all-reduce's arithmetic on one GPU -- the in-order sum of p partials, with the optional
// residual add -- and the replicated RMSNorm that follows it.
//   "How does tensor parallelism split a transformer feed-forward block's two matmuls",
//   "One collective"; "Tensor Parallelism" (klaylearn), Notes: Y = sum_i Z_i.
#include "reduce.cuh"

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
