// Shard-layout packers: copy user weights W[in][out] into the per-shard device layouts of
// tp_block.h, and scatter packed gradients back.  All are tiled transposes through shared memory
// (coalesced on both sides).  Pure data movement: bit-exact.
#pragma once

#include "tp_common.cuh"

namespace tp {
namespace pack {

constexpr int kT = 32;

// Column map of a "rows of the packed matrix are columns of the user matrices" layout: packed
// row r reads column col of source src (ld elements per source row), or is zero when src < 0.
struct ColMap {
  // segments of one shard's rows, in order: [0, seg_end[0]) from source 0, ...; the kind selects
  // the index arithmetic
  int kind;            // 0: plain (W1 / one matrix), 1: SwiGLU gate/up blocks, 2: Q|K|V
  int64_t R;           // packed rows per shard
  int64_t F_s;         // valid features per shard (kinds 0/1)
  int64_t q_rows, k_rows;            // kind 2: rows from Wq, then Wk, then Wv per shard
  const void* src[3];
  int64_t ld[3];
  __device__ __forceinline__ void map(int64_t r, int& s, int64_t& col) const {
    const int64_t i = r / R, rr = r - i * R;
    if (kind == 0) {
      s = rr < F_s ? 0 : -1;
      col = i * F_s + rr;
    } else if (kind == 1) {
      const int64_t blk = rr >> 8, o = rr & 255;
      const int64_t f = blk * 128 + (o & 127);
      s = f < F_s ? (o < 128 ? 0 : 1) : -1;
      col = i * F_s + f;
    } else {
      if (rr < q_rows) { s = 0; col = i * q_rows + rr; }
      else if (rr < q_rows + k_rows) { s = 1; col = i * k_rows + (rr - q_rows); }
      else { s = 2; col = i * k_rows + (rr - q_rows - k_rows); }
    }
  }
};

// out[r][k] = src_s(r)[k][col(r)] for r < rows, k < K.
template <typename T>
__global__ void pack_cols_kernel(T* out, int64_t rows, int64_t K, ColMap cm) {
  __shared__ T tile[kT][kT + 1];
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kT, k0 = static_cast<int64_t>(blockIdx.y) * kT;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int j = ty; j < kT; j += 8) {
    const int64_t r = r0 + tx, k = k0 + j;
    T v = from_f<T>(0.f);
    if (r < rows && k < K) {
      int s; int64_t col;
      cm.map(r, s, col);
      if (s >= 0) v = static_cast<const T*>(cm.src[s])[k * cm.ld[s] + col];
    }
    tile[j][tx] = v;
  }
  __syncthreads();
  for (int j = ty; j < kT; j += 8) {
    const int64_t r = r0 + j, k = k0 + tx;
    if (r < rows && k < K) out[r * K + k] = tile[tx][j];
  }
}

// out[i][n][c] = (c < Ks) ? src[(i*Ks + c) * ld + n] : 0  for i < p, n < nrows, c < Kp.
// (Row-parallel weights: shard i's row slice, transposed.)
template <typename T>
__global__ void pack_rows_kernel(T* out, int p, int64_t nrows, int64_t Kp, int64_t Ks,
                                 const T* src, int64_t ld) {
  __shared__ T tile[kT][kT + 1];
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kT, c0 = static_cast<int64_t>(blockIdx.y) * kT;
  const int64_t i = blockIdx.z;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int j = ty; j < kT; j += 8) {
    const int64_t c = c0 + j, n = n0 + tx;
    T v = from_f<T>(0.f);
    if (c < Ks && n < nrows) v = src[(i * Ks + c) * ld + n];
    tile[j][tx] = v;
  }
  __syncthreads();
  for (int j = ty; j < kT; j += 8) {
    const int64_t n = n0 + j, c = c0 + tx;
    if (n < nrows && c < Kp) out[(i * nrows + n) * Kp + c] = tile[tx][j];
  }
}

// Inverse of pack_cols for fp32 gradients: dst_s[k][col] = in[r][k] for every valid packed row r
// (each valid (s, col) is hit by exactly one r).  Tiles run over packed rows.
static __global__ void unpack_cols_kernel(const float* in, int64_t rows, int64_t K, ColMap cm,
                                   float* dst0, float* dst1, float* dst2) {
  __shared__ float tile[kT][kT + 1];
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kT, k0 = static_cast<int64_t>(blockIdx.y) * kT;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int j = ty; j < kT; j += 8) {
    const int64_t r = r0 + j, k = k0 + tx;
    tile[j][tx] = (r < rows && k < K) ? in[r * K + k] : 0.f;
  }
  __syncthreads();
  for (int j = ty; j < kT; j += 8) {
    const int64_t r = r0 + tx, k = k0 + j;
    if (r < rows && k < K) {
      int s; int64_t col;
      cm.map(r, s, col);
      float* d = s == 0 ? dst0 : (s == 1 ? dst1 : (s == 2 ? dst2 : nullptr));
      if (d) d[k * cm.ld[s] + col] = tile[tx][j];
    }
  }
}

// Inverse of pack_rows for fp32: dst[(i*Ks + c) * ld + n] = in[i][n][c] for c < Ks.
static __global__ void unpack_rows_kernel(const float* in, int p, int64_t nrows, int64_t Kp, int64_t Ks,
                                   float* dst, int64_t ld) {
  __shared__ float tile[kT][kT + 1];
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kT, c0 = static_cast<int64_t>(blockIdx.y) * kT;
  const int64_t i = blockIdx.z;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int j = ty; j < kT; j += 8) {
    const int64_t n = n0 + j, c = c0 + tx;
    tile[j][tx] = (n < nrows && c < Kp) ? in[(i * nrows + n) * Kp + c] : 0.f;
  }
  __syncthreads();
  for (int j = ty; j < kT; j += 8) {
    const int64_t c = c0 + j, n = n0 + tx;
    if (c < Ks && n < nrows) dst[(i * Ks + c) * ld + n] = tile[tx][j];
  }
}

inline bool grid_ok(int64_t gx, int64_t gy, int64_t gz) {
  return gx > 0 && gx < (1ll << 31) && gy > 0 && gy <= 65535 && gz > 0 && gz <= 65535;
}

}  // namespace pack
}  // namespace tp
