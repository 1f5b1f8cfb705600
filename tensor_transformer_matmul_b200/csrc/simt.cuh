// CUDA-core (SIMT) kernels: the exact-fp32 path of the block, the path for shapes the tensor-core
// kernels cannot address (unaligned rows), and the elementwise steps those paths need.
#pragma once

#include "tp_common.cuh"

namespace tp {
namespace simt {

// D[b][m][n] = sum_k A(b, m, k) * B(b, n, k), fp32 accumulation, arbitrary element strides.
struct GemmArgs {
  const void* a; int64_t a_bs, a_sm, a_sk;
  const void* b; int64_t b_bs, b_sm, b_sk;
  void* out; int64_t o_bs, o_sm, o_sn;
  int64_t M, N, K, batch;
  int out_f32;   // 1: out is float, 0: out is the input element type
};

constexpr int kTile = 32;

template <typename T>
__global__ void __launch_bounds__(256) gemm_kernel(GemmArgs g) {
  __shared__ float As[kTile][kTile + 1];
  __shared__ float Bs[kTile][kTile + 1];
  const T* A = static_cast<const T*>(g.a);
  const T* B = static_cast<const T*>(g.b);
  const int64_t bz = blockIdx.z;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kTile;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kTile;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t k0 = 0; k0 < g.K; k0 += kTile) {
    for (int r = ty; r < kTile; r += 8) {
      const int64_t m = m0 + r, n = n0 + r, k = k0 + tx;
      As[r][tx] = (m < g.M && k < g.K) ? to_f(A[bz * g.a_bs + m * g.a_sm + k * g.a_sk]) : 0.f;
      Bs[r][tx] = (n < g.N && k < g.K) ? to_f(B[bz * g.b_bs + n * g.b_sm + k * g.b_sk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kTile; ++kk) {
      const float bv = Bs[tx][kk];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(As[ty + 8 * i][kk], bv, acc[i]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 8 * i, n = n0 + tx;
    if (m < g.M && n < g.N) {
      const int64_t o = bz * g.o_bs + m * g.o_sm + n * g.o_sn;
      if (g.out_f32) static_cast<float*>(g.out)[o] = acc[i];
      else static_cast<T*>(g.out)[o] = from_f<T>(acc[i]);
    }
  }
}

template <typename T>
inline tp_status gemm(const GemmArgs& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return TP_OK;
  if (ceil_div(g.M, kTile) > 65535 || g.batch > 65535)
    return set_error(TP_ERR_UNSUPPORTED, "SIMT GEMM grid too large");
  dim3 grid(static_cast<unsigned>(ceil_div(g.N, kTile)), static_cast<unsigned>(ceil_div(g.M, kTile)),
            static_cast<unsigned>(g.batch));
  ProfScope prof(s, "simt_gemm");
  gemm_kernel<T><<<grid, 256, 0, s>>>(g);
  TP_LAUNCH_CHECK();
  return TP_OK;
}

// Forward activation on packed pre-activations: z [T][p*R] (w1p row order) -> h [T][p*F_sp].
template <typename T>
__global__ void act_fwd_kernel(const T* z, T* h, int64_t T_, int p, int64_t R, int64_t F_sp,
                               int act) {
  const int64_t total = T_ * p * F_sp;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = idx / (p * F_sp);
    const int64_t rem = idx - t * p * F_sp;
    const int64_t i = rem / F_sp, c = rem - i * F_sp;
    const T* zr = z + t * p * R + i * R;
    float hv;
    if (act == TP_ACT_SWIGLU) {
      const int64_t zc = (c >> 7) * 256 + (c & 127);
      hv = silu_f(to_f(zr[zc])) * to_f(zr[zc + 128]);
    } else {
      hv = act_f(act, to_f(zr[c]));
    }
    h[idx] = from_f<T>(hv);
  }
}

// Backward activation: dh [T][p*F_sp] (fp32) and z -> dz [T][p*R] (w1p row order).
template <typename T>
__global__ void act_bwd_kernel(const float* dh, const T* z, T* dz, int64_t T_, int p, int64_t R,
                               int64_t F_sp, int act) {
  const int64_t total = T_ * p * F_sp;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = idx / (p * F_sp);
    const int64_t rem = idx - t * p * F_sp;
    const int64_t i = rem / F_sp, c = rem - i * F_sp;
    const int64_t base = t * p * R + i * R;
    const float d = dh[idx];
    if (act == TP_ACT_SWIGLU) {
      const int64_t zc = (c >> 7) * 256 + (c & 127);
      const float g = to_f(z[base + zc]), u = to_f(z[base + zc + 128]);
      dz[base + zc] = from_f<T>(d * u * silu_grad_f(g));
      dz[base + zc + 128] = from_f<T>(d * silu_f(g));
    } else {
      dz[base + c] = from_f<T>(d * act_grad_f(act, to_f(z[base + c])));
    }
  }
}

inline int elementwise_grid(int64_t total) {
  int64_t blocks = ceil_div(total, 256);
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  return static_cast<int>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace simt
}  // namespace tp
