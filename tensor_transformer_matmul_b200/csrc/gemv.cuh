// Decode GEMV for a handful of tokens: out[t][r] = sum_k W[r][k] x[t][k] over the packed, K-major
// weights of the tensor-parallel block.
//
// With one to four tokens the block's matmuls are matrix-vector products that read every weight
// byte once and do two flops per byte per token: HBM-bound work.  So instead of tensor-core tiles
// (whose 128-row M side and N >= 16 would pad the token count sixteen-fold) they run as a
// streaming kernel laid out for coalescing and balance:
//   * the weights of all rows (all shards) form one sequence of 512-byte "steps" (256 bf16 of one
//     row; every K here is a multiple of 256, so a step never straddles two rows);
//   * every warp of a grid that is resident all at once (4 blocks of 8 warps per SM) takes an
//     equal contiguous range of steps: lane l reads 16 bytes at l*16 of each step, with eight (one
//     or two tokens) or four steps' weight loads in flight per lane;
//   * a warp keeps fp32 dot products per token for its current row and, where the row changes or
//     its range ends, reduces them over the lanes and writes one "piece" of that row;
//   * a fix-up kernel adds each row's pieces in warp order (so in k order: deterministic) and
//     applies the epilogue (activation, bf16 store, or fp32 partial store).
// x is read through the read-only path (its rows are small and stay in L1/L2).
#pragma once

#include "tp_common.cuh"

namespace tp {
namespace gemv {

constexpr int kMaxT = 4;              // tokens handled here
constexpr int kThreads = 256;
constexpr int kBlocksPerSm = 4;       // resident together (launch bounds cap the registers)
constexpr int kStep = 256;            // elements of one warp step (16 bytes per lane)
constexpr size_t kMaxStagedX = 48 * 1024;   // x staged per block (fp32): K <= 12288
// weight steps whose loads a lane keeps in flight: 128 (T <= 2) or 64 bytes per lane, i.e.
// 128 or 64 KB per SM
template <int T>
constexpr int unroll() { return T <= 2 ? 8 : 4; }
static_assert(kMaxT <= 4, "the unroll and register budget assume at most four tokens");

// Operand set: W [batch][rows][K] bf16 (row stride K, batch stride rows*K); x for batch b at
// x + b*x_bs, token t at + t*x_ts.
struct Args {
  const __nv_bfloat16* w;
  const __nv_bfloat16* x;
  int64_t rows;          // rows per batch
  int64_t K;             // multiple of 256
  int64_t batch;
  int64_t x_bs, x_ts;    // element strides of x
  int T;
  int64_t steps_per_warp;
  int max_pieces;
  float* pieces;         // [batch*rows][max_pieces][T]
};

// Steps of the whole problem and the warps of the grid.
struct Plan {
  int64_t total_steps, warps, steps_per_warp;
  int max_pieces, blocks;
  size_t pieces_bytes;
};

inline Plan plan(int64_t rows, int64_t K, int64_t batch, int T, int sms) {
  Plan P;
  const int64_t spr = K / kStep;
  P.total_steps = batch * rows * spr;
  P.blocks = sms * kBlocksPerSm;
  P.warps = static_cast<int64_t>(P.blocks) * (kThreads / 32);
  P.steps_per_warp = std::max<int64_t>(1, (P.total_steps + P.warps - 1) / P.warps);
  // a row of spr steps meets at most ceil((spr - 1) / C) + 1 warp ranges
  P.max_pieces = static_cast<int>((spr - 1 + P.steps_per_warp - 1) / P.steps_per_warp + 1);
  P.pieces_bytes = static_cast<size_t>(batch * rows) * P.max_pieces * T * sizeof(float);
  return P;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int T>
__global__ void __launch_bounds__(kThreads, kBlocksPerSm) gemv_kernel(Args a) {
  constexpr int kUnroll = unroll<T>();
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t spr = a.K / kStep;
  const int64_t s_begin = warp * a.steps_per_warp;
  const int64_t total = a.batch * a.rows * spr;
  const int64_t s_end = min(total, s_begin + a.steps_per_warp);
  if (s_begin >= s_end) return;
  float acc[T];
#pragma unroll
  for (int t = 0; t < T; ++t) acc[t] = 0.f;
  int64_t cur_row = s_begin / spr;
  // the warp whose range holds the row's first step: this warp's piece index is its distance
  auto flush = [&](int64_t row) {
#pragma unroll
    for (int t = 0; t < T; ++t) {
      float v = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[t] = 0.f;
      if (lane == 0) {
        const int64_t first = (row * spr) / a.steps_per_warp;
        const int64_t piece = warp - first;
        a.pieces[(row * a.max_pieces + piece) * T + t] = v;
      }
    }
  };
  // (row, kst): the next step to load; the row's batch offset of x changes only with the row
  int64_t row = cur_row;
  int kst = static_cast<int>(s_begin - cur_row * spr);
  int64_t xb = (cur_row / a.rows) * a.x_bs;
  const int spr32 = static_cast<int>(spr);
  for (int64_t left = s_end - s_begin; left > 0; left -= kUnroll) {
    // the weight loads of kUnroll steps first (the HBM stream), then, walking the same steps
    // again, the x loads (L1/L2 hits) and the FMAs
    uint4 wv[kUnroll];
    const int64_t row0 = row;
    const int kst0 = kst;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (u < left) {
        wv[u] = __ldcs(reinterpret_cast<const uint4*>(a.w + row * a.K + kst * kStep + lane * 8));
        if (++kst == spr32) {
          kst = 0;
          ++row;
        }
      }
    }
    int64_t r = row0;
    int kc = kst0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (u >= left) break;                                // warp-uniform
      if (r != cur_row) {
        flush(cur_row);
        cur_row = r;
        xb = (cur_row / a.rows) * a.x_bs;
      }
      const int k = kc * kStep + lane * 8;
      float wf[8];
      bf16x8_to_f32(wv[u], wf);
#pragma unroll
      for (int t = 0; t < T; ++t) {
        float xf[8];
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a.x + xb + t * a.x_ts + k)), xf);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[t] = fmaf(wf[e], xf[e], acc[t]);
      }
      if (++kc == spr32) {
        kc = 0;
        ++r;
      }
    }
  }
  flush(cur_row);
}

// One token and one batch (the column-parallel projections): x is staged once per block in shared
// memory as fp32, so a step costs one 16-byte weight load, its bf16 -> fp32 unpacking, two shared
// loads and four packed fp32 FMAs (fma.rn.f32x2).
__device__ __forceinline__ uint64_t pair_of(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float pair_sum(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return a + b;
}

static __global__ void __launch_bounds__(kThreads, kBlocksPerSm) gemv_x1_kernel(Args a) {
  constexpr int kUnroll = 8;
  extern __shared__ __align__(16) float xs[];          // [K] fp32
  pdl_wait();
  pdl_trigger();
  for (int64_t k = threadIdx.x * 8; k < a.K; k += kThreads * 8) {
    float f[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a.x + k)), f);
    *reinterpret_cast<float4*>(xs + k) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4*>(xs + k + 4) = make_float4(f[4], f[5], f[6], f[7]);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t spr = a.K / kStep;
  const int64_t s_begin = warp * a.steps_per_warp;
  const int64_t total = a.rows * spr;
  const int64_t s_end = min(total, s_begin + a.steps_per_warp);
  if (s_begin >= s_end) return;
  uint64_t acc = 0;                                     // a packed pair of fp32 partial sums
  int64_t cur_row = s_begin / spr;
  auto flush = [&](int64_t row) {
    float v = pair_sum(acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    acc = 0;
    if (lane == 0) {
      const int64_t first = (row * spr) / a.steps_per_warp;
      a.pieces[row * a.max_pieces + (warp - first)] = v;
    }
  };
  int64_t row = cur_row;
  int kst = static_cast<int>(s_begin - cur_row * spr);
  const int spr32 = static_cast<int>(spr);
  const float* xl = xs + lane * 8;
  for (int64_t left = s_end - s_begin; left > 0; left -= kUnroll) {
    uint4 wv[kUnroll];
    const int64_t row0 = row;
    const int kst0 = kst;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (u < left) {
        wv[u] = __ldcs(reinterpret_cast<const uint4*>(a.w + row * a.K + kst * kStep + lane * 8));
        if (++kst == spr32) {
          kst = 0;
          ++row;
        }
      }
    }
    int64_t r = row0;
    int kc = kst0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (u >= left) break;                                // warp-uniform
      if (r != cur_row) {
        flush(cur_row);
        cur_row = r;
      }
      const float4 x0 = *reinterpret_cast<const float4*>(xl + kc * kStep);
      const float4 x1 = *reinterpret_cast<const float4*>(xl + kc * kStep + 4);
      const uint32_t w4[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
      const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t wp = pair_of(__uint_as_float(w4[i] << 16), __uint_as_float(w4[i] & 0xFFFF0000u));
        acc = ffma2(wp, pair_of(xv[2 * i], xv[2 * i + 1]), acc);
      }
      if (++kc == spr32) {
        kc = 0;
        ++r;
      }
    }
  }
  flush(cur_row);
}

// Sum of a row's pieces in warp order.
__device__ __forceinline__ float row_sum(const float* pieces, int64_t row, int64_t spr,
                                         int64_t steps_per_warp, int max_pieces, int T, int t) {
  const int64_t first = (row * spr) / steps_per_warp;
  const int64_t last = ((row + 1) * spr - 1) / steps_per_warp;
  float v = 0.f;
  for (int64_t q = 0; q <= last - first; ++q) v += pieces[(row * max_pieces + q) * T + t];
  return v;
}

struct FixArgs {
  const float* pieces;
  int64_t spr, steps_per_warp;
  int max_pieces, T;
};

// Plain epilogues: out[b][t][r] as fp32 (the row-parallel partials, batch = shard) or
// out[t][b*rows + r] as bf16 (the column-parallel projection of all shards).
static __global__ void __launch_bounds__(256) fix_store_kernel(FixArgs f, int64_t batch, int64_t rows,
                                                        float* out_f32, __nv_bfloat16* out_bf16,
                                                        int64_t ld_bf16) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = batch * rows * f.T;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i % f.T);
    const int64_t row = i / f.T;
    const float v = row_sum(f.pieces, row, f.spr, f.steps_per_warp, f.max_pieces, f.T, t);
    if (out_f32) {
      const int64_t b = row / rows, r = row - b * rows;
      out_f32[(b * f.T + t) * rows + r] = v;
    } else {
      out_bf16[t * ld_bf16 + row] = __float2bfloat16_rn(v);
    }
  }
}

__device__ __forceinline__ float gelu_exact(float z) {
  return 0.5f * z * (1.f + erff(z * 0.70710678118654752f));
}

// The column-parallel up projection's epilogue on the packed w1p rows [p][R][d]: h = act(z)
// (SwiGLU: rows 0..127 of every 256-row block are gate features, 128..255 the same up features),
// h[t][i*Fsp + f]; the pre-activations optionally saved as z[t][i*R + row] (bf16).
static __global__ void __launch_bounds__(256) fix_hidden_kernel(FixArgs f, int p, int64_t R, int64_t Fsp,
                                                         int act, __nv_bfloat16* h,
                                                         __nv_bfloat16* z) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = static_cast<int64_t>(p) * Fsp * f.T;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i % f.T);
    const int64_t fi = i / f.T;                 // i * Fsp + feature
    const int64_t sh = fi / Fsp, feat = fi - sh * Fsp;
    float hv;
    if (act == TP_ACT_SWIGLU) {
      const int64_t rg = sh * R + (feat >> 7) * 256 + (feat & 127);
      const float g = row_sum(f.pieces, rg, f.spr, f.steps_per_warp, f.max_pieces, f.T, t);
      const float u = row_sum(f.pieces, rg + 128, f.spr, f.steps_per_warp, f.max_pieces, f.T, t);
      hv = g / (1.f + __expf(-g)) * u;
      if (z) {
        z[t * (p * R) + rg] = __float2bfloat16_rn(g);
        z[t * (p * R) + rg + 128] = __float2bfloat16_rn(u);
      }
    } else {
      const int64_t rg = sh * R + feat;
      const float g = row_sum(f.pieces, rg, f.spr, f.steps_per_warp, f.max_pieces, f.T, t);
      hv = act == TP_ACT_GELU ? gelu_exact(g) : act == TP_ACT_RELU ? fmaxf(g, 0.f) : g;
      if (z) z[t * (p * R) + rg] = __float2bfloat16_rn(g);
    }
    h[t * (p * Fsp) + fi] = __float2bfloat16_rn(hv);
  }
}

// Whether these shapes take the GEMV path.
inline bool usable(int64_t T, int64_t K) { return T >= 1 && T <= kMaxT && K % kStep == 0; }

inline tp_status run(const Args& a0, const Plan& P, cudaStream_t s, const char* label) {
  Args a = a0;
  a.steps_per_warp = P.steps_per_warp;
  a.max_pieces = P.max_pieces;
  ProfScope prof(s, label);
  const size_t xs_bytes = static_cast<size_t>(a.K) * sizeof(float);
  if (a.T == 1 && a.batch == 1 && xs_bytes <= kMaxStagedX) {
    static int attr_set[64] = {0};
    int dev = 0;
    TP_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 64 && !attr_set[dev]) {
      TP_CUDA_TRY(cudaFuncSetAttribute(gemv_x1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kMaxStagedX)));
      attr_set[dev] = 1;
    }
    TP_LAUNCH_PDL(gemv_x1_kernel, dim3(P.blocks), dim3(kThreads), xs_bytes, s, a);
    return TP_OK;
  }
  switch (a.T) {
    case 1: TP_LAUNCH_PDL(gemv_kernel<1>, dim3(P.blocks), dim3(kThreads), 0, s, a); break;
    case 2: TP_LAUNCH_PDL(gemv_kernel<2>, dim3(P.blocks), dim3(kThreads), 0, s, a); break;
    case 3: TP_LAUNCH_PDL(gemv_kernel<3>, dim3(P.blocks), dim3(kThreads), 0, s, a); break;
    case 4: TP_LAUNCH_PDL(gemv_kernel<4>, dim3(P.blocks), dim3(kThreads), 0, s, a); break;
    default: return set_error(TP_ERR_UNSUPPORTED, "GEMV path takes 1..4 tokens");
  }
  return TP_OK;
}

inline FixArgs fix_args(const Args& a, const Plan& P) {
  return FixArgs{a.pieces, a.K / kStep, P.steps_per_warp, P.max_pieces, a.T};
}

inline unsigned fix_grid(int64_t n) {
  return static_cast<unsigned>(std::min<int64_t>(std::max<int64_t>(1, (n + 255) / 256), 148 * 8));
}

}  // namespace gemv
}  // namespace tp
