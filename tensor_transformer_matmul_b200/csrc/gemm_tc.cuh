// Persistent, warp-specialised tcgen05 GEMM core for sm_100a.
//
//   D[b][m][n] = sum_k A_b(m, k) * B_b(n, k)      (bf16 operands, fp32 accumulator in TMEM)
//
// Roles (192 threads):  warp 0 lane 0 -- TMA producer: fills a ring of shared-memory stages;
//                       warp 1 lane 0 -- MMA issuer: tcgen05.mma into one of two TMEM
//                                        accumulators, frees stages with tcgen05.commit;
//                       warps 2..5    -- epilogue: read the accumulator, apply the fused
//                                        elementwise step, store to global memory.
//
// Work is cut into segments, each one accumulator's worth of k-blocks.  Two schedules:
//   * tiles: segment = one whole output tile (all of K); tile = blockIdx.x + i * gridDim.x.
//   * stream-K: the k-blocks of the first sk_groups tiles, in order, are split into gridDim.x
//     equal contiguous ranges, one per CTA.  A tile whose k-blocks fall in several segments
//     ("split") is finished by whichever CTA arrives last: each writes its fp32 partial to a
//     slot, and the last one adds the slots in k order and applies the epilogue.  No CTA ever
//     waits for another.  The remaining tiles (a whole number of waves) follow as whole tiles,
//     tile sk_groups + c + i * gridDim.x on CTA c, after the CTA's split range: so every SM
//     streams the same number of k-blocks, and the fix-ups of the split tiles overlap the
//     streaming of the whole ones instead of trailing the kernel.
//   With sum_batch, the problem index (the shard) is part of the k space of an output tile:
//   each shard's k-range is its own segment, and the finishing CTA adds the shards' partial
//   tiles in shard order 0..p-1 -- the partial-sum reduce fused into the GEMM.
//
// Operands are 3-D TMA tensors (inner, outer, batch) with 128-byte swizzle.  A K-major operand has
// K as its inner dimension (box 64 x rows); an MN-major operand has M (or N) as its inner
// dimension and is loaded in 64-wide MN blocks (box 64 x 64), which lets the backward pass use
// transposed operands without materialising transposes.  Out-of-range boxes are zero-filled by
// TMA, so ragged M, N and K need no special casing in the main loop.
//
// Every wait is bounded (tp::kWaitTimeoutNs); a wait that runs out raises a shared abort flag,
// records the site in the device error word, lets in-flight copies and MMAs land (bounded), frees
// TMEM and returns.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include <type_traits>

#include "sm100.cuh"
#include "tp_common.cuh"

namespace tp {
namespace tc {

constexpr int kBK = 64;          // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kUmmaK = 16;       // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kMaxGroupSegs = 16;   // segments one split tile may have (checked on the host)

// Compile-time tile configuration.
//   BN     : N of each MMA (columns of the accumulator), 16..256, multiple of 16
//   A_SUB  : 128-row MMAs per tile (1 or 2); A tile = 128*A_SUB rows, each sub-tile has its own
//            accumulator (columns s*BN .. s*BN+BN-1)
//   A_MN / B_MN : operand is MN-major (else K-major)
//   STAGES : depth of the shared-memory ring
template <int BN_, int A_SUB_, bool A_MN_, bool B_MN_, int STAGES_>
struct TileCfg {
  static constexpr int BN = BN_;
  static constexpr int A_SUB = A_SUB_;
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_MN = B_MN_;
  static constexpr int STAGES = STAGES_;
  static constexpr int A_ROWS = 128 * A_SUB;
  static constexpr int A_STAGE_BYTES = A_ROWS * kBK * 2;
  static constexpr int B_STAGE_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr int ACC_COLS = A_SUB * BN;
  static constexpr int TMEM_COLS = (2 * ACC_COLS <= 32) ? 32 : (2 * ACC_COLS <= 64) ? 64
                                   : (2 * ACC_COLS <= 128) ? 128 : (2 * ACC_COLS <= 256) ? 256 : 512;
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5) + 32;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr uint32_t IDESC = sm100::make_idesc_bf16(128, BN, A_MN, B_MN);
  static constexpr int SLOT_FLOATS = 128 * ACC_COLS;   // one partial accumulator tile
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128 is 16..256 step 16");
  static_assert(A_SUB == 1 || A_SUB == 2, "A_SUB");
  static_assert(2 * ACC_COLS <= 512, "two accumulators must fit in TMEM");
  static_assert(!B_MN || BN % 64 == 0, "MN-major operands are loaded in 64-wide blocks");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct GemmParams {
  int32_t M, N, K;        // per problem
  int32_t batch;          // independent problems (e.g. shards)
  int32_t m_blocks, n_blocks, k_blocks;
  int32_t m_fastest;      // tile order: walk M blocks first (1) or N blocks first (0)
  int32_t a_batched, b_batched;  // operand's batch coordinate = problem index (else 0)
  uint32_t* err;          // device error word
  // stream-K schedule
  int32_t stream_k;       // 0: whole tiles; 1: equal contiguous k-block ranges per CTA
  int32_t sum_batch;      // stream-K: the problems are summed into one output (fused reduce)
  int64_t units;          // stream-K: k-blocks over the split tiles (the first sk_groups tiles)
  int32_t sk_groups;      // stream-K: tiles cut into ranges; the tiles after them run whole
  int32_t slots_per_cta;  // partial-tile slots reserved per CTA
  float* slots;           // [gridDim.x][slots_per_cta][SLOT_FLOATS]
  int32_t* counters;      // [output tiles] arrivals of split tiles (zero before the launch)
  // Start each segment's k loop at a tile-dependent k-block (wrapping around).  Weight-streaming
  // GEMMs set it: concurrent CTAs then read different column offsets of their row-major tiles,
  // which spreads the loads over the HBM channels instead of having every CTA hit the same
  // offset within the row pitch at the same moment.
  int32_t rotate_k;
  // Grouped problems (mixture of experts; whole tiles only): problem b belongs to group
  // e = b / grp_div, whose A rows are rows grp_off[e] .. grp_off[e] + grp_cnt[e] - 1 of one
  // K-major A, read at A batch coordinate b % grp_div.  grp_mbp[e] = sum over groups < e of
  // their 128-row blocks (grp_mbp[grp_n] = all of them), so the tiles that hold rows are
  // enumerated directly: tile t -> (block of all groups' blocks, shard, N block), its group found
  // by binary search.  With sum_batch the grp_div problems of a group are summed into one output:
  // a tile's k loop runs problem e*grp_div's k-blocks, then e*grp_div+1's, ... (the shard sum in
  // the accumulator) and the tile space drops the problem index.  grp_cnt == nullptr: ungrouped.
  const int32_t* grp_cnt;
  const int32_t* grp_off;
  const int32_t* grp_mbp;
  int32_t grp_n;
  int32_t grp_div;
  // Swapped grouped problems: the group ranges run along N (B = the gathered rows, A = problem
  // b's weights at A batch coordinate b); grp_mbp then counts BN-row blocks, the tile space is
  // (block of all groups' blocks, [problem of the group,] m block), and each tile's MMAs take
  // N = its block's rows rounded up to 16.
  int32_t grp_swap;
};

// One accumulator's worth of work.
struct Seg {
  int g;          // output tile (group)
  int b;          // problem of this segment (for operand coordinates)
  int mb, nb;     // tile coordinates in blocks
  int kb0, kb1;   // k-block range
  int local;      // index of this segment within its CTA (slot index)
  int rot;        // the k loop visits kb0 + (i + rot) % (kb1 - kb0), i = 0, 1, ...
  int ab;         // A batch coordinate
  int row0;       // first A row of the problem (grouped), else 0
  int n_off;      // first B row of the problem (swapped grouped), else 0
  int row_end;    // end of the problem's gathered rows (A rows, or B rows when swapped);
                  // INT32_MAX when ungrouped
};

// What the epilogue of one tile sees.
struct EpiCtx {
  int row;          // accumulator row (A row within the tile) held by this thread, 0..127
  int b;            // problem index (0 when the problems were summed; A batch when grouped)
  int m0;           // first A row of the tile
  int n0;           // first B row of the tile
  int row_end = 0x7fffffff;   // gathered rows (A rows, or B rows when swapped) at or past this
                              // belong to no problem of the tile
  float* stage = nullptr;     // this warp's 32 x 32 fp32 shared-memory staging tile, if any
};

__device__ __forceinline__ void decode_mn(int r, const GemmParams& gp, int& mb, int& nb) {
  if (gp.m_fastest) {
    mb = r % gp.m_blocks;
    nb = r / gp.m_blocks;
  } else {
    nb = r % gp.n_blocks;
    mb = r / gp.n_blocks;
  }
}

__device__ __forceinline__ int64_t units_per_group(const GemmParams& gp) {
  return gp.sum_batch ? static_cast<int64_t>(gp.batch) * gp.k_blocks : gp.k_blocks;
}
__device__ __forceinline__ int num_groups(const GemmParams& gp) {
  return gp.sum_batch ? gp.m_blocks * gp.n_blocks : gp.batch * gp.m_blocks * gp.n_blocks;
}
__device__ __forceinline__ int64_t cta_start(int c, const GemmParams& gp, int grid) {
  return static_cast<int64_t>(c) * gp.units / grid;
}
// the CTA whose range holds unit u (the largest c with cta_start(c) <= u)
__device__ __forceinline__ int cta_of(int64_t u, const GemmParams& gp, int grid) {
  const int64_t c = ((u + 1) * grid + gp.units - 1) / gp.units - 1;
  return static_cast<int>(c < grid - 1 ? c : grid - 1);
}

// Segment iterator over one CTA's work (both schedules); all roles walk the same sequence.
struct SegIter {
  int64_t u, end;   // stream-K: unit cursor and end; tiles: tile cursor and count
  int local;        // segments so far (stream-K: split segments only; the slot index)
  int dp;           // stream-K: the CTA's next whole tile (after its split range)
  __device__ __forceinline__ void init(const GemmParams& gp, int cta, int grid) {
    local = 0;
    dp = gp.sk_groups + cta;
    if (gp.stream_k) {
      u = cta_start(cta, gp, grid);
      end = cta_start(cta + 1, gp, grid);
    } else if (gp.grp_cnt) {
      u = cta;
      end = static_cast<int64_t>(gp.grp_mbp[gp.grp_n]) * (gp.sum_batch ? 1 : gp.grp_div) *
            (gp.grp_swap ? gp.m_blocks : gp.n_blocks);
    } else {
      u = cta;
      end = num_groups(gp);
    }
  }
  __device__ __forceinline__ bool next(const GemmParams& gp, int grid, Seg& s) {
    if (gp.stream_k && u >= end) {
      // the whole tiles after the split range (never with sum_batch: the host keeps them out)
      if (dp >= num_groups(gp)) return false;
      s.g = dp;
      dp += grid;
      const int per = gp.m_blocks * gp.n_blocks;
      s.b = s.g / per;
      decode_mn(s.g - s.b * per, gp, s.mb, s.nb);
      s.ab = s.b;
      s.row0 = 0;
      s.n_off = 0;
      s.row_end = 0x7fffffff;
      s.kb0 = 0;
      s.kb1 = gp.k_blocks;
      s.local = -1;   // whole: no slot
      s.rot = gp.rotate_k ? static_cast<int>((static_cast<int64_t>(s.g) * 37) % gp.k_blocks) : 0;
      return true;
    }
    if (u >= end) return false;
    if (!gp.stream_k) {
      s.g = static_cast<int>(u);
      u += grid;
      if (gp.grp_cnt) {
        const int other = gp.grp_swap ? gp.m_blocks : gp.n_blocks;
        const int ob = s.g % other;
        const int r = s.g / other;
        const int i = gp.sum_batch ? 0 : r % gp.grp_div;
        const int bg = gp.sum_batch ? r : r / gp.grp_div;   // block among all groups' blocks
        int lo = 0, hi = gp.grp_n;   // the last group whose first block is <= bg
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (gp.grp_mbp[mid] <= bg) lo = mid;
          else hi = mid;
        }
        if (gp.grp_swap) {
          // A = problem (lo, i)'s weights, B = the group's gathered rows (batch: i)
          s.mb = ob;
          s.nb = bg - gp.grp_mbp[lo];
          s.b = i;
          s.ab = lo * gp.grp_div + i;
          s.row0 = 0;
          s.n_off = gp.grp_off[lo];
        } else {
          s.nb = ob;
          s.mb = bg - gp.grp_mbp[lo];
          s.b = lo * gp.grp_div + i;
          s.ab = i;
          s.row0 = gp.grp_off[lo];
          s.n_off = 0;
        }
        s.row_end = gp.grp_off[lo] + gp.grp_cnt[lo];
      } else {
        const int per = gp.m_blocks * gp.n_blocks;
        s.b = s.g / per;
        decode_mn(s.g - s.b * per, gp, s.mb, s.nb);
        s.ab = s.b;
        s.row0 = 0;
        s.n_off = 0;
        s.row_end = 0x7fffffff;
      }
      s.kb0 = 0;
      s.kb1 = (gp.grp_cnt && gp.sum_batch) ? gp.grp_div * gp.k_blocks : gp.k_blocks;
      s.local = local++;
      s.rot = gp.rotate_k ? static_cast<int>((static_cast<int64_t>(s.g) * 37) % gp.k_blocks) : 0;
      return true;
    }
    s.row0 = 0;
    s.n_off = 0;
    s.row_end = 0x7fffffff;
    const int64_t U = units_per_group(gp);
    const int64_t g = u / U, o = u - g * U;
    s.g = static_cast<int>(g);
    int64_t lim;
    if (gp.sum_batch) {
      s.b = static_cast<int>(o / gp.k_blocks);
      s.kb0 = static_cast<int>(o - static_cast<int64_t>(s.b) * gp.k_blocks);
      lim = static_cast<int64_t>(s.b + 1) * gp.k_blocks;
      decode_mn(s.g, gp, s.mb, s.nb);
    } else {
      const int per = gp.m_blocks * gp.n_blocks;
      s.b = s.g / per;
      decode_mn(s.g - s.b * per, gp, s.mb, s.nb);
      s.kb0 = static_cast<int>(o);
      lim = U;
    }
    const int64_t seg_end = lim < end - g * U ? lim : end - g * U;
    s.kb1 = s.kb0 + static_cast<int>(seg_end - o);
    s.local = local++;
    s.rot = gp.rotate_k ? static_cast<int>((static_cast<int64_t>(s.g) * 37) % (s.kb1 - s.kb0)) : 0;
    s.ab = s.b;
    u = g * U + seg_end;
    return true;
  }
};

// TMA coordinates of the i-th k step of segment sg (its k loop starts at kb0 + rot and wraps):
// the K offset and the A and B batch coordinates (with sum_batch, k steps past the first
// problem's k-blocks belong to the next problems).
struct KStep {
  int k0, za, zb;
};
__device__ __forceinline__ KStep k_step(const GemmParams& gp, const Seg& sg, int i) {
  const int nk = sg.kb1 - sg.kb0;
  int kb = sg.kb0 + i + sg.rot;
  if (kb >= sg.kb1) kb -= nk;
  const int pi = kb / gp.k_blocks;
  KStep r;
  r.k0 = (kb - pi * gp.k_blocks) * kBK;
  r.za = gp.a_batched ? sg.ab + pi : 0;
  r.zb = gp.b_batched ? sg.b + pi : 0;
  return r;
}

// All segments of output tile g, in k order: slot pointer and problem index of each.  Returns the
// count (0 if more than kMaxGroupSegs, which the host rules out).
template <int SLOT_FLOATS>
__device__ __forceinline__ int group_segments(const GemmParams& gp, int grid, int g,
                                              const float* (&ptr)[kMaxGroupSegs],
                                              int (&bs)[kMaxGroupSegs]) {
  const int64_t U = units_per_group(gp);
  const int c0 = cta_of(static_cast<int64_t>(g) * U, gp, grid);
  const int c1 = cta_of(static_cast<int64_t>(g) * U + U - 1, gp, grid);
  int n = 0;
  for (int c = c0; c <= c1; ++c) {
    SegIter it;
    it.init(gp, c, grid);
    Seg s;
    while (it.next(gp, grid, s)) {
      if (s.local < 0 || s.g < g) continue;   // a whole tile, or a split tile before g
      if (s.g > g) break;
      if (n == kMaxGroupSegs) return 0;
      ptr[n] = gp.slots + (static_cast<int64_t>(c) * gp.slots_per_cta + s.local) * SLOT_FLOATS;
      bs[n] = s.b;
      ++n;
    }
  }
  return n;
}

// Bounded wait used on the abort path only: ignores the abort flag.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const uint64_t t0 = globaltimer_ns();
  while (!sm100::mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
      record_device_error(err, DEVERR_WAIT_DRAIN);
      return false;
    }
  }
  return true;
}

// barrier among the four epilogue warps (barrier 0 is __syncthreads)
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// the same barrier, returning the AND of v over the 128 epilogue threads
__device__ __forceinline__ int epi_bar_and(int v) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.s32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(v)
      : "memory");
  return r;
}

// ---------------------------------------------------------------------------------------------
// Accumulator value sources for the epilogues
// ---------------------------------------------------------------------------------------------
// From TMEM: 32 lanes x consecutive fp32 columns (warp-collective).
struct TmemSrc {
  uint32_t taddr;   // this warp's 32 lanes, column 0 of the tile's accumulator
  __device__ __forceinline__ void load32(int col, float (&v)[32]) const {
    uint32_t r[32];
    sm100::tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(col), r);
    sm100::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  }
  __device__ __forceinline__ void load16(int col, float (&v)[16]) const {
    uint32_t r[16];
    sm100::tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>(col), r);
    sm100::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  }
};

// From the partial slots of a split tile: the sum over its segments, in k order; with several
// problems (shards), each shard's segments are added first, then the shards in order.  For
// 16-column pieces the loads of up to G16 segments are issued before their adds (one L2 round
// trip per G16 segments, not per segment); the additions keep the order above.
template <int ACC_COLS, int G16>
struct FixupSrc {
  const float* const* ptr;
  const int* bs;
  int n;
  int row;
  template <int W>
  __device__ __forceinline__ void load(int col, float (&v)[W]) const {
    constexpr int G = W <= 16 ? G16 : 1;
    float tot[W], cur[W];
#pragma unroll
    for (int e = 0; e < W; ++e) {
      tot[e] = 0.f;
      cur[e] = 0.f;
    }
    int cur_b = -1;
#pragma unroll 1
    for (int s0 = 0; s0 < n; s0 += G) {
      float x[G][W];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        if (s0 + j < n) {
          const float4* p4 = reinterpret_cast<const float4*>(ptr[s0 + j] + row * ACC_COLS + col);
#pragma unroll
          for (int q = 0; q < W / 4; ++q) {
            const float4 f = __ldcg(p4 + q);
            x[j][4 * q] = f.x; x[j][4 * q + 1] = f.y; x[j][4 * q + 2] = f.z; x[j][4 * q + 3] = f.w;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        if (s0 + j >= n) break;
        if (bs[s0 + j] != cur_b) {
          if (cur_b >= 0) {
#pragma unroll
            for (int e = 0; e < W; ++e) tot[e] += cur[e];
          }
#pragma unroll
          for (int e = 0; e < W; ++e) cur[e] = x[j][e];
          cur_b = bs[s0 + j];
        } else {
#pragma unroll
          for (int e = 0; e < W; ++e) cur[e] += x[j][e];
        }
      }
    }
#pragma unroll
    for (int e = 0; e < W; ++e) v[e] = tot[e] + cur[e];
  }
  __device__ __forceinline__ void load32(int col, float (&v)[32]) const { load<32>(col, v); }
  __device__ __forceinline__ void load16(int col, float (&v)[16]) const { load<16>(col, v); }
};

// Segments whose loads a fix-up issues together (FixupSrc): 3 unless the epilogue asks for fewer
// (a kernel that also carries another epilogue path with high register demand).
template <class E, class = void>
struct FixupGroup {
  static constexpr int value = 3;
};
template <class E>
struct FixupGroup<E, std::void_t<decltype(E::kFixupGroup)>> {
  static constexpr int value = E::kFixupGroup;
};

template <class Cfg, class Epi>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tma_a,
                const __grid_constant__ CUtensorMap tma_b, const GemmParams gp,
                const typename Epi::Params ep) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* a_smem = smem;
  uint8_t* b_smem = smem + Cfg::STAGES * Cfg::A_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(b_smem + Cfg::STAGES * Cfg::B_STAGE_BYTES);
  uint64_t* empty = full + Cfg::STAGES;
  uint64_t* acc_full = empty + Cfg::STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* drain = acc_empty + 2;           // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grid = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tma_a);
    tma_prefetch_desc(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above may overlap the previous kernel's tail; global memory only from here on
  // (the TMA producer waits below, after requesting the weight tiles no earlier kernel writes)
  if (threadIdx.x != 0) pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0;   // stages that received at least one load
      uint32_t last_parity = 0;   // parity of the last phase issued into each stage
      bool ok = true;
      SegIter it;
      it.init(gp, blockIdx.x, grid);
      auto load_a = [&](int st, const Seg& sg, const KStep& ks) {
        const int m0 = sg.row0 + sg.mb * Cfg::A_ROWS;
        uint8_t* sa = a_smem + st * Cfg::A_STAGE_BYTES;
        if (Cfg::A_MN) {
#pragma unroll
          for (int j = 0; j < Cfg::A_ROWS / 64; ++j)
            tma_load_3d(&tma_a, &full[st], sa + j * 64 * kBK * 2, m0 + 64 * j, ks.k0, ks.za);
        } else {
          tma_load_3d(&tma_a, &full[st], sa, ks.k0, m0, ks.za);
        }
      };
      // Weight-streaming GEMMs (rotate_k: A is a weight that no earlier kernel writes, and the
      // schedule is plain arithmetic): the first ring's worth of A tiles is requested before the
      // programmatic-launch wait, so it streams while the previous kernel finishes; B (the
      // activations) is loaded only after the wait.
      int pre = 0;
      if (gp.rotate_k && !gp.grp_cnt) {
        SegIter it0 = it;
        Seg s0;
        if (it0.next(gp, grid, s0)) {
          pre = min(Cfg::STAGES, s0.kb1 - s0.kb0);
          for (int i = 0; i < pre; ++i) {
            mbar_arrive_expect_tx(&full[i], Cfg::STAGE_BYTES);
            load_a(i, s0, k_step(gp, s0, i));
            issued_mask |= 1u << i;   // phase 0
          }
        }
      }
      pdl_wait();
      Seg sg;
      while (ok && it.next(gp, grid, sg)) {
        const int n0 = sg.n_off + sg.nb * Cfg::BN;
        const int nk = sg.kb1 - sg.kb0;
        for (int i = 0; i < nk; ++i) {
          const KStep ks = k_step(gp, sg, i);
          const int k0 = ks.k0, zbi = ks.zb;
          if (pre > 0) {
            --pre;   // this stage's A tile and byte count went out before the wait
          } else {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, gp.err, DEVERR_WAIT_EMPTY)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
            load_a(stage, sg, ks);
          }
          uint8_t* sb = b_smem + stage * Cfg::B_STAGE_BYTES;
          if (Cfg::B_MN) {
#pragma unroll
            for (int j = 0; j < Cfg::BN / 64; ++j)
              tma_load_3d(&tma_b, &full[stage], sb + j * 64 * kBK * 2, n0 + 64 * j, k0, zbi);
          } else {
            tma_load_3d(&tma_b, &full[stage], sb, k0, n0, zbi);
          }
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let every copy already issued land before the CTA can exit
        for (int s = 0; s < Cfg::STAGES; ++s)
          if (issued_mask & (1u << s)) drain_wait(&full[s], (last_parity >> s) & 1u, gp.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it_n = 0;
      bool ok = true;
      bool issued_any = false;
      SegIter it;
      it.init(gp, blockIdx.x, grid);
      Seg sg;
      while (ok && it.next(gp, grid, sg)) {
        const int acc = it_n & 1;
        const uint32_t acc_phase = (it_n >> 1) & 1;
        ++it_n;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, gp.err,
                       DEVERR_WAIT_ACC_EMPTY)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_base = tmem_base + acc * Cfg::ACC_COLS;
        const int nk = sg.kb1 - sg.kb0;
        uint32_t idesc = Cfg::IDESC;
        if (gp.grp_swap) {
          // only the block's rows of the group: N = those rows rounded up to 16
          const int left = sg.row_end - (sg.n_off + sg.nb * Cfg::BN);
          const int n_mma = left >= Cfg::BN ? Cfg::BN : ((left + 15) & ~15);
          idesc = make_idesc_bf16(128, n_mma < 16 ? 16 : n_mma, Cfg::A_MN, Cfg::B_MN);
        }
        for (int i = 0; i < nk; ++i) {
          if (!mbar_wait(&full[stage], phase, abort_flag, gp.err, DEVERR_WAIT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(a_smem + stage * Cfg::A_STAGE_BYTES);
          const uint32_t b_addr = smem_addr(b_smem + stage * Cfg::B_STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t bdesc =
                Cfg::B_MN ? make_sdesc_sw128(b_addr + kk * (kUmmaK * 128), 64 * kBK * 2, 1024)
                          : make_sdesc_sw128(b_addr + kk * (kUmmaK * 2), 16, 1024);
#pragma unroll
            for (int s = 0; s < Cfg::A_SUB; ++s) {
              const uint32_t a_sub = a_addr + s * 128 * kBK * 2;
              const uint64_t adesc =
                  Cfg::A_MN ? make_sdesc_sw128(a_sub + kk * (kUmmaK * 128), 64 * kBK * 2, 1024)
                            : make_sdesc_sw128(a_sub + kk * (kUmmaK * 2), 16, 1024);
              umma_f16(d_base + s * Cfg::BN, adesc, bdesc, idesc, (i > 0 || kk != 0) ? 1u : 0u);
            }
          }
          issued_any = true;
          umma_commit(&empty[stage]);
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
      }
      if (!ok && issued_any) {
        // every MMA issued so far must finish before TMEM is released
        umma_commit(drain);
        drain_wait(drain, 0, gp.err);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const int64_t U = units_per_group(gp);
    const int64_t my_start = gp.stream_k ? cta_start(blockIdx.x, gp, grid) : 0;
    const int64_t my_end = gp.stream_k ? cta_start(blockIdx.x + 1, gp, grid) : 0;
    int it_n = 0;
    SegIter it;
    it.init(gp, blockIdx.x, grid);
    Seg sg;
    while (it.next(gp, grid, sg)) {
      const int acc = it_n & 1;
      const uint32_t acc_phase = (it_n >> 1) & 1;
      ++it_n;
      int ok = 0;
      if (lane == 0)
        ok = mbar_wait(&acc_full[acc], acc_phase, abort_flag, gp.err, DEVERR_WAIT_ACC_FULL);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // all four epilogue warps agree, so none of them can be left waiting at a named barrier
      if (!epi_bar_and(ok)) break;
      tc_fence_after();
      TmemSrc tsrc;
      tsrc.taddr = tmem_base + acc * Cfg::ACC_COLS + (static_cast<uint32_t>(quarter * 32) << 16);
      EpiCtx ctx;
      ctx.row = row;
      ctx.b = gp.sum_batch ? 0 : (gp.grp_cnt ? sg.ab : sg.b);
      ctx.m0 = sg.row0 + sg.mb * Cfg::A_ROWS;
      ctx.n0 = sg.n_off + sg.nb * Cfg::BN;
      ctx.row_end = sg.row_end;
      // the tile is whole when all its k-blocks lie in this CTA's range (then it is one segment)
      const int64_t g0 = static_cast<int64_t>(sg.g) * U;
      const bool whole = !gp.stream_k || sg.g >= gp.sk_groups ||
                         (g0 >= my_start && g0 + U <= my_end && (!gp.sum_batch || gp.batch == 1));
      if (whole) {
        Epi::template run<Cfg>(ep, gp, ctx, tsrc);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        continue;
      }
      // split tile: park the partial in this CTA's slot and free the accumulator
      float* slot = gp.slots +
                    (static_cast<int64_t>(blockIdx.x) * gp.slots_per_cta + sg.local) * Cfg::SLOT_FLOATS +
                    static_cast<int64_t>(row) * Cfg::ACC_COLS;
#pragma unroll 1
      for (int col = 0; col < Cfg::ACC_COLS; col += 16) {
        float v[16];
        tsrc.load16(col, v);
        float4* d4 = reinterpret_cast<float4*>(slot + col);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          __stcg(d4 + q, make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      __threadfence();
      epi_bar();
      const float* ptrs[kMaxGroupSegs];
      int bs[kMaxGroupSegs];
      const int nseg = group_segments<Cfg::SLOT_FLOATS>(gp, grid, sg.g, ptrs, bs);
      if (threadIdx.x == 64) {
        const int old = atomicAdd(&gp.counters[sg.g], 1);
        const int last = (old == nseg - 1) ? 1 : 0;
        if (last) gp.counters[sg.g] = 0;   // ready for the next launch
        *last_flag = last;
      }
      epi_bar();
      const int last = *last_flag;
      epi_bar();   // every thread has read the flag before it can be rewritten
      if (last) {
        __threadfence();
        FixupSrc<Cfg::ACC_COLS, FixupGroup<Epi>::value> fsrc{ptrs, bs, nseg, row};
        Epi::template run<Cfg>(ep, gp, ctx, fsrc);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
}

// ---------------------------------------------------------------------------------------------
// Epilogue helpers
// ---------------------------------------------------------------------------------------------

// 32 bf16 values to 64 contiguous bytes (16-byte aligned destination).
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = w;
  }
}
__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w = s[q];
    v[8 * q + 0] = bf16lo(w.x); v[8 * q + 1] = bf16hi(w.x);
    v[8 * q + 2] = bf16lo(w.y); v[8 * q + 3] = bf16hi(w.y);
    v[8 * q + 4] = bf16lo(w.z); v[8 * q + 5] = bf16hi(w.z);
    v[8 * q + 6] = bf16lo(w.w); v[8 * q + 7] = bf16hi(w.w);
  }
}

__device__ __forceinline__ float fast_silu(float z) { return z / (1.0f + __expf(-z)); }
__device__ __forceinline__ float fast_sigmoid(float z) { return 1.0f / (1.0f + __expf(-z)); }

// ---------------------------------------------------------------------------------------------
// Forward up-projection epilogue: h = act(acc) (or silu(gate) * up), optional saved z.
//   Non-swapped (A = x tokens, B = packed W1 rows): accumulator row = token, column = packed row.
//   Swapped (A = packed W1 rows, B = x tokens):     accumulator row = packed row, column = token.
// SwiGLU tiles hold 128 gate features and the same 128 up features: non-swapped BN = 256 with
// gate in columns 0..127 and up in 128..255; swapped A_SUB = 2 with gate in sub-tile 0 and up in
// sub-tile 1.  h column of feature (block j, offset o) is j*128 + o in the padded layout.
// ---------------------------------------------------------------------------------------------
struct EpiHiddenParams {
  __nv_bfloat16* h;   // [tokens][ld_h]
  __nv_bfloat16* z;   // [tokens][ld_z] or null
  int64_t ld_h, ld_z;
  int32_t tokens;     // valid tokens
  int32_t rows;       // valid packed rows (columns of z)
  int32_t act;        // tp_act
  int32_t swap;       // 1: A = weights, B = tokens
};

// MODE 0: p.swap chooses the orientation at run time; MODE 1: swapped only (the decode GEMMs),
// so their kernels carry neither the other path's code nor its register demand.
template <int MODE>
struct EpiHiddenT {
  using Params = EpiHiddenParams;
  static constexpr int kFixupGroup = MODE == 1 ? 3 : 1;

  template <class Cfg, class Src>
  __device__ __forceinline__ static void run(const Params& p, const GemmParams&, const EpiCtx& c,
                                             const Src& src) {
    const bool swiglu = p.act == TP_ACT_SWIGLU;
    if (MODE == 0 && !p.swap) {
      const int t = c.m0 + c.row;
      const bool live = t < p.tokens && t < c.row_end;
      if (swiglu) {
        // BN == 256, n0 multiple of 256
        const int blk = c.n0 >> 8;
#pragma unroll 1
        for (int col = 0; col < 128; col += 32) {
          float g[32], u[32];
          src.load32(col, g);
          src.load32(128 + col, u);
          if (live) {
            if (p.z) {
              store_bf16x32(p.z + t * p.ld_z + c.n0 + col, g);
              store_bf16x32(p.z + t * p.ld_z + c.n0 + 128 + col, u);
            }
            float hv[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) hv[e] = fast_silu(g[e]) * u[e];
            store_bf16x32(p.h + t * p.ld_h + blk * 128 + col, hv);
          }
        }
      } else {
#pragma unroll 1
        for (int col = 0; col < Cfg::BN; col += 32) {
          float v[32];
          src.load32(col, v);
          const int r0 = c.n0 + col;
          if (live && r0 + 32 <= p.rows) {
            if (p.z) store_bf16x32(p.z + t * p.ld_z + r0, v);
            float hv[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) hv[e] = act_f(p.act, v[e]);
            store_bf16x32(p.h + t * p.ld_h + r0, hv);
          } else if (live) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (r0 + e < p.rows) {
                if (p.z) p.z[t * p.ld_z + r0 + e] = __float2bfloat16_rn(v[e]);
                p.h[t * p.ld_h + r0 + e] = __float2bfloat16_rn(act_f(p.act, v[e]));
              }
            }
          }
        }
      }
    } else {
      // swapped: this thread owns packed row (m0 + row); columns are tokens n0 + col
      if (swiglu) {
        const int blk = c.m0 >> 8;
        const int feat = blk * 128 + c.row;
        const int zg = c.m0 + c.row, zu = c.m0 + 128 + c.row;
#pragma unroll 1
        for (int col = 0; col < Cfg::BN; col += 16) {
          float g[16], u[16];
          src.load16(col, g);
          src.load16(Cfg::BN + col, u);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int t = c.n0 + col + e;
            if (t < p.tokens && t < c.row_end) {
              p.h[t * p.ld_h + feat] = __float2bfloat16_rn(fast_silu(g[e]) * u[e]);
              if (p.z) {
                p.z[t * p.ld_z + zg] = __float2bfloat16_rn(g[e]);
                p.z[t * p.ld_z + zu] = __float2bfloat16_rn(u[e]);
              }
            }
          }
        }
      } else {
        const int r = c.m0 + c.row;
        const bool live = r < p.rows;
#pragma unroll 1
        for (int col = 0; col < Cfg::BN; col += 16) {
          float v[16];
          src.load16(col, v);  // whole warp: a TMEM source is warp-collective
          if (!live) continue;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int t = c.n0 + col + e;
            if (t < p.tokens && t < c.row_end) {
              p.h[t * p.ld_h + r] = __float2bfloat16_rn(act_f(p.act, v[e]));
              if (p.z) p.z[t * p.ld_z + r] = __float2bfloat16_rn(v[e]);
            }
          }
        }
      }
    }
  }
};
using EpiHidden = EpiHiddenT<0>;
using EpiHiddenSwap = EpiHiddenT<1>;

// ---------------------------------------------------------------------------------------------
// fp32 store of the accumulator: out[b][i][j] = D (or D^T when swapped), with i < rows_valid and
// j < cols_valid.  Used for the row-parallel partial sums y_i, the dx partials and the weight
// gradients.  Non-swapped: i = m (A row), j = n.  Swapped: i = n (token), j = m (feature).
// ---------------------------------------------------------------------------------------------
struct EpiStoreF32 {
  // not swapped: requires Cfg::A_SUB == 1; swapped: sub-tile s holds A rows m0 + 128 s + row
  struct Params {
    float* out;
    int64_t ld;            // elements between rows
    int64_t batch_stride;  // elements between problems
    int32_t rows_valid, cols_valid;
    int32_t swap;
  };

  template <class Cfg, class Src>
  __device__ __forceinline__ static void run(const Params& p, const GemmParams&, const EpiCtx& c,
                                             const Src& src) {
    float* base = p.out + static_cast<int64_t>(c.b) * p.batch_stride;
    if (!p.swap) {
      const int i = c.m0 + c.row;
      const bool live = i < p.rows_valid && i < c.row_end;
      // With a staging tile, each 32-column chunk of the warp's 32 rows goes through shared
      // memory so that the global stores are whole 128-byte row segments (8 lanes per row, 4
      // rows per instruction) instead of 16 bytes in each of 32 rows.  Float4 slots are XOR
      // swizzled by row, so both the row-wise writes and the transposed reads are conflict-free.
      const bool staged = c.stage != nullptr && (p.ld & 3) == 0 &&
                          (reinterpret_cast<uintptr_t>(base) & 15) == 0;
      const int lane = threadIdx.x & 31;
      const int i_warp = i - lane;   // the warp's first row
#pragma unroll 1
      for (int col = 0; col < Cfg::BN; col += 32) {
        float v[32];
        src.load32(col, v);
        const int j0 = c.n0 + col;
        if (staged) {
          float4* mine = reinterpret_cast<float4*>(c.stage + lane * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            mine[q ^ (lane & 7)] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          __syncwarp();
          const int jq = lane & 7;
          const int jc = j0 + 4 * jq;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int r = 4 * k + (lane >> 3);
            const float4 val = reinterpret_cast<const float4*>(c.stage + r * 32)[jq ^ (r & 7)];
            const int ir = i_warp + r;
            if (ir < p.rows_valid && ir < c.row_end) {
              float* dst = base + static_cast<int64_t>(ir) * p.ld + jc;
              if (jc + 4 <= p.cols_valid) {
                *reinterpret_cast<float4*>(dst) = val;
              } else {
                const float e4[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (jc + e < p.cols_valid) dst[e] = e4[e];
              }
            }
          }
          __syncwarp();
          continue;
        }
        if (live) {
          float* dst = base + i * p.ld + j0;
          if (j0 + 32 <= p.cols_valid && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
            float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (j0 + e < p.cols_valid) dst[e] = v[e];
          }
        }
      }
    } else {
#pragma unroll 1
      for (int sub = 0; sub < Cfg::A_SUB; ++sub) {
        const int j = c.m0 + sub * 128 + c.row;
        const bool live = j < p.cols_valid;
#pragma unroll 1
        for (int col = 0; col < Cfg::BN; col += 16) {
          float v[16];
          src.load16(sub * Cfg::BN + col, v);
          if (live) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int i = c.n0 + col + e;
              if (i < p.rows_valid && i < c.row_end) base[i * p.ld + j] = v[e];
            }
          }
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------------------------
// Fused partial-sum reduce: with sum_batch the source already holds sum_i y_i (shards added in
// order 0..p-1 in fp32); this adds the residual once and rounds to the output dtype.
// out[i][j] with i = token, j = output feature (swapped: i = n, j = m).  Requires A_SUB == 1.
// ---------------------------------------------------------------------------------------------
struct EpiReduceOut {
  struct Params {
    void* out;
    const void* residual;   // same dtype and layout as out, or null
    int64_t ld;
    int32_t rows_valid, cols_valid;
    int32_t out_bf16;
    int32_t swap;
  };

  __device__ __forceinline__ static void put(const Params& p, int64_t idx, float v) {
    if (p.residual)
      v = (p.out_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.residual)[idx])
                      : static_cast<const float*>(p.residual)[idx]) + v;
    if (p.out_bf16) static_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
    else static_cast<float*>(p.out)[idx] = v;
  }

  template <class Cfg, class Src>
  __device__ __forceinline__ static void run(const Params& p, const GemmParams&, const EpiCtx& c,
                                             const Src& src) {
    if (!p.swap) {
      // one thread per output row: a whole 32-column chunk goes out as 16-byte stores (and the
      // residual comes in as 16-byte loads); chunks at the right edge or off 16-byte alignment
      // take the element path.  Both add the residual in fp32 and round the same way.
      const int i = c.m0 + c.row;
      const bool live = i < p.rows_valid;
      const int eb = p.out_bf16 ? 2 : 4;
#pragma unroll 1
      for (int col = 0; col < Cfg::BN; col += 32) {
        float v[32];
        src.load32(col, v);
        if (!live) continue;
        const int j0 = c.n0 + col;
        const int64_t idx0 = static_cast<int64_t>(i) * p.ld + j0;
        const uintptr_t oa = reinterpret_cast<uintptr_t>(p.out) + idx0 * eb;
        const uintptr_t ra = reinterpret_cast<uintptr_t>(p.residual) + idx0 * eb;
        if (j0 + 32 <= p.cols_valid && (oa & 15) == 0 && (ra & 15) == 0) {
          if (p.out_bf16) {
            if (p.residual) {
              float r[32];
              load_bf16x32(reinterpret_cast<const __nv_bfloat16*>(ra), r);
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = r[e] + v[e];
            }
            store_bf16x32(reinterpret_cast<__nv_bfloat16*>(oa), v);
          } else {
            if (p.residual) {
              const float4* r4 = reinterpret_cast<const float4*>(ra);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 r = r4[q];
                v[4 * q] = r.x + v[4 * q];
                v[4 * q + 1] = r.y + v[4 * q + 1];
                v[4 * q + 2] = r.z + v[4 * q + 2];
                v[4 * q + 3] = r.w + v[4 * q + 3];
              }
            }
            float4* d4 = reinterpret_cast<float4*>(oa);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
          continue;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (j0 + e < p.cols_valid) put(p, idx0 + e, v[e]);
      }
    } else {
      const int j = c.m0 + c.row;
      const bool live = j < p.cols_valid;
#pragma unroll 1
      for (int col = 0; col < Cfg::BN; col += 16) {
        float v[16];
        src.load16(col, v);
        if (!live) continue;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = c.n0 + col + e;
          if (i < p.rows_valid) put(p, static_cast<int64_t>(i) * p.ld + j, v[e]);
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------------------------
// Backward epilogue of dH_i = dY W2_i^T (A = dY tokens, B = w2p[i] MN-major, problem = shard):
// turns dH into the pre-activation gradient dz using the saved z, written in w1p's row order.
//   SwiGLU: dg = dH * u * silu'(g), du = dH * silu(g);  other activations: dz = dH * act'(z).
// ---------------------------------------------------------------------------------------------
struct EpiActBwd {
  struct Params {
    const __nv_bfloat16* z;   // saved pre-activations [T][ld]
    __nv_bfloat16* dz;        // [T][ld]
    int64_t ld;               // p * R
    int32_t R;                // packed rows per shard
    int32_t tokens;
    int32_t act;
  };

  template <class Cfg, class Src>
  __device__ __forceinline__ static void run(const Params& p, const GemmParams&, const EpiCtx& c,
                                             const Src& src) {
    const int t = c.m0 + c.row;
    const bool live = t < p.tokens;
    const int64_t rowoff = static_cast<int64_t>(t) * p.ld + static_cast<int64_t>(c.b) * p.R;
#pragma unroll 1
    for (int col = 0; col < Cfg::BN; col += 32) {
      float dh[32];
      src.load32(col, dh);
      if (!live) continue;
      const int f = c.n0 + col;                  // shard-local padded feature (multiple of 32)
      if (p.act == TP_ACT_SWIGLU) {
        const int zc = (f >> 7) * 256 + (f & 127);   // gate column; up column is zc + 128
        float g[32], u[32], dg[32], du[32];
        load_bf16x32(p.z + rowoff + zc, g);
        load_bf16x32(p.z + rowoff + zc + 128, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float s = fast_sigmoid(g[e]);
          dg[e] = dh[e] * u[e] * (s * (1.0f + g[e] * (1.0f - s)));
          du[e] = dh[e] * g[e] * s;
        }
        store_bf16x32(p.dz + rowoff + zc, dg);
        store_bf16x32(p.dz + rowoff + zc + 128, du);
      } else {
        float zv[32], d[32];
        load_bf16x32(p.z + rowoff + f, zv);
#pragma unroll
        for (int e = 0; e < 32; ++e) d[e] = dh[e] * act_grad_f(p.act, zv[e]);
        store_bf16x32(p.dz + rowoff + f, d);
      }
    }
  }
};

// ---------------------------------------------------------------------------------------------
// bf16 store of the accumulator, problem b's columns placed b * col_off to the right:
// out[i][b * col_off + j] = D[i][j] for i < rows_valid, j < cols_valid (not swapped).  Used for
// the attention backward's dO_i = dY Wo_i^T, which lands in the [tokens][n_q hd] layout of o.
// ---------------------------------------------------------------------------------------------
struct EpiStoreBf16 {
  struct Params {
    __nv_bfloat16* out;
    int64_t ld;        // elements between rows
    int64_t col_off;   // column offset per problem
    int32_t rows_valid, cols_valid;
  };

  template <class Cfg, class Src>
  __device__ __forceinline__ static void run(const Params& p, const GemmParams&, const EpiCtx& c,
                                             const Src& src) {
    const int i = c.m0 + c.row;
    const bool live = i < p.rows_valid;
    __nv_bfloat16* base =
        p.out + static_cast<int64_t>(i) * p.ld + static_cast<int64_t>(c.b) * p.col_off;
#pragma unroll 1
    for (int col = 0; col < Cfg::BN; col += 32) {
      float v[32];
      src.load32(col, v);   // warp-collective: every lane loads
      const int j0 = c.n0 + col;
      if (!live) continue;
      __nv_bfloat16* dst = base + j0;
      if (j0 + 32 <= p.cols_valid && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
        store_bf16x32(dst, v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (j0 + e < p.cols_valid) dst[e] = __float2bfloat16_rn(v[e]);
      }
    }
  }
};

}  // namespace tc
}  // namespace tp
