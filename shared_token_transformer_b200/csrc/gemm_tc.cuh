// gemm_tc.cuh -- per-token linear layers on the 5th-generation tensor cores.
//
// [TileShare] Fig. 2 / Tab. S1: QKV projection, out-projection and MLP run once per
// token of the shared state (per tile row in the released layers).  Each is a GEMM
// Y[M, N] = A[M, K] * W[N, K]^T with a fused epilogue:
//   EPI_BIAS   y = acc + b
//   EPI_GELU   y = GELU(acc + b)                              (MLP up)
//   EPI_RESID  y = y + acc + b   (y is the residual stream)   (out-proj, MLP down)
//   EPI_QKV    q, k: QK-RMSNorm over each head of 64 channels, gain, then RoPE at
//              the row's coordinates; v: acc + b               (QKV projection)
//   EPI_SWIGLU y = silu(acc_g + b_g) * (acc_u + b_u)          (SwiGLU MLP up, Tab. S6)
//              W holds N/2 gate rows above N/2 up rows; a 128 x BN tile loads BN/2
//              gate rows and the BN/2 matching up rows, so the two sums of an
//              output sit in one accumulator, BN/2 columns apart; y is [M, N/2].
// For e4m3 operands acc is first multiplied by the row scale of A and the column
// scale of W.
//
// Kernel design: persistent, warp-specialised, 320 threads, CTAs walk the
// 128 x BN output tiles in a static round-robin order over banded tiles.
//   warp 8   TMA producer: A and W tiles of 128-byte K slices (64 bf16 / 128 e4m3)
//            into a STAGES-deep ring of 128-byte-swizzled shared buffers
//            (no multicast);
//   warp 9   allocates 2 x BN TMEM columns (two accumulators) and, from one lane,
//            issues tcgen05.mma (M = 128, N = BN, K = 16 bf16 / 32 e4m3 per
//            instruction); tcgen05.commit frees ring slots and hands a finished
//            accumulator to the epilogue;
//   warps 0-7  epilogue in two warpgroups: warp w reads TMEM lane quarter w % 4
//            (one output row per thread), warpgroup w / 4 takes every other
//            64-column chunk; the fused math runs while the MMA warp already
//            accumulates the next tile into the other TMEM buffer.
// Every mbarrier wait is bounded (mbar_wait).
#pragma once

#include "common.cuh"

namespace ts {

enum GemmEpi : int { EPI_BIAS = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_QKV = 3, EPI_SWIGLU = 4 };


struct GemmArgs {
  int M, N, K;            // N: accumulator columns (2 x the output width for EPI_SWIGLU)
  const float* bias;      // [N] or null
  bf16* out;              // [M, ldo]
  int ldo;
  const float* a_scale;   // e4m3 only: [M] per-row scale of A
  const float* w_scale;   // e4m3 only: [N] per-row scale of W
  // EPI_QKV
  int d;                  // model width: columns [0, d) q, [d, 2d) k, [2d, 3d) v
  const float* q_g;       // [64]
  const float* k_g;       // [64]
  float eps_qk;
  const int4* pos;        // [M] (f, y, x, unused) coordinates of each row
  const float2* rope_cs;  // RoPE table (see RopeTable), filled by the preceding LayerNorm
  int rope_off[3];        // first entry of each axis in rope_cs
};

constexpr int kGemmThreads = 320;   // 8 epilogue warps + TMA warp + MMA warp
constexpr int kGemmTmaWarp = 8;
constexpr int kGemmMmaWarp = 9;

template <int BN, int STAGES, int CG = 1>
struct GemmSmem {
  static constexpr int A_BYTES = 128 * 128;
  static constexpr int B_BYTES = (BN / CG) * 128;   // a CTA of a two-SM pair holds half of W's tile rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_OFFSET = STAGES * STAGE_BYTES;   // 8 x 4 KB: one 32 x 64 output chunk per epilogue warp
  static constexpr int BAR_OFFSET = EPI_OFFSET + 8 * 4096;
  static constexpr int NBARS = 2 * STAGES + 4 + 8;      // full, empty, tmem full x2, tmem empty x2, residual x8
  static constexpr int BYTES = BAR_OFFSET + NBARS * 8 + 16;
  static constexpr int LAUNCH_BYTES = BYTES + 1024;     // slack for 1024-byte alignment
};

// QK-RMSNorm (gain g) then RoPE over one head of 64 channels held by this thread.
// Channels of axis a form a block of R_a channels; channel j of a block pairs with
// j + R_a / 2 and turns by the table's angle for (axis a, coordinate, pair j).
template <int R0, int R1, int R2>
__device__ __forceinline__ void qk_norm_rope64(float* v, const float* __restrict__ g, float eps, const int4 pos,
                                               const GemmArgs& args) {
  static_assert(R0 + R1 + R2 == 64, "rope split must cover the 64-channel head");
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < 64; ++c) ss = fmaf(v[c], v[c], ss);
  const float r = rsqrtf(ss * (1.0f / 64.0f) + eps);
#pragma unroll
  for (int c = 0; c < 64; c += 4) {
    const float4 gg = __ldg(reinterpret_cast<const float4*>(g + c));
    v[c] *= r * gg.x;
    v[c + 1] *= r * gg.y;
    v[c + 2] *= r * gg.z;
    v[c + 3] *= r * gg.w;
  }
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const int D = a == 0 ? R0 : (a == 1 ? R1 : R2);
    if (D == 0) continue;
    const int off = a == 0 ? 0 : (a == 1 ? R0 : R0 + R1);
    const int p = a == 0 ? pos.x : (a == 1 ? pos.y : pos.z);
    const float4* tab = reinterpret_cast<const float4*>(args.rope_cs + args.rope_off[a] + p * (D / 2));
#pragma unroll
    for (int j = 0; j < D / 2; j += 2) {
      const float4 cs = __ldg(tab + j / 2);      // (cos, sin) of pairs j and j + 1
      const float x0 = v[off + j], y0 = v[off + j + D / 2];
      const float x1 = v[off + j + 1], y1 = v[off + j + 1 + D / 2];
      v[off + j] = x0 * cs.x - y0 * cs.y;
      v[off + j + D / 2] = x0 * cs.y + y0 * cs.x;
      v[off + j + 1] = x1 * cs.z - y1 * cs.w;
      v[off + j + 1 + D / 2] = x1 * cs.w + y1 * cs.z;
    }
  }
}

// Epilogue arithmetic of one 64-column chunk of a row held by this thread: e4m3
// scales, bias, then GELU or QK-RMSNorm + RoPE (the residual is added by the caller).
template <int EPI, bool FP8, int R0, int R1, int R2>
__device__ __forceinline__ void gemm_epilogue64(float* v, int col, float rs, const int4 pos, const GemmArgs& args) {
  if (FP8 && args.bias) {
    // dequantisation scale and bias in one FMA per value
#pragma unroll
    for (int i = 0; i < 64; i += 4) {
      const float4 ws = __ldg(reinterpret_cast<const float4*>(args.w_scale + col + i));
      const float4 b = __ldg(reinterpret_cast<const float4*>(args.bias + col + i));
      v[i] = fmaf(v[i], rs * ws.x, b.x);
      v[i + 1] = fmaf(v[i + 1], rs * ws.y, b.y);
      v[i + 2] = fmaf(v[i + 2], rs * ws.z, b.z);
      v[i + 3] = fmaf(v[i + 3], rs * ws.w, b.w);
    }
  } else if (FP8) {
#pragma unroll
    for (int i = 0; i < 64; i += 4) {
      const float4 ws = __ldg(reinterpret_cast<const float4*>(args.w_scale + col + i));
      v[i] *= rs * ws.x;
      v[i + 1] *= rs * ws.y;
      v[i + 2] *= rs * ws.z;
      v[i + 3] *= rs * ws.w;
    }
  } else if (args.bias) {
#pragma unroll
    for (int i = 0; i < 64; i += 4) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(args.bias + col + i));
      v[i] += b.x;
      v[i + 1] += b.y;
      v[i + 2] += b.z;
      v[i + 3] += b.w;
    }
  }
  if (EPI == EPI_GELU) {
    if (FP8) {
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const uint64_t y = gelu_erf_one_sfu2(pack_f32x2(v[i], v[i + 1]));
        v[i] = lo_f32(y);
        v[i + 1] = hi_f32(y);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const uint64_t y = gelu_erf2(pack_f32x2(v[i], v[i + 1]));
        v[i] = lo_f32(y);
        v[i + 1] = hi_f32(y);
      }
    }
  } else if (EPI == EPI_QKV) {
    if (col < 2 * args.d)
      qk_norm_rope64<R0, R1, R2>(v, col < args.d ? args.q_g : args.k_g, args.eps_qk, pos, args);
  }
}

// SwiGLU of 32 outputs held by this thread: g (gate sums) is overwritten with
// silu(g * sg + b_g) * (u * su + b_u); col is the output column of g[0], F the
// output width (gate row col + i, up row F + col + i of W, bias and w_scale).
template <bool FP8>
__device__ __forceinline__ void swiglu32(float* g, const float* u, int col, int F, float rs, const GemmArgs& args) {
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    float gg[4] = {g[i], g[i + 1], g[i + 2], g[i + 3]};
    float uu[4] = {u[i], u[i + 1], u[i + 2], u[i + 3]};
    if (FP8) {
      const float4 wg = __ldg(reinterpret_cast<const float4*>(args.w_scale + col + i));
      const float4 wu = __ldg(reinterpret_cast<const float4*>(args.w_scale + F + col + i));
      gg[0] *= rs * wg.x; gg[1] *= rs * wg.y; gg[2] *= rs * wg.z; gg[3] *= rs * wg.w;
      uu[0] *= rs * wu.x; uu[1] *= rs * wu.y; uu[2] *= rs * wu.z; uu[3] *= rs * wu.w;
    }
    if (args.bias) {
      const float4 bg = __ldg(reinterpret_cast<const float4*>(args.bias + col + i));
      const float4 bu = __ldg(reinterpret_cast<const float4*>(args.bias + F + col + i));
      gg[0] += bg.x; gg[1] += bg.y; gg[2] += bg.z; gg[3] += bg.w;
      uu[0] += bu.x; uu[1] += bu.y; uu[2] += bu.z; uu[3] += bu.w;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) g[i + e] = gg[e] / (1.0f + __expf(-gg[e])) * uu[e];
  }
}

// TMA tile store of a shared-memory box to global memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const void* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Output tile order: bands of kGemmBand row tiles, each band walked across all
// column tiles with the row tile fastest.  The CTAs in flight then share one or
// two bands of A and the whole of W, which stay in L2 even when A does not.
constexpr int kGemmBand = 16;
__device__ __forceinline__ void gemm_tile_origin(int tile, int mt, int nt, int bn, int& m0, int& n0, int tm = 128) {
  const int band = tile / (kGemmBand * nt);
  const int first = band * kGemmBand;
  const int rows = min(kGemmBand, mt - first);
  const int r = tile - first * nt;
  m0 = (first + r % rows) * tm;
  n0 = (r / rows) * bn;
}

// CG = 2: a two-SM pair (cluster of two CTAs) computes 256 x BN tiles with
// tcgen05 cta_group::2.  Each CTA loads its own 128 rows of A and half of the
// tile's W rows into its own shared memory (no multicast), both CTAs' loads
// completing on the even CTA's ring barriers; the even CTA's MMA warp issues the
// M = 256 MMAs, and its commits arrive on the ring and accumulator barriers of both
// CTAs.  Each CTA's TMEM holds the accumulators of its own 128 rows, which its
// epilogue warps read as in a single CTA; they release an accumulator on the even
// CTA's barrier.  Half the W bytes per CTA leave room for deeper rings.
template <int BN, int STAGES, int EPI, bool FP8, int R0, int R1, int R2, int CG = 1>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmD, const GemmArgs args) {
  static_assert(CG == 1 || CG == 2, "one CTA or a two-SM pair");
  using SM = GemmSmem<BN, STAGES, CG>;
  constexpr int NMMA = 128 / 32;                  // MMAs per 128-byte K slice (32 bytes each)
  constexpr uint32_t TMEM_COLS = 2 * BN;          // two accumulators: 128, 256 or 512 columns
  constexpr uint32_t IDESC = idesc_make(FP8 ? 0u : 1u, BN, 128 * CG);
  constexpr int TM = 128 * CG;                    // output rows per tile
  constexpr int KE = FP8 ? 128 : 64;              // K elements per slice
  constexpr bool GLU = EPI == EPI_SWIGLU;
  static_assert(!GLU || BN >= 128, "SwiGLU tiles need 64-column output chunks");
  constexpr int NCHUNK = GLU ? BN / 128 : BN / 64;   // 64-column output chunks per tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + SM::BAR_OFFSET;       // STAGES
  const uint32_t bar_empty = bar_full + 8 * STAGES;       // STAGES
  const uint32_t bar_tfull = bar_empty + 8 * STAGES;      // 2
  const uint32_t bar_tempty = bar_tfull + 16;             // 2
  const uint32_t bar_resid = bar_tempty + 16;             // 8: residual chunk of each epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::BAR_OFFSET + SM::NBARS * 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt = (args.M + TM - 1) / TM;
  const int ntiles = mt * (args.N / BN);
  const int KB = args.K / KE;
  // tiles are walked per CTA, or per pair (the two CTAs of a pair walk the same tiles)
  const uint32_t rank = CG == 2 ? cluster_rank() : 0u;
  const int unit = CG == 2 ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int units = CG == 2 ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const bool leader = rank == 0;

  if (warp == kGemmTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmD);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull + 8 * b, 1);
      mbar_init(bar_tempty + 8 * b, 8 * CG);      // one arrival per epilogue warp (of both CTAs of a pair)
    }
    for (int w = 0; w < 8; ++w) mbar_init(bar_resid + 8 * w, 1);
    fence_barrier_init();
  }
  if (warp == kGemmMmaWarp) {
    if (CG == 2) {
      tmem_alloc2(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish2();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();      // the pair's barriers exist before either CTA touches the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();        // A and the output/residual belong to the previous kernel
  pdl_trigger();

  if (warp == kGemmTmaWarp) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = unit; tile < ntiles && ok; tile += units) {
        int m0, n0;
        gemm_tile_origin(tile, mt, args.N / BN, BN, m0, n0, TM);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          if (it >= STAGES && !mbar_wait(bar_empty + 8 * s, ((it / STAGES) - 1) & 1)) { ok = false; break; }
          const uint32_t sa = sbase + s * SM::STAGE_BYTES;
          if (CG == 2) {
            // both CTAs' bytes complete on the even CTA's barrier, which expects them all
            const uint32_t fb = cluster_map(bar_full + 8 * s, 0);
            if (leader) mbar_expect_tx(bar_full + 8 * s, 2 * SM::STAGE_BYTES);
            tma_load_2d_pair(sa, &tmA, fb, kb * KE, m0 + static_cast<int>(rank) * 128);
            if (GLU)    // the even CTA holds the BN/2 gate rows, the odd one the BN/2 up rows
              tma_load_2d_pair(sa + SM::A_BYTES, &tmB, fb, kb * KE, (rank ? args.N / 2 : 0) + n0 / 2);
            else
              tma_load_2d_pair(sa + SM::A_BYTES, &tmB, fb, kb * KE, n0 + static_cast<int>(rank) * (BN / 2));
          } else {
            mbar_expect_tx(bar_full + 8 * s, SM::STAGE_BYTES);
            tma_load_2d(sa, &tmA, bar_full + 8 * s, kb * KE, m0);
            if (GLU) {    // BN/2 gate rows, then the BN/2 up rows of the same outputs
              tma_load_2d(sa + SM::A_BYTES, &tmB, bar_full + 8 * s, kb * KE, n0 / 2);
              tma_load_2d(sa + SM::A_BYTES + (BN / 2) * 128, &tmB, bar_full + 8 * s, kb * KE, args.N / 2 + n0 / 2);
            } else {
              tma_load_2d(sa + SM::A_BYTES, &tmB, bar_full + 8 * s, kb * KE, n0);
            }
          }
        }
      }
    }
  } else if (warp == kGemmMmaWarp) {
    if (lane == 0 && leader) {        // the odd CTA of a pair issues no MMA
      uint32_t it = 0, j = 0;
      bool ok = true;
      for (int tile = unit; tile < ntiles && ok; tile += units, ++j) {
        const uint32_t acc = j & 1, use = j >> 1;
        if (j >= 2 && !mbar_wait(bar_tempty + 8 * acc, (use - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem + acc * BN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          if (!mbar_wait(bar_full + 8 * s, (it / STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = sbase + s * SM::STAGE_BYTES;
          const uint64_t da = sdesc_sw128(sa);
          const uint64_t db = sdesc_sw128(sa + SM::A_BYTES);
#pragma unroll
          for (int k = 0; k < NMMA; ++k) {
            // +32 bytes of K = +2 in the descriptor's (address >> 4) field
            if (CG == 2) {
              if (FP8)
                tc_mma_f8_pair(dt, da + 2 * k, db + 2 * k, IDESC, (kb | k) != 0);
              else
                tc_mma_f16_pair(dt, da + 2 * k, db + 2 * k, IDESC, (kb | k) != 0);
            } else {
              if (FP8)
                tc_mma_f8(dt, da + 2 * k, db + 2 * k, IDESC, (kb | k) != 0);
              else
                tc_mma_f16(dt, da + 2 * k, db + 2 * k, IDESC, (kb | k) != 0);
            }
          }
          if (CG == 2)
            tc_commit_pair(bar_empty + 8 * s);
          else
            tc_commit(bar_empty + 8 * s);
        }
        if (CG == 2)
          tc_commit_pair(bar_tfull + 8 * acc);
        else
          tc_commit(bar_tfull + 8 * acc);
      }
    }
  } else {
    // epilogue warps 0..7: lane quarter warp % 4, column half warp / 4
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const uint32_t stg = sbase + SM::EPI_OFFSET + warp * 4096;
    const uint32_t rbar = bar_resid + 8 * warp;
    uint32_t nres = 0;                 // residual chunks this warp has loaded
    bool store_pending = false;        // a tile store may still be reading the staging buffer
    bool eok = true;
    uint32_t j = 0;
    // accumulator release: on this CTA's barrier, or on the even CTA's for a pair
    const uint32_t tempty = CG == 2 ? cluster_map(bar_tempty, 0) : bar_tempty;
    auto release = [&](uint32_t acc) {
      if (CG == 2)
        mbar_arrive_cluster(tempty + 8 * acc);
      else
        mbar_arrive(tempty + 8 * acc);
    };
    for (int tile = unit; tile < ntiles; tile += units, ++j) {
      const uint32_t acc = j & 1, use = j >> 1;
      int m0, n0;
      gemm_tile_origin(tile, mt, args.N / BN, BN, m0, n0, TM);
      m0 += static_cast<int>(rank) * 128;      // this CTA's rows of the tile
      const int row = m0 + quarter * 32 + lane;
      // the row's scale and coordinates are loaded while the accumulator fills
      float rs = 1.f;
      if (FP8 && row < args.M) rs = __ldg(args.a_scale + row);
      int4 pos = make_int4(0, 0, 0, 0);
      if (EPI == EPI_QKV && row < args.M) pos = __ldg(args.pos + row);
      if (!mbar_wait(bar_tfull + 8 * acc, use & 1)) break;
      tc_fence_after();
      const uint32_t trow = tmem + acc * BN + (static_cast<uint32_t>(quarter * 32) << 16);
      int mine = 0;
#pragma unroll 1
      for (int c = half; c < NCHUNK; c += 2) ++mine;
      if (mine == 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release(acc);
      }
#pragma unroll 1
      for (int c = half, k = 0; c < NCHUNK; c += 2, ++k) {
        // the chunk goes out through this warp's 4 KB staging buffer (32 rows x 128 B,
        // 128-byte swizzle) as one TMA tile store; the residual comes in the same way
        if (store_pending) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          store_pending = false;
        }
        const int col = (GLU ? n0 / 2 : n0) + c * 64, row0 = m0 + quarter * 32;
        if (EPI == EPI_RESID && lane == 0) {
          mbar_expect_tx(rbar, 4096);
          tma_load_2d(stg, &tmD, rbar, col, row0);
        }
        float v[64];
        tmem_ld32(trow + c * 64, v);
        tmem_ld32(trow + c * 64 + 32, v + 32);
        tmem_wait_ld();
        if (GLU) {
          float u[32];
          tmem_ld32(trow + BN / 2 + c * 64, u);
          tmem_wait_ld();
          swiglu32<FP8>(v, u, col, args.N / 2, rs, args);
          tmem_ld32(trow + BN / 2 + c * 64 + 32, u);
          tmem_wait_ld();
          if (k == mine - 1) {         // last TMEM read of this warp for this tile
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release(acc);
          }
          swiglu32<FP8>(v + 32, u, col + 32, args.N / 2, rs, args);
        } else {
          if (k == mine - 1) {         // last TMEM read of this warp for this tile
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release(acc);
          }
          gemm_epilogue64<EPI, FP8, R0, R1, R2>(v, col, rs, pos, args);
        }
        uint8_t* srow = smem + SM::EPI_OFFSET + warp * 4096 + lane * 128;
        if (EPI == EPI_RESID) {
          if (!mbar_wait(rbar, nres & 1)) {
            eok = false;
            break;
          }
          ++nres;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float r[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(srow + ((q ^ (lane & 7)) << 4)), r);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[8 * q + e] += r[e];
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) *reinterpret_cast<uint4*>(srow + ((q ^ (lane & 7)) << 4)) = f32_to_bf16x8(v + 8 * q);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmD, stg, col, row0);     // rows past M are clipped by the copy
          bulk_commit();
        }
        store_pending = true;
      }
      if (!eok) break;
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();      // neither CTA leaves while the pair's MMAs or arrivals may still touch it
  if (warp == kGemmMmaWarp) {
    tc_fence_after();
    if (CG == 2)
      tmem_dealloc2(tmem, TMEM_COLS);
    else
      tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace ts
