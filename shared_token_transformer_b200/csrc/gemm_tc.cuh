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
// For e4m3 operands acc is first multiplied by the row scale of A and the column
// scale of W.
//
// Kernel design (one 128 x BN output tile per CTA, 192 threads):
//   warp 0   TMA producer: A and W tiles of 128-byte K slices (64 bf16 / 128 e4m3)
//            into a STAGES-deep ring of 128-byte-swizzled shared buffers;
//   warp 1   allocates BN TMEM columns and, from one lane, issues tcgen05.mma
//            (M = 128, N = BN, K = 16 bf16 / 32 e4m3 per instruction) into the fp32
//            accumulator in TMEM; tcgen05.commit frees each ring slot and finally
//            signals the epilogue;
//   warps 2-5  epilogue: tcgen05.ld of their 32 TMEM lanes (one output row per
//            thread), fused math, bf16 stores.
// Every mbarrier wait is bounded (mbar_wait).
#pragma once

#include "common.cuh"

namespace ts {

enum GemmEpi : int { EPI_BIAS = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_QKV = 3 };

struct RopeTheta {
  float hi[32];  // per rotation pair p of a 64-channel head: theta as hi + lo floats
  float lo[32];
};

struct GemmArgs {
  int M, N, K;
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
  RopeTheta theta;
};

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int A_BYTES = 128 * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_OFFSET = STAGES * STAGE_BYTES;
  static constexpr int BYTES = BAR_OFFSET + (2 * STAGES + 1) * 8 + 16;
  static constexpr int LAUNCH_BYTES = BYTES + 1024;  // slack for 1024-byte alignment
};

// QK-RMSNorm (gain g) then RoPE over one head of 64 channels held by this thread.
// Channels of axis a form a block of R_a channels; channel j of a block pairs with
// j + R_a / 2.  Pair index p runs over the blocks in order (the theta table order).
template <int R0, int R1, int R2>
__device__ __forceinline__ void qk_norm_rope64(float* v, const float* __restrict__ g, float eps, const int4 pos,
                                               const RopeTheta& th) {
  static_assert(R0 + R1 + R2 == 64, "rope split must cover the 64-channel head");
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < 64; ++c) ss = fmaf(v[c], v[c], ss);
  const float r = rsqrtf(ss * (1.0f / 64.0f) + eps);
#pragma unroll
  for (int c = 0; c < 64; ++c) v[c] = v[c] * r * __ldg(g + c);
  const float p[3] = {static_cast<float>(pos.x), static_cast<float>(pos.y), static_cast<float>(pos.z)};
  constexpr int R[3] = {R0, R1, R2};
  int off = 0, pair = 0;
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const int half = R[a] / 2;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      float c, s;
      rope_cos_sin(p[a], th.hi[pair + j], th.lo[pair + j], c, s);
      const float x = v[off + j], y = v[off + j + half];
      v[off + j] = x * c - y * s;
      v[off + j + half] = x * s + y * c;
    }
    off += R[a];
    pair += half;
  }
}

template <int BN, int STAGES, int EPI, bool FP8, int R0, int R1, int R2>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs args) {
  using SM = GemmSmem<BN, STAGES>;
  constexpr int MMA_K_BYTES = 32;                 // 16 bf16 or 32 e4m3 per MMA
  constexpr int NMMA = 128 / MMA_K_BYTES;         // MMAs per 128-byte K slice
  constexpr uint32_t TMEM_COLS = BN;              // 64, 128 or 256 (power of two >= 32)
  constexpr uint32_t IDESC = idesc_make(FP8 ? 0u : 1u, BN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + SM::BAR_OFFSET;      // STAGES barriers
  const uint32_t bar_empty = bar_full + 8 * STAGES;      // STAGES barriers
  const uint32_t bar_tmem = bar_empty + 8 * STAGES;      // 1 barrier
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::BAR_OFFSET + (2 * STAGES + 1) * 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int n0 = blockIdx.y * BN;
  const int KB = args.K / (FP8 ? 128 : 64);

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_tmem, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        if (kb >= STAGES && !mbar_wait(bar_empty + 8 * s, ((kb / STAGES) - 1) & 1)) break;
        const uint32_t sa = sbase + s * SM::STAGE_BYTES;
        mbar_expect_tx(bar_full + 8 * s, SM::STAGE_BYTES);
        tma_load_2d(sa, &tmA, bar_full + 8 * s, kb * (FP8 ? 128 : 64), m0);
        tma_load_2d(sa + SM::A_BYTES, &tmB, bar_full + 8 * s, kb * (FP8 ? 128 : 64), n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(bar_full + 8 * s, (kb / STAGES) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = sbase + s * SM::STAGE_BYTES;
        const uint64_t da = sdesc_sw128(sa);
        const uint64_t db = sdesc_sw128(sa + SM::A_BYTES);
#pragma unroll
        for (int k = 0; k < NMMA; ++k) {
          // +32 bytes of K = +2 in the descriptor's (address >> 4) field
          if (FP8)
            tc_mma_f8(tmem, da + 2 * k, db + 2 * k, IDESC, (kb | k) != 0);
          else
            tc_mma_f16(tmem, da + 2 * k, db + 2 * k, IDESC, (kb | k) != 0);
        }
        tc_commit(bar_empty + 8 * s);
      }
      (void)ok;
      tc_commit(bar_tmem);
    }
  } else {
    // epilogue: warps 2..5 own TMEM lane quarters (warp % 4)
    const int quarter = warp & 3;
    const int row = m0 + quarter * 32 + lane;
    const bool waited = mbar_wait(bar_tmem, 0);
    tc_fence_after();
    if (waited) {
      const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      float rs = 1.f;
      if (FP8 && row < args.M) rs = __ldg(args.a_scale + row);
      int4 pos = make_int4(0, 0, 0, 0);
      if (EPI == EPI_QKV && row < args.M) pos = __ldg(args.pos + row);
#pragma unroll 1
      for (int c = 0; c < BN; c += 64) {
        float v[64];
        tmem_ld32(trow + c, v);
        tmem_ld32(trow + c + 32, v + 32);
        tmem_wait_ld();
        if (row < args.M) {
          const int col = n0 + c;
          if (FP8) {
#pragma unroll
            for (int i = 0; i < 64; ++i) v[i] *= rs * __ldg(args.w_scale + col + i);
          }
          if (args.bias) {
#pragma unroll
            for (int i = 0; i < 64; i += 4) {
              const float4 b = __ldg(reinterpret_cast<const float4*>(args.bias + col + i));
              v[i] += b.x; v[i + 1] += b.y; v[i + 2] += b.z; v[i + 3] += b.w;
            }
          }
          bf16* dst = args.out + static_cast<size_t>(row) * args.ldo + col;
          if (EPI == EPI_GELU) {
#pragma unroll
            for (int i = 0; i < 64; ++i) v[i] = gelu_erf(v[i]);
          } else if (EPI == EPI_RESID) {
#pragma unroll
            for (int i = 0; i < 64; i += 8) {
              float r[8];
              bf16x8_to_f32(*reinterpret_cast<const uint4*>(dst + i), r);
#pragma unroll
              for (int e = 0; e < 8; ++e) v[i + e] += r[e];
            }
          } else if (EPI == EPI_QKV) {
            if (col < 2 * args.d) qk_norm_rope64<R0, R1, R2>(v, col < args.d ? args.q_g : args.k_g, args.eps_qk, pos,
                                                          args.theta);
          }
#pragma unroll
          for (int i = 0; i < 64; i += 8) *reinterpret_cast<uint4*>(dst + i) = f32_to_bf16x8(v + i);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace ts
