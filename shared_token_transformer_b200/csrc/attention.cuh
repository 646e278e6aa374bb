// attention.cuh -- per-tile dense attention over gathered rows.
//
// [TileShare] Tab. S1 "Attention (dense, per tile)" and Fig. 2: for tile t and head h
// the keys, values and queries are the rows [global token of t, window slots of t];
// O = softmax(q k^T / sqrt(hd)) v with no mask.  In a shared layer the rows come
// from the shared q/k/v through the tile's index map (the "gather"); in a per-tile
// layer they are the tile's own contiguous rows.  q and k arrive already rotated
// (RoPE runs once per row in the QKV epilogue), so this is a plain gathered
// attention.
//
// bf16 kernel (hd = 64), grid (nqb + 1, heads, T), 288 threads, 2 CTAs per SM:
//   blocks qb < nqb: 128 window queries.
//     warps 4-7  loaders: cp.async gathers of Q (once) and of 128-key K/V blocks
//                through the row map into 128-byte-swizzled shared rows; two
//                warp pairs fill the two buffers independently and publish each
//                block with fence.proxy.async and an mbarrier;
//     warp 8     MMA issuer (one lane): S = Q K^T (tcgen05 kind::f16, M = 128,
//                N = 128 keys) into TMEM, then O += P V (M = 128, N = 64, V read
//                as an MN-major operand) into TMEM; S of block j+1 is issued while
//                the softmax of block j runs;
//     warps 0-3  softmax, one query row per thread (TMEM lane = row): tcgen05.ld
//                of S, online softmax in the exp2 domain, P as bf16 into swizzled
//                shared memory, rescale of the O row in TMEM when the max moves;
//                the global key (slot 0) seeds the running max and sum and is
//                added back at the end with its running coefficient.
//   block qb == nqb: the global token's own query row (one row attends to N keys):
//     warps split the keys, lanes own channel pairs, partial states merged at the end.
// fp32 kernel (any hd <= 64, multiple of 4): one thread per query row, keys in
//   shared memory, online softmax; for the fp32 reference-precision path.
#pragma once

#include "common.cuh"

namespace ts {

struct AttnArgs {
  const void* qkv;    // [rows, 3d]
  const int* rowmap;  // [T * N]: qkv row of slot s of tile t (null: row = t*N + s)
  void* O;            // [T * N, d]
  int N, Nw, d, heads, T;
  float scale_log2;   // log2(e) / sqrt(hd)
  float scale;        // 1 / sqrt(hd)
};

__device__ __forceinline__ int attn_row(const AttnArgs& a, int t, int s) {
  return a.rowmap ? __ldg(a.rowmap + t * a.N + s) : t * a.N + s;
}

// byte offset of 16-byte chunk `ch` of row `r` in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz(int r, int ch) { return r * 128 + ((ch ^ (r & 7)) << 4); }

constexpr int kAttnThreads = 288;        // 4 softmax + 4 loader + 1 MMA warps
constexpr int kAttnBQ = 128;             // queries per CTA
constexpr int kAttnBK = 128;             // keys per block

struct AttnSmem {
  static constexpr int Q = 0;                 // 16 KB
  static constexpr int K = 16384;             // 2 x 16 KB
  static constexpr int V = 16384 * 3;         // 2 x 16 KB
  static constexpr int P = 16384 * 5;         // 2 x 16 KB (keys 0-63, keys 64-127)
  static constexpr int KG = 16384 * 7;        // 64 floats k_g, 64 floats v_g
  static constexpr int BAR = KG + 512;        // barriers
  static constexpr int NBAR = 8;
  static constexpr int BYTES = BAR + NBAR * 8 + 16;
  static constexpr int LAUNCH_BYTES = BYTES;  // base must be 1024-aligned (checked): two CTAs per SM
};
// global-row blocks reuse the same dynamic shared memory
constexpr int kAttnGlobalBytes = (32 + 32 + 32 * 64) * 4;
static_assert(kAttnGlobalBytes <= AttnSmem::LAUNCH_BYTES, "global-row scratch must fit");

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle: rows
// of 128 bytes along K (here: keys), 64 elements along N contiguous in a row,
// 8-row atoms of 1024 bytes (stride byte offset), a single atom along N.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(16384u >> 4) << 16;   // leading byte offset: next N atom (unused, N = 64)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;    // stride byte offset: next 8 K rows
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------------------
// window-query block (tcgen05)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void attn_window_block_tc(const AttnArgs& a, int qb, int h, int t, uint8_t* smem) {
  const bf16* qkv = reinterpret_cast<const bf16*>(a.qkv);
  const int ld = 3 * a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_kvfull = sb + AttnSmem::BAR;        // 2, count 64 (one loader pair each)
  const uint32_t bar_kvempty = bar_kvfull + 16;          // 2, count 1 (commit)
  const uint32_t bar_sfull = bar_kvempty + 16;           // 1, count 1 (commit)
  const uint32_t bar_sfree = bar_sfull + 8;              // 1, count 4 (softmax warps)
  const uint32_t bar_pfull = bar_sfree + 8;              // 1, count 4 (softmax warps)
  const uint32_t bar_odone = bar_pfull + 8;              // 1, count 1 (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + AttnSmem::BAR + AttnSmem::NBAR * 8);
  float* sKg = reinterpret_cast<float*>(smem + AttnSmem::KG);
  float* sVg = sKg + 64;
  const int nkb = (a.Nw + kAttnBK - 1) / kAttnBK;
  const int q0 = 1 + qb * kAttnBQ;  // first slot of this query block

  if (warp == 8 && lane == 0) {
    mbar_init(bar_kvfull, 64);
    mbar_init(bar_kvfull + 8, 64);
    mbar_init(bar_kvempty, 1);
    mbar_init(bar_kvempty + 8, 1);
    mbar_init(bar_sfull, 1);
    mbar_init(bar_sfree, 4);
    mbar_init(bar_pfull, 4);
    mbar_init(bar_odone, 1);
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), 256);    // S: columns 0-127, O: columns 128-191
    tmem_relinquish();
  }
  pdl_wait();
  pdl_trigger();
  if (tid < 64) {
    const size_t grow = static_cast<size_t>(attn_row(a, t, 0)) * ld + h * 64 + tid;
    sKg[tid] = __bfloat162float(qkv[grow + a.d]);
    sVg[tid] = __bfloat162float(qkv[grow + 2 * a.d]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp >= 4 && warp < 8) {
    // ---------------- loaders ----------------
    // Two independent pairs of warps, one per K/V buffer: pair b loads the blocks
    // j = b, b + 2, ... so that publishing one buffer never waits on the other.
    const int grp = (warp - 4) >> 1;
    const int lt = tid - 128 - grp * 64;       // 0..63
    // thread lt copies 16-byte chunk (lt & 7) of rows (lt >> 3) + 8 i, i = 0..15; the
    // row indices are read up front so that their loads overlap
    const int ch = lt & 7, r0 = lt >> 3;
    if (grp == 0) {
      // Q rows travel with the first K/V block
      int rows[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int slot = q0 + r0 + 8 * i;
        rows[i] = slot < a.N ? attn_row(a, t, slot) : -1;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = r0 + 8 * i;
        const bool ok = rows[i] >= 0;
        const bf16* src = qkv + (ok ? static_cast<size_t>(rows[i]) * ld + h * 64 + ch * 8 : 0);
        cp_async16(sb + AttnSmem::Q + swz(r, ch), src, ok);
      }
    }
    for (int j = grp; j < nkb; j += 2) {
      const int b = grp;
      if (j >= 2 && !mbar_wait(bar_kvempty + 8 * b, ((j >> 1) - 1) & 1)) break;
      int rows[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int slot = 1 + j * kAttnBK + r0 + 8 * i;
        rows[i] = slot < a.N ? attn_row(a, t, slot) : -1;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = r0 + 8 * i;
        const bool ok = rows[i] >= 0;
        const size_t base = ok ? static_cast<size_t>(rows[i]) * ld + h * 64 + ch * 8 : 0;
        cp_async16(sb + AttnSmem::K + b * 16384 + swz(r, ch), qkv + base + (ok ? a.d : 0), ok);
        cp_async16(sb + AttnSmem::V + b * 16384 + swz(r, ch), qkv + base + (ok ? 2 * a.d : 0), ok);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(bar_kvfull + 8 * b);
    }
    cp_async_wait<0>();
  } else if (warp == 8) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_make(1u, 128);                 // Q K^T: M 128, N 128
      constexpr uint32_t IDESC_O = idesc_make(1u, 64) | (1u << 16);     // P V: M 128, N 64, B MN-major
      const uint64_t dq = sdesc_sw128(sb + AttnSmem::Q);
      bool ok = mbar_wait(bar_kvfull, 0);
      if (ok) {
        tc_fence_after();
        const uint64_t dk = sdesc_sw128(sb + AttnSmem::K);
#pragma unroll
        for (int k = 0; k < 4; ++k) tc_mma_f16(tS, dq + 2 * k, dk + 2 * k, IDESC_S, k != 0);
        tc_commit(bar_sfull);
      }
      for (int j = 0; j < nkb && ok; ++j) {
        const int b = j & 1;
        if (j + 1 < nkb) {
          const int b1 = (j + 1) & 1;
          ok = mbar_wait(bar_kvfull + 8 * b1, ((j + 1) >> 1) & 1) && mbar_wait(bar_sfree, j & 1);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dk = sdesc_sw128(sb + AttnSmem::K + b1 * 16384);
#pragma unroll
          for (int k = 0; k < 4; ++k) tc_mma_f16(tS, dq + 2 * k, dk + 2 * k, IDESC_S, k != 0);
          tc_commit(bar_sfull);
        }
        if (!mbar_wait(bar_pfull, j & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t dp = sdesc_sw128(sb + AttnSmem::P + (kk >> 2) * 16384) + 2 * (kk & 3);
          const uint64_t dv = sdesc_sw128_mn(sb + AttnSmem::V + b * 16384 + kk * 2048);
          tc_mma_f16(tO, dp, dv, IDESC_O, (j | kk) != 0);
        }
        tc_commit(bar_odone);
        tc_commit(bar_kvempty + 8 * b);
      }
    }
  } else {
    // ---------------- softmax: one query row per thread ----------------
    const int row = tid;                     // 0..127, TMEM lane = row
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    bool ok = mbar_wait(bar_kvfull, 0);      // Q rows are in shared memory
    float m = -INFINITY, l = 0.f, gcoef = 0.f;
    if (ok) {
      // score of the global key
      float sg = 0.f;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(smem + AttnSmem::Q + swz(row, ch)), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) sg = fmaf(f[e], sKg[ch * 8 + e], sg);
      }
      m = sg * a.scale_log2;
      l = 1.f;
      gcoef = 1.f;
    }
    for (int j = 0; j < nkb && ok; ++j) {
      if (!mbar_wait(bar_sfull, j & 1)) { ok = false; break; }
      tc_fence_after();
      const int kbase = j * kAttnBK;
      // pass 1: row maximum of the block (32-column chunks of S read from TMEM)
      float mx = m;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float sv[32];
        tmem_ld32(tS + lane_off + c * 32, sv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (kbase + c * 32 + i < a.Nw) mx = fmaxf(mx, sv[i] * a.scale_log2);
      }
      const float alpha = exp2f(m - mx);
      // P_{j-1} and O are in use by the previous P V until it completes
      if (j >= 1) {
        if (!mbar_wait(bar_odone, (j - 1) & 1)) { ok = false; break; }
        tc_fence_after();
      }
      // pass 2: probabilities as bf16 into P (keys 0-63 low block, 64-127 high block)
      float sum = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float sv[32];
        tmem_ld32(tS + lane_off + c * 32, sv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p = (kbase + c * 32 + i < a.Nw) ? exp2f(sv[i] * a.scale_log2 - mx) : 0.f;
          sv[i] = p;
          sum += p;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = c * 4 + q;     // 16-byte chunk of the 256-byte P row
          uint4 u;
          u.x = pack_bf16(sv[q * 8 + 0], sv[q * 8 + 1]);
          u.y = pack_bf16(sv[q * 8 + 2], sv[q * 8 + 3]);
          u.z = pack_bf16(sv[q * 8 + 4], sv[q * 8 + 5]);
          u.w = pack_bf16(sv[q * 8 + 6], sv[q * 8 + 7]);
          *reinterpret_cast<uint4*>(smem + AttnSmem::P + (ch >> 3) * 16384 + swz(row, ch & 7)) = u;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_sfree);   // S fully read: the next Q K^T may overwrite it
      l = l * alpha + sum;
      gcoef *= alpha;
      m = mx;
      // rescale the running output when this warp's maxima moved
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          float o[32];
          tmem_ld32(tO + lane_off + hh * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= alpha;
          tmem_st32(tO + lane_off + hh * 32, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull);
    }
    if (ok && mbar_wait(bar_odone, (nkb - 1) & 1)) {
      tc_fence_after();
      const int slot = q0 + row;
      const float inv = 1.f / l;
      bf16* dst = reinterpret_cast<bf16*>(a.O) + (static_cast<size_t>(t) * a.N + slot) * a.d + h * 64;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        float o[32];
        tmem_ld32(tO + lane_off + hh * 32, o);
        tmem_wait_ld();
        if (slot < a.N) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = (o[c + e] + gcoef * sVg[hh * 32 + c + e]) * inv;
            *reinterpret_cast<uint4*>(dst + hh * 32 + c) = f32_to_bf16x8(f);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// the global token's query (slot 0): each warp takes every nw-th key, its lanes
// own two of the 64 channels; the warps' partial softmax states are merged at the
// end by warp 0.
__device__ __forceinline__ void attn_global_row(const AttnArgs& a, int h, int t, uint8_t* smem) {
  const bf16* qkv = reinterpret_cast<const bf16*>(a.qkv);
  const int ld = 3 * a.d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  float* sm = reinterpret_cast<float*>(smem);     // nw maxima
  float* sl = sm + 32;                            // nw sums
  float* sacc = sl + 32;                          // nw x 64
  pdl_wait();
  pdl_trigger();
  const __nv_bfloat162 q2 =
      *reinterpret_cast<const __nv_bfloat162*>(qkv + static_cast<size_t>(attn_row(a, t, 0)) * ld + h * 64 + 2 * lane);
  const float2 q = __bfloat1622float2(q2);
  float m = -INFINITY, l = 0.f, acc0 = 0.f, acc1 = 0.f;
  for (int s = warp; s < a.N; s += nw) {
    const bf16* kr = qkv + static_cast<size_t>(attn_row(a, t, s)) * ld + a.d + h * 64 + 2 * lane;
    const float2 k = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kr));
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kr + a.d));
    const float sc = warp_sum(q.x * k.x + q.y * k.y) * a.scale_log2;
    const float mn = fmaxf(m, sc);
    const float al = exp2f(m - mn), p = exp2f(sc - mn);
    l = l * al + p;
    acc0 = acc0 * al + p * v.x;
    acc1 = acc1 * al + p * v.y;
    m = mn;
  }
  if (lane == 0) {
    sm[warp] = m;
    sl[warp] = l;
  }
  sacc[warp * 64 + 2 * lane] = acc0;
  sacc[warp * 64 + 2 * lane + 1] = acc1;
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, sm[w]);
    float L = 0.f, o0 = 0.f, o1 = 0.f;
    for (int w = 0; w < nw; ++w) {
      const float f = sm[w] == -INFINITY ? 0.f : exp2f(sm[w] - M);
      L += f * sl[w];
      o0 += f * sacc[w * 64 + 2 * lane];
      o1 += f * sacc[w * 64 + 2 * lane + 1];
    }
    bf16* O = reinterpret_cast<bf16*>(a.O) + static_cast<size_t>(t) * a.N * a.d + h * 64 + 2 * lane;
    *reinterpret_cast<__nv_bfloat162*>(O) = __floats2bfloat162_rn(o0 / L, o1 / L);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 2) attn_bf16_kernel(const AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {          // swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) set_status(kStatusDeviceCheck);
    return;
  }
  const int nqb = gridDim.x - 1;
  const int qb = blockIdx.x, h = blockIdx.y, t = blockIdx.z;
  if (qb < nqb)
    attn_window_block_tc(a, qb, h, t, smem);
  else
    attn_global_row(a, h, t, smem);
}

// ---------------------------------------------------------------------------
// fp32 attention: one thread per query row (reference-precision path)
// ---------------------------------------------------------------------------
template <int HD>
__global__ void __launch_bounds__(64) attn_f32_kernel(const AttnArgs a) {
  const float* qkv = reinterpret_cast<const float*>(a.qkv);
  const int ld = 3 * a.d;
  const int h = blockIdx.y, t = blockIdx.z;
  const int slot = blockIdx.x * 64 + threadIdx.x;
  __shared__ float sk[64][HD + 1];
  __shared__ float sv[64][HD + 1];
  float q[HD], acc[HD];
  const bool active = slot < a.N;
  if (active) {
    const float* qr = qkv + static_cast<size_t>(attn_row(a, t, slot)) * ld + h * HD;
#pragma unroll
    for (int c = 0; c < HD; ++c) q[c] = qr[c];
  }
#pragma unroll
  for (int c = 0; c < HD; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int k0 = 0; k0 < a.N; k0 += 64) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 64 * HD; idx += 64) {
      const int r = idx / HD, c = idx % HD;
      const int s = k0 + r;
      float kv = 0.f, vv = 0.f;
      if (s < a.N) {
        const float* base = qkv + static_cast<size_t>(attn_row(a, t, s)) * ld + h * HD + c;
        kv = base[a.d];
        vv = base[2 * a.d];
      }
      sk[r][c] = kv;
      sv[r][c] = vv;
    }
    __syncthreads();
    if (active) {
      const int nk = min(64, a.N - k0);
      for (int r = 0; r < nk; ++r) {
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < HD; ++c) dot = fmaf(q[c], sk[r][c], dot);
        const float sc = dot * a.scale;
        const float mn = fmaxf(m, sc);
        const float al = expf(m - mn), p = expf(sc - mn);
        l = l * al + p;
#pragma unroll
        for (int c = 0; c < HD; ++c) acc[c] = acc[c] * al + p * sv[r][c];
        m = mn;
      }
    }
  }
  if (active) {
    float* O = reinterpret_cast<float*>(a.O) + (static_cast<size_t>(t) * a.N + slot) * a.d + h * HD;
    const float inv = 1.f / l;
#pragma unroll
    for (int c = 0; c < HD; ++c) O[c] = acc[c] * inv;
  }
}

}  // namespace ts
