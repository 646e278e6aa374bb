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
// bf16 kernel (hd = 64), grid (nqb, heads, T), 288 threads, 2 CTAs per SM:
//   blocks qb < nqb: 128 window queries, keys in blocks of 64.
//     warps 4-7  loaders: cp.async gathers of Q (once) and of K/V blocks through
//                the row map into 128-byte-swizzled shared rows; loader warp w
//                owns K/V buffer w (blocks w, w+4, ...), so three blocks are in
//                flight ahead of the math; each block is published with
//                fence.proxy.async and an mbarrier;
//     warp 8     MMA issuer (one lane): S = Q K^T (tcgen05 kind::f16, M = 128,
//                N = 64) into one of two TMEM S buffers, then O += P V (M = 128,
//                N = 64, V read as an MN-major operand) into TMEM; S of block j+1
//                is issued as soon as the softmax has read block j-1's buffer;
//     warps 0-3  softmax, one query row per thread (TMEM lane = row): one tcgen05
//                round trip brings the row's 64 scores into registers; online
//                softmax in the exp2 domain with a lazily moved reference maximum
//                (O rescaled in TMEM only when a score exceeds it by 2^8); P as
//                bf16 into one of two swizzled shared buffers; the global key
//                (slot 0) seeds the running max and sum and is added back at the
//                end with its running coefficient.
//   The global token's own query row (slot 0) rides along in query block 0: its
//     loader warps update an online softmax for it on every K/V block they load
//     (lanes own channel pairs) and merge their partial states at the end.
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
constexpr int kAttnBK = 64;              // keys per block
constexpr int kAttnKV = 4;               // K/V buffers (one loader warp each)
constexpr float kAttnRescale = 8.0f;     // lazy rescale threshold (log2 units)

struct AttnSmem {
  static constexpr int Q = 0;                 // 16 KB: 128 rows x 128 B
  static constexpr int K = 16384;             // 4 x 8 KB: 64 rows x 128 B
  static constexpr int V = 16384 + 32768;     // 4 x 8 KB
  static constexpr int P = 16384 + 65536;     // 2 x 16 KB: 128 rows x 64 keys
  static constexpr int KG = P + 32768;        // 64 floats k_g, 64 floats v_g
  static constexpr int BAR = KG + 512;        // barriers
  static constexpr int NBAR = 17;
  static constexpr int BYTES = BAR + NBAR * 8 + 16;
  static constexpr int LAUNCH_BYTES = BYTES;  // base must be 1024-aligned (checked): two CTAs per SM
};

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
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 2^x by the PTX approximate base-2 exponential (2 ulp; -inf gives 0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// packed pairs of floats (low = first) and the sm_100 f32x2 arithmetic on them
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float lo_f32(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo;
}
__device__ __forceinline__ float hi_f32(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return hi;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------------------
// window-query block (tcgen05)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void attn_window_block_tc(const AttnArgs& a, int qb, int h, int t, uint8_t* smem) {
  const bf16* qkv = reinterpret_cast<const bf16*>(a.qkv);
  const int ld = 3 * a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_kvfull = sb + AttnSmem::BAR;        // 4, count 32 (one loader warp each)
  const uint32_t bar_kvempty = bar_kvfull + 32;          // 4, count 1 (commit after P V)
  const uint32_t bar_sfull = bar_kvempty + 32;           // 2, count 1 (commit after Q K^T)
  const uint32_t bar_sfree = bar_sfull + 16;             // 2, count 4 (softmax warps read S)
  const uint32_t bar_pfull = bar_sfree + 16;             // 2, count 4 (softmax warps wrote P)
  const uint32_t bar_odone = bar_pfull + 16;             // 2, count 1 (commit after P V)
  const uint32_t bar_ofinal = bar_odone + 16;            // 1, count 1 (commit after the last P V)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + AttnSmem::BAR + AttnSmem::NBAR * 8);
  float* sKg = reinterpret_cast<float*>(smem + AttnSmem::KG);
  float* sVg = sKg + 64;
  const int nkb = (a.Nw + kAttnBK - 1) / kAttnBK;
  const int q0 = 1 + qb * kAttnBQ;  // first slot of this query block

  if (warp == 8 && lane == 0) {
    for (int i = 0; i < kAttnKV; ++i) {
      mbar_init(bar_kvfull + 8 * i, 32);
      mbar_init(bar_kvempty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sfull + 8 * i, 1);
      mbar_init(bar_sfree + 8 * i, 4);
      mbar_init(bar_pfull + 8 * i, 4);
      mbar_init(bar_odone + 8 * i, 1);
    }
    mbar_init(bar_ofinal, 1);
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), 256);    // S0: cols 0-63, S1: 64-127, O: 128-191
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
  const uint32_t tO = tmem + 128;

  if (warp >= 4 && warp < 8) {
    // ---------------- loaders: warp wl owns K/V buffer wl, blocks wl, wl + 4, ... ----------------
    // The row indices of a block are read with one coalesced load (lane l holds
    // rows l and 32 + l) and handed to the lanes that copy them by shuffles; the
    // indices of a warp's next block are fetched before it waits for its buffer.
    const int wl = warp - 4;
    const int ch = lane & 7, r0 = lane >> 3;       // chunk ch of rows r0 + 4 i
    auto row_of = [&](int slot) { return slot < a.N ? attn_row(a, t, slot) : -1; };
    if (wl == 0) {
      // Q rows (128 x 8 chunks) travel with block 0
      int vq[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) vq[k] = row_of(q0 + 32 * k + lane);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = r0 + 4 * i;
        const int row = __shfl_sync(0xffffffffu, vq[i >> 3], r & 31);
        const bool ok = row >= 0;
        const bf16* src = qkv + (ok ? static_cast<size_t>(row) * ld + h * 64 + ch * 8 : 0);
        cp_async16(sb + AttnSmem::Q + swz(r, ch), src, ok);
      }
    }
    int v0 = wl < nkb ? row_of(1 + wl * kAttnBK + lane) : -1;
    int v1 = wl < nkb ? row_of(1 + wl * kAttnBK + 32 + lane) : -1;
    // The CTA of query block 0 also computes the global token's own query row
    // (slot 0): every loader warp runs an online softmax for it over the K/V
    // blocks it has just loaded, its lanes owning channels 2 lane and 2 lane + 1.
    const bool grow_row = qb == 0;
    float gm = -INFINITY, gl = 0.f, ga0 = 0.f, ga1 = 0.f;
    float2 gq = make_float2(0.f, 0.f);
    if (grow_row) {
      const size_t r = static_cast<size_t>(attn_row(a, t, 0));
      gq = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qkv + r * ld + h * 64 + 2 * lane));
      if (wl == 0) {   // the global key itself
        gm = warp_sum(gq.x * sKg[2 * lane] + gq.y * sKg[2 * lane + 1]) * a.scale_log2;
        gl = 1.f;
        ga0 = sVg[2 * lane];
        ga1 = sVg[2 * lane + 1];
      }
    }
    for (int j = wl; j < nkb; j += kAttnKV) {
      if (j >= kAttnKV && !mbar_wait(bar_kvempty + 8 * wl, ((j / kAttnKV) - 1) & 1)) break;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = r0 + 4 * i;
        const int row = __shfl_sync(0xffffffffu, i < 8 ? v0 : v1, r & 31);
        const bool ok = row >= 0;
        const size_t base = ok ? static_cast<size_t>(row) * ld + h * 64 + ch * 8 : 0;
        cp_async16(sb + AttnSmem::K + wl * 8192 + swz(r, ch), qkv + base + (ok ? a.d : 0), ok);
        cp_async16(sb + AttnSmem::V + wl * 8192 + swz(r, ch), qkv + base + (ok ? 2 * a.d : 0), ok);
      }
      cp_async_commit();
      const int jn = j + kAttnKV;
      v0 = jn < nkb ? row_of(1 + jn * kAttnBK + lane) : -1;
      v1 = jn < nkb ? row_of(1 + jn * kAttnBK + 32 + lane) : -1;
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(bar_kvfull + 8 * wl);
      if (grow_row) {
        __syncwarp();                    // the block's rows were copied by all lanes of this warp
        const uint8_t* kbuf = smem + AttnSmem::K + wl * 8192;
        const uint8_t* vbuf = smem + AttnSmem::V + wl * 8192;
        const int nvalid = min(kAttnBK, a.Nw - j * kAttnBK);
#pragma unroll 1
        for (int rb = 0; rb < nvalid; rb += 8) {
          float sc[8];
          float2 vv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t off = swz(rb + i, lane >> 2) + (lane & 3) * 4;
            const float2 kk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kbuf + off));
            vv[i] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vbuf + off));
            sc[i] = gq.x * kk.x + gq.y * kk.y;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int i = 0; i < 8; ++i) sc[i] += __shfl_xor_sync(0xffffffffu, sc[i], o);
          float mx = gm;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            sc[i] = rb + i < nvalid ? sc[i] * a.scale_log2 : -INFINITY;
            mx = fmaxf(mx, sc[i]);
          }
          const float al = exp2f(gm - mx);
          gl *= al;
          ga0 *= al;
          ga1 *= al;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float pr = exp2f(sc[i] - mx);
            gl += pr;
            ga0 = fmaf(pr, vv[i].x, ga0);
            ga1 = fmaf(pr, vv[i].y, ga1);
          }
          gm = mx;
        }
      }
    }
    cp_async_wait<0>();
    if (grow_row) {
      // merge the four loader warps' states through the P buffer, idle once the
      // last P V has completed; the named barrier spans the loader warps only
      const bool ok_g = mbar_wait(bar_ofinal, 0);
      float* gbuf = reinterpret_cast<float*>(smem + AttnSmem::P);
      if (ok_g) {
        if (lane == 0) {
          gbuf[wl * 66] = gm;
          gbuf[wl * 66 + 1] = gl;
        }
        gbuf[wl * 66 + 2 + 2 * lane] = ga0;
        gbuf[wl * 66 + 3 + 2 * lane] = ga1;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (ok_g && wl == 0) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttnKV; ++w) M = fmaxf(M, gbuf[w * 66]);
        float L = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
        for (int w = 0; w < kAttnKV; ++w) {
          const float f = gbuf[w * 66] == -INFINITY ? 0.f : exp2f(gbuf[w * 66] - M);
          L += f * gbuf[w * 66 + 1];
          o0 += f * gbuf[w * 66 + 2 + 2 * lane];
          o1 += f * gbuf[w * 66 + 3 + 2 * lane];
        }
        bf16* O = reinterpret_cast<bf16*>(a.O) + static_cast<size_t>(t) * a.N * a.d + h * 64 + 2 * lane;
        *reinterpret_cast<__nv_bfloat162*>(O) = __floats2bfloat162_rn(o0 / L, o1 / L);
      }
    }
  } else if (warp == 8) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_make(1u, kAttnBK);             // Q K^T: M 128, N 64
      constexpr uint32_t IDESC_O = idesc_make(1u, 64) | (1u << 16);     // P V: M 128, N 64, B MN-major
      const uint64_t dq = sdesc_sw128(sb + AttnSmem::Q);
      auto issue_s = [&](int j) -> bool {
        const int b = j % kAttnKV, sbuf = j & 1;
        if (!mbar_wait(bar_kvfull + 8 * b, (j / kAttnKV) & 1)) return false;
        if (j >= 2 && !mbar_wait(bar_sfree + 8 * sbuf, ((j >> 1) - 1) & 1)) return false;
        tc_fence_after();
        const uint64_t dk = sdesc_sw128(sb + AttnSmem::K + b * 8192);
#pragma unroll
        for (int k = 0; k < 4; ++k) tc_mma_f16(tmem + sbuf * 64, dq + 2 * k, dk + 2 * k, IDESC_S, k != 0);
        tc_commit(bar_sfull + 8 * sbuf);
        return true;
      };
      bool ok = issue_s(0);
      for (int j = 0; j < nkb && ok; ++j) {
        if (j + 1 < nkb && !(ok = issue_s(j + 1))) break;
        const int pb = j & 1, b = j % kAttnKV;
        if (!mbar_wait(bar_pfull + 8 * pb, (j >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dp = sdesc_sw128(sb + AttnSmem::P + pb * 16384);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t dv = sdesc_sw128_mn(sb + AttnSmem::V + b * 8192 + kk * 2048);
          tc_mma_f16(tO, dp + 2 * kk, dv, IDESC_O, (j | kk) != 0);
        }
        tc_commit(bar_odone + 8 * pb);
        tc_commit(bar_kvempty + 8 * b);
      }
      // single-phase barrier: waiters may arrive any number of phases early
      if (ok) tc_commit(bar_ofinal);
    }
  } else {
    // ---------------- softmax: one query row per thread ----------------
    const int row = tid;                     // 0..127, TMEM lane = row
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    bool ok = mbar_wait(bar_kvfull, 0);      // Q rows are in shared memory
    float m = -INFINITY, l = 0.f, gcoef = 0.f;
    if (ok) {
      // score of the global key seeds the running maximum and sum
      float sg = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(smem + AttnSmem::Q + swz(row, c)), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) sg = fmaf(f[e], sKg[c * 8 + e], sg);
      }
      m = sg * a.scale_log2;
      l = 1.f;
      gcoef = 1.f;
    }
    for (int j = 0; j < nkb && ok; ++j) {
      const int sbuf = j & 1;
      if (!mbar_wait(bar_sfull + 8 * sbuf, (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      float sv[kAttnBK];
      tmem_ld32(tmem + sbuf * 64 + lane_off, sv);
      tmem_ld32(tmem + sbuf * 64 + lane_off + 32, sv + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_sfree + 8 * sbuf);   // S buffer may be overwritten
      const int kbase = j * kAttnBK;
      // row maximum of the raw scores (the scale is positive); keys beyond the
      // window exist only in the last block
      if (kbase + kAttnBK > a.Nw) {
#pragma unroll
        for (int i = 0; i < kAttnBK; ++i)
          if (kbase + i >= a.Nw) sv[i] = -INFINITY;
      }
      // eight independent partial maxima keep the dependency chains short
      float mp[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mp[q] = sv[q];
#pragma unroll
      for (int i = 8; i < kAttnBK; ++i) mp[i & 7] = fmaxf(mp[i & 7], sv[i]);
      const float mr = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      const float mx = mr * a.scale_log2;
      // lazy rescale: the reference maximum moves only when a score exceeds it by
      // more than 2^8, so probabilities stay below 256 and O is rarely touched
      const bool grow = mx > m + kAttnRescale;
      const float mnew = grow ? mx : m;
      const float alpha = exp2f(m - mnew);
      const bool warp_grow = __any_sync(0xffffffffu, grow);
      l *= alpha;
      gcoef *= alpha;
      m = mnew;
      // pairs of scores through packed f32x2 arithmetic: one FMA per pair forms the
      // exponents, the SFU takes each exponential, four packed partial sums
      const uint64_t sc2 = pack_f32x2(a.scale_log2, a.scale_log2), nm2 = pack_f32x2(-m, -m);
      uint64_t sp2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int i = 0; i < kAttnBK; i += 2) {
        const uint64_t x2 = fma_f32x2(pack_f32x2(sv[i], sv[i + 1]), sc2, nm2);
        sv[i] = ex2_approx(lo_f32(x2));
        sv[i + 1] = ex2_approx(hi_f32(x2));
        sp2[(i >> 1) & 3] = add_f32x2(sp2[(i >> 1) & 3], pack_f32x2(sv[i], sv[i + 1]));
      }
      const uint64_t s01 = add_f32x2(sp2[0], sp2[1]), s23 = add_f32x2(sp2[2], sp2[3]);
      const uint64_t s0123 = add_f32x2(s01, s23);
      l += lo_f32(s0123) + hi_f32(s0123);
      // P buffer sbuf was last read by P V of block j-2
      if (j >= 2 && !mbar_wait(bar_odone + 8 * sbuf, ((j - 2) >> 1) & 1)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = pack_bf16(sv[c * 8 + 0], sv[c * 8 + 1]);
        u.y = pack_bf16(sv[c * 8 + 2], sv[c * 8 + 3]);
        u.z = pack_bf16(sv[c * 8 + 4], sv[c * 8 + 5]);
        u.w = pack_bf16(sv[c * 8 + 6], sv[c * 8 + 7]);
        *reinterpret_cast<uint4*>(smem + AttnSmem::P + sbuf * 16384 + swz(row, c)) = u;
      }
      if (warp_grow && j >= 1) {
        // O holds the sum up to block j-1: wait for that P V, then rescale the row
        if (!mbar_wait(bar_odone + 8 * ((j - 1) & 1), ((j - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int hh = 0; hh < 4; ++hh) {
          float o[16];
          tmem_ld16(tO + lane_off + hh * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] *= alpha;
          tmem_st16(tO + lane_off + hh * 16, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull + 8 * sbuf);
    }
    if (ok && mbar_wait(bar_ofinal, 0)) {
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

__global__ void __launch_bounds__(kAttnThreads, 2) attn_bf16_kernel(const AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {          // swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) set_status(kStatusDeviceCheck);
    return;
  }
  attn_window_block_tc(a, blockIdx.x, blockIdx.y, blockIdx.z, smem);
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
