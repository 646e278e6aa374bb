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
// bf16 kernel (hd = 64), 320 threads, 2 CTAs per SM, each CTA two query tiles of
// 128 rows that share one K/V stream: eight softmax warps per CTA, so that four
// softmax warps share each scheduler and one tile's softmax runs while the other
// tile's MMAs do.  Shared layer: grid (nqb + 1, T, heads), the head slowest, so that
// CTAs in flight together work on one head of neighbouring tiles, whose overlapping
// q/k/v rows (one head's slice of the whole shared state: a few MB) then come from
// L2 instead of DRAM.  Per-tile layer (no rows shared between tiles): grid
// (nqb + 1, heads, T), the tile slowest, so that the heads of one tile run together
// and each tile's q/k/v rows (all heads' column slices of the same rows) leave DRAM
// once.
//   blocks qb < nqb: 256 window queries (two tiles), keys in blocks of 64.
//     warp 8     TMA producer of Q (once) and of K/V blocks into 128-byte-
//                swizzled shared rows: one box of a 3-D map over the grid per
//                block when a block is whole window rows of one frame, else one
//                2-D box per run of consecutive rows, else tile::gather4 loads
//                through the row map (four rows per instruction); four K/V
//                buffers, completion by transaction bytes on one mbarrier each;
//     warp 9     MMA issuer (one lane): per tile S = Q K^T (tcgen05 kind::f16,
//                M = 128, N = 64) into the tile's TMEM S buffer, then O += P V
//                with P read from TMEM (A operand) and V from shared memory as an
//                MN-major operand; S of block j+1 overwrites P of block j and is
//                issued after its P V (tcgen05.mma runs in issue order); the two
//                tiles alternate;
//     warps 0-7  softmax, one query row per thread (warps 0-3 tile 0, 4-7 tile 1;
//                TMEM lane = row): one tcgen05 round trip brings the row's 64
//                scores into registers; online softmax in the exp2 domain with a
//                lazily moved reference maximum (O rescaled in TMEM only when a
//                score exceeds it by 2^8); P goes back over the scores as packed
//                bf16; the global key (slot 0) seeds the running max and sum and
//                is added back at the end with its running coefficient.
//   block qb = nqb: the global token's own query row (slot 0) of the tile and
//                head: warp 8 streams the K/V blocks as for a window block, eight
//                warps score them from shared memory (lane = key) with an online
//                softmax each, merged at the end.
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
  int load;           // K/V/Q loads: 0 four-row gathers, 1 runs of `run` rows (2-D boxes), 2 grid boxes
  int run;            // load 1: slots 1 + k*run ... come in runs of `run` consecutive rows
  int gw;             // load 2: grid width; shared row u is grid row u / gw, column u % gw
  float scale_log2;   // log2(e) / sqrt(hd)
  float scale;        // 1 / sqrt(hd)
  int head_major;     // bf16 grid: 1 (nqb + 1, T, heads), head slowest; 0 (nqb + 1, heads, T), tile slowest
  int nqb;            // bf16: window query blocks (256 queries) per tile; block x = nqb is the global row
};

__device__ __forceinline__ int attn_row(const AttnArgs& a, int t, int s) {
  return a.rowmap ? __ldg(a.rowmap + t * a.N + s) : t * a.N + s;
}

// byte offset of 16-byte chunk `ch` of row `r` in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz(int r, int ch) { return r * 128 + ((ch ^ (r & 7)) << 4); }

constexpr int kAttnThreads = 320;        // 8 softmax warps (two query tiles), TMA producer, MMA issuer
constexpr int kAttnCtasPerSm = 2;
constexpr int kAttnTileQ = 128;          // queries per tile (M of the MMAs)
constexpr int kAttnBQ = 2 * kAttnTileQ;  // queries per CTA
constexpr int kAttnBK = 64;              // keys per block
constexpr int kAttnKV = 4;               // K/V buffers
constexpr int kAttnTmemCols = 256;       // per tile: S / P (64 columns), then O (64 columns)
constexpr int kAttnTmemTile = 128;       // TMEM columns of one query tile
constexpr float kAttnRescale = 8.0f;     // lazy rescale threshold (log2 units)
#ifndef TS_ATTN_EMU_EVERY
#define TS_ATTN_EMU_EVERY 4
#endif
constexpr int kAttnEmuEvery = TS_ATTN_EMU_EVERY;   // one score pair in this many: 2^x on the FMA pipe

struct AttnSmem {
  static constexpr int KV_BYTES = kAttnBK * 128;       // one K or V block: 64 rows x 128 B
  static constexpr int Q = 0;                          // 32 KB: 2 tiles x 128 rows x 128 B
  static constexpr int K = kAttnBQ * 128;              // kAttnKV x 8 KB
  static constexpr int V = K + kAttnKV * KV_BYTES;     // kAttnKV x 8 KB
  static constexpr int KG = V + kAttnKV * KV_BYTES;    // 64 floats k_g, 64 floats v_g
  static constexpr int BAR = KG + 512;                 // barriers
  static constexpr int NBAR = 2 * kAttnKV + 2 + 2 + 2 + 1; // kvfull, kvempty, sfull[2], pfull[2], ofinal[2], qfull1
  static constexpr int BYTES = BAR + NBAR * 8 + 8;
  static_assert((8 * 66 + 8 + 64) * 4 <= kAttnBQ * 128, "global-row states and query in the Q region");
  // the base is rounded up to 1024 bytes inside the kernel (swizzled tiles)
  static constexpr int LAUNCH_BYTES = BYTES + 1024;
  static_assert(kAttnCtasPerSm * (LAUNCH_BYTES + 1024) <= 228 * 1024, "shared memory for 2 CTAs per SM");
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

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
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
// 2^x of a pair of exponents on the FMA pipe, for x <= 2^7 (x below -125 is
// taken as -125, whose power is below every probability that matters here).
// Range reduction by the round-to-nearest addition of 1.5 * 2^23: the sum's low
// mantissa bits hold the integer j nearest to x, and f = x - j lies in
// [-1/2, 1/2] exactly.  2^f is a cubic fitted here for least maximum relative
// error on [-1/2, 1/2] (Lawson's iteration; 7.5e-5, far below the 2^-9 of the
// bf16 rounding of P), evaluated by Horner's rule on pairs; 2^j enters by adding
// j to the result's exponent field (j << 23 wraps the 1.5 * 2^23 offset away).
__device__ __forceinline__ void exp2_fma2(uint64_t x2, float& e0, float& e1) {
  const float x0 = fmaxf(lo_f32(x2), -125.f), x1 = fmaxf(hi_f32(x2), -125.f);
  const uint64_t xc = pack_f32x2(x0, x1);
  const uint64_t t = add_f32x2(xc, pack_f32x2(12582912.f, 12582912.f));
  const uint64_t j = add_f32x2(t, pack_f32x2(-12582912.f, -12582912.f));
  const uint64_t f = fma_f32x2(j, pack_f32x2(-1.f, -1.f), xc);
  uint64_t p = fma_f32x2(pack_f32x2(0.0551716685295105f, 0.0551716685295105f), f,
                         pack_f32x2(0.2426111251115799f, 0.2426111251115799f));
  p = fma_f32x2(p, f, pack_f32x2(0.6932609677314758f, 0.6932609677314758f));
  p = fma_f32x2(p, f, pack_f32x2(0.9999280571937561f, 0.9999280571937561f));
  e0 = __uint_as_float(__float_as_uint(lo_f32(p)) + (__float_as_uint(lo_f32(t)) << 23));
  e1 = __uint_as_float(__float_as_uint(hi_f32(p)) + (__float_as_uint(hi_f32(t)) << 23));
}
// true in exactly one lane of the (fully active) warp
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(pred));
  return pred != 0;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Four rows (r0..r3) of one 128-byte column box (x = first element) gathered by
// TMA into 512 consecutive bytes of shared memory, 128-byte swizzled like a
// tiled load; completion is signalled on `bar` as transaction bytes.  The tensor
// map's box is one row high.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const void* map, uint32_t bar, int x, int r0, int r1, int r2,
                                            int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem desc): A is read from tensor memory (row i in lane
// i, two bf16 K elements per 32-bit column, the lower K index in the low half).
__device__ __forceinline__ void tc_mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// What the three load variants of the producer warp share.
struct AttnLoad {
  const CUtensorMap* tm;
  uint32_t sb, bar_kvfull, bar_kvempty, bar_q1;   // bar_q1 = 0: K/V only (global-row block), no Q
  int q0, nkb, t, h, lane;
};

// Tile 0's Q (128 rows) travels with K/V block 0 on its barrier, tile 1's Q on a
// barrier of its own.
constexpr uint32_t kAttnTxFirst = kAttnTileQ * 128 + 2 * AttnSmem::KV_BYTES;
constexpr uint32_t kAttnTxQ1 = kAttnTileQ * 128;
constexpr uint32_t kAttnTxBlock = 2 * AttnSmem::KV_BYTES;

__device__ __forceinline__ void attn_load_grid(const AttnArgs& a, const AttnLoad& c) {
  const CUtensorMap* tm = c.tm;
  const uint32_t sb = c.sb, bar_kvfull = c.bar_kvfull, bar_kvempty = c.bar_kvempty;
  const int q0 = c.q0, nkb = c.nkb, t = c.t, h = c.h, lane = c.lane;
  // ---------------- TMA producer, one grid box per 64 slots ----------------
  // A block of 64 window slots is 64 / bx whole window rows of one frame (or a
  // part of one row): one box of the 3-D map (channels, grid column, grid row)
  // starting at the grid position of its first slot.  Blocks past the tile's
  // last slot load block 0 again.
  auto box_at = [&](int slot, int& x, int& y) {
    const int u = attn_row(a, t, slot < a.N ? slot : 1);
    x = u % a.gw;
    y = u / a.gw;
  };
  if (lane == 0) {
    const int xq = h * 64, xk = a.d + h * 64, xv = 2 * a.d + h * 64;
    int x, y;
    if (c.bar_q1) {
      mbar_expect_tx(bar_kvfull, kAttnTxFirst);
      mbar_expect_tx(c.bar_q1, kAttnTxQ1);
#pragma unroll
      for (int i = 0; i < kAttnBQ / kAttnBK; ++i) {
        box_at(q0 + i * kAttnBK, x, y);
        tma_load_3d(sb + AttnSmem::Q + i * AttnSmem::KV_BYTES, tm, i < kAttnTileQ / kAttnBK ? bar_kvfull : c.bar_q1,
                    xq, x, y);
      }
    } else {
      mbar_expect_tx(bar_kvfull, kAttnTxBlock);
    }
    int xn, yn;
    box_at(1, xn, yn);
    int armed = 0;
    for (int j = 0; j < nkb; ++j) {
      const int b = j % kAttnKV;
      const int xc = xn, yc = yn;
      if (j + 1 < nkb) box_at(1 + (j + 1) * kAttnBK, xn, yn);
      if (j > 0) {
        if (j >= kAttnKV && !mbar_wait(bar_kvempty + 8 * b, ((j / kAttnKV) - 1) & 1)) break;
        mbar_expect_tx(bar_kvfull + 8 * b, kAttnTxBlock);
      }
      tma_load_3d(sb + AttnSmem::K + b * AttnSmem::KV_BYTES, tm, bar_kvfull + 8 * b, xk, xc, yc);
      tma_load_3d(sb + AttnSmem::V + b * AttnSmem::KV_BYTES, tm, bar_kvfull + 8 * b, xv, xc, yc);
      armed = j + 1;
    }
    // no copy may still be landing when the CTA exits (matters only after a timeout)
    for (int j = max(0, armed - kAttnKV); j < armed; ++j) mbar_wait(bar_kvfull + 8 * (j % kAttnKV), (j / kAttnKV) & 1);
    if (c.bar_q1) mbar_wait(c.bar_q1, 0);
  }
}

__device__ __forceinline__ void attn_load_runs(const AttnArgs& a, const AttnLoad& c) {
  const CUtensorMap* tm = c.tm;
  const uint32_t sb = c.sb, bar_kvfull = c.bar_kvfull, bar_kvempty = c.bar_kvempty;
  const int q0 = c.q0, nkb = c.nkb, t = c.t, h = c.h, lane = c.lane;
  // ---------------- TMA producer, runs of consecutive rows ----------------
  // Each run of `run` slots (8, 16, 32 or 64) is one tiled box (128 bytes x run rows)
  // of the q/k/v columns of head h.  Runs past the tile's last slot (padding of
  // the last key or query block) load the first run again: their scores are
  // masked and their outputs are not stored.  Lane i looks up the row of run i one
  // block ahead; lane 0 issues the copies.
  const int L = a.run, nrun = kAttnBK / L;
  auto run_row = [&](int slot) { return attn_row(a, t, slot < a.N ? slot : 1); };
  const int xq = h * 64, xk = a.d + h * 64, xv = 2 * a.d + h * 64;
  if (c.bar_q1) {
    const int rq = lane < kAttnBQ / L ? run_row(q0 + lane * L) : 0;
    if (lane == 0) {
      mbar_expect_tx(bar_kvfull, kAttnTxFirst);
      mbar_expect_tx(c.bar_q1, kAttnTxQ1);
    }
    for (int i = 0; i < kAttnBQ / L; ++i) {
      const int r = __shfl_sync(0xffffffffu, rq, i);
      if (lane == 0) tma_load_2d(sb + AttnSmem::Q + i * L * 128, tm, i < kAttnTileQ / L ? bar_kvfull : c.bar_q1, xq, r);
    }
  } else if (lane == 0) {
    mbar_expect_tx(bar_kvfull, kAttnTxBlock);
  }
  int rnext = lane < nrun ? run_row(1 + lane * L) : 0;
  int armed = 0;
  for (int j = 0; j < nkb; ++j) {
    const int b = j % kAttnKV;
    const int rcur = rnext;
    if (j + 1 < nkb && lane < nrun) rnext = run_row(1 + (j + 1) * kAttnBK + lane * L);
    if (j > 0) {
      int ok = 1;
      if (lane == 0 && j >= kAttnKV) ok = mbar_wait(bar_kvempty + 8 * b, ((j / kAttnKV) - 1) & 1);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane == 0) mbar_expect_tx(bar_kvfull + 8 * b, kAttnTxBlock);
    }
    for (int i = 0; i < nrun; ++i) {
      const int r = __shfl_sync(0xffffffffu, rcur, i);
      if (lane == 0) {
        tma_load_2d(sb + AttnSmem::K + b * AttnSmem::KV_BYTES + i * L * 128, tm, bar_kvfull + 8 * b, xk, r);
        tma_load_2d(sb + AttnSmem::V + b * AttnSmem::KV_BYTES + i * L * 128, tm, bar_kvfull + 8 * b, xv, r);
      }
    }
    armed = j + 1;
  }
  // no copy may still be landing when the CTA exits (matters only after a timeout)
  if (lane == 0) {
    for (int j = max(0, armed - kAttnKV); j < armed; ++j) mbar_wait(bar_kvfull + 8 * (j % kAttnKV), (j / kAttnKV) & 1);
    if (c.bar_q1) mbar_wait(c.bar_q1, 0);
  }
}

__device__ __forceinline__ void attn_load_gather(const AttnArgs& a, const AttnLoad& c) {
  const CUtensorMap* tm = c.tm;
  const uint32_t sb = c.sb, bar_kvfull = c.bar_kvfull, bar_kvempty = c.bar_kvempty;
  const int q0 = c.q0, nkb = c.nkb, t = c.t, h = c.h, lane = c.lane;
  // ---------------- TMA producer, gathered rows ----------------
  // Rows are gathered four at a time (tile::gather4) from the q/k/v columns of
  // head h.  Slots past the tile's last one (padding of the last key or query
  // block) repeat the last slot's row, so every coordinate is in range; their
  // scores are masked and their outputs are not stored.  Lane i holds the rows of
  // slots i and 32 + i of the block.
  auto row_of = [&](int slot) { return attn_row(a, t, min(slot, a.N - 1)); };
  const int xq = h * 64, xk = a.d + h * 64, xv = 2 * a.d + h * 64;
  int vq[kAttnBQ / 32];
#pragma unroll
  for (int k = 0; k < kAttnBQ / 32; ++k) vq[k] = row_of(q0 + 32 * k + lane);
  if (c.bar_q1) {
    if (lane == 0) {
      mbar_expect_tx(bar_kvfull, kAttnTxFirst);
      mbar_expect_tx(c.bar_q1, kAttnTxQ1);
    }
#pragma unroll
    for (int g = 0; g < kAttnBQ / 4; ++g) {
      int r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) r[i] = __shfl_sync(0xffffffffu, vq[g >> 3], (4 * g + i) & 31);
      if (lane == 0)
        tma_gather4(sb + AttnSmem::Q + g * 512, tm, g < kAttnTileQ / 4 ? bar_kvfull : c.bar_q1, xq, r[0], r[1], r[2],
                    r[3]);
    }
  } else if (lane == 0) {
    mbar_expect_tx(bar_kvfull, kAttnTxBlock);
  }
  int armed = 0;
  for (int j = 0; j < nkb; ++j) {
    const int b = j % kAttnKV;
    const int v0 = row_of(1 + j * kAttnBK + lane), v1 = row_of(1 + j * kAttnBK + 32 + lane);
    if (j > 0) {
      int ok = 1;
      if (lane == 0 && j >= kAttnKV) ok = mbar_wait(bar_kvempty + 8 * b, ((j / kAttnKV) - 1) & 1);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane == 0) mbar_expect_tx(bar_kvfull + 8 * b, kAttnTxBlock);
    }
#pragma unroll
    for (int g = 0; g < kAttnBK / 4; ++g) {
      int r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) r[i] = __shfl_sync(0xffffffffu, g < 8 ? v0 : v1, (4 * g + i) & 31);
      if (lane == 0) {
        tma_gather4(sb + AttnSmem::K + b * AttnSmem::KV_BYTES + g * 512, tm, bar_kvfull + 8 * b, xk, r[0], r[1], r[2],
                    r[3]);
        tma_gather4(sb + AttnSmem::V + b * AttnSmem::KV_BYTES + g * 512, tm, bar_kvfull + 8 * b, xv, r[0], r[1], r[2],
                    r[3]);
      }
    }
    armed = j + 1;
  }
  // no copy may still be landing when the CTA exits (matters only after a timeout)
  if (lane == 0) {
    for (int j = max(0, armed - kAttnKV); j < armed; ++j) mbar_wait(bar_kvfull + 8 * (j % kAttnKV), (j / kAttnKV) & 1);
    if (c.bar_q1) mbar_wait(c.bar_q1, 0);
  }
}

// ---------------------------------------------------------------------------
// window-query block (tcgen05)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void attn_window_block_tc(const CUtensorMap* tm, const AttnArgs& a, int qb, int h, int t,
                                                     uint8_t* smem) {
  const bf16* qkv = reinterpret_cast<const bf16*>(a.qkv);
  const int ld = 3 * a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_kvfull = sb + AttnSmem::BAR;        // kAttnKV, count 1 (producer's expect_tx) + TMA bytes
  const uint32_t bar_kvempty = bar_kvfull + 8 * kAttnKV; // kAttnKV, count 1 (commit after tile 1's P V)
  const uint32_t bar_sfull = bar_kvempty + 8 * kAttnKV;  // 2 (one per tile), count 1 (commit after Q K^T)
  const uint32_t bar_pfull = bar_sfull + 16;             // 2 (one per tile), count 4 (the tile's softmax warps)
  const uint32_t bar_ofinal = bar_pfull + 16;            // 2 (one per tile), count 1 (commit after its last P V)
  const uint32_t bar_q1 = bar_ofinal + 16;               // 1, count 1 (producer's expect_tx) + TMA bytes of tile 1's Q
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + AttnSmem::BAR + AttnSmem::NBAR * 8);
  float* sKg = reinterpret_cast<float*>(smem + AttnSmem::KG);
  float* sVg = sKg + 64;
  const int nkb = (a.Nw + kAttnBK - 1) / kAttnBK;
  const int q0 = 1 + qb * kAttnBQ;  // first slot of this query block (tile 0; tile 1 follows)

  uint32_t tmem = 0;
  if (warp == 8) {
    // ---------------- TMA producer ----------------
    // Its copies start as soon as the barriers exist; the other warps learn of
    // the initialisation through a named barrier that this warp only arrives at.
    if (lane == 0) {
      for (int i = 0; i < kAttnKV; ++i) {
        mbar_init(bar_kvfull + 8 * i, 1);
        mbar_init(bar_kvempty + 8 * i, 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar_sfull + 8 * i, 1);
        mbar_init(bar_pfull + 8 * i, 4);
      }
      for (int i = 0; i < 2; ++i) mbar_init(bar_ofinal + 8 * i, 1);
      mbar_init(bar_q1, 1);
      fence_barrier_init();
      tma_prefetch_desc(tm);
    }
    __syncwarp();
    asm volatile("bar.arrive 2, %0;" ::"n"(kAttnThreads) : "memory");
    pdl_wait();
    pdl_trigger();
    const AttnLoad c{tm, sb, bar_kvfull, bar_kvempty, bar_q1, q0, nkb, t, h, lane};
    if (a.load == 2)
      attn_load_grid(a, c);
    else if (a.load == 1)
      attn_load_runs(a, c);
    else
      attn_load_gather(a, c);
  } else {
    if (warp == 9) {
      tmem_alloc(smem_u32(tmem_slot), kAttnTmemCols);   // tile i: S / P at 128i .. 128i + 63, O at 128i + 64 ..
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
    asm volatile("bar.sync 2, %0;" ::"n"(kAttnThreads) : "memory");
    tc_fence_after();
    tmem = *tmem_slot;
    if (warp == 9) {
      // ---------------- MMA issuer ----------------
      // Per tile one S / P buffer: S of block j+1 goes into the columns that hold
      // P of block j and is issued after P V of block j (tcgen05.mma runs in issue
      // order), so the commit that announces S of block j+1 also means that O
      // holds the sum up to block j.  The two tiles alternate: P V and the next S
      // of tile 0, then of tile 1, whose P V commit also releases the K/V buffer.
      // The whole warp waits on the barriers (lane 0's outcome decides for all);
      // one elected lane issues the MMAs and commits.
      constexpr uint32_t IDESC_S = idesc_make(1u, kAttnBK);             // Q K^T: M 128, N 64
      constexpr uint32_t IDESC_O = idesc_make(1u, 64) | (1u << 16);     // P V: M 128, N 64, B MN-major
      const bool leader = elect_one();
      auto wait_all = [&](uint32_t bar, uint32_t parity) -> bool {
        return __shfl_sync(0xffffffffu, mbar_wait(bar, parity) ? 1 : 0, 0) != 0;
      };
      auto issue_s = [&](int i, int j) {   // S of tile i, block j (K block j is in shared memory)
        if (leader) {
          const int b = j % kAttnKV;
          const uint64_t dq = sdesc_sw128(sb + AttnSmem::Q + i * kAttnTileQ * 128);
          const uint64_t dk = sdesc_sw128(sb + AttnSmem::K + b * AttnSmem::KV_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) tc_mma_f16(tmem + i * kAttnTmemTile, dq + 2 * k, dk + 2 * k, IDESC_S, k != 0);
          tc_commit(bar_sfull + 8 * i);
        }
        __syncwarp();
      };
      auto issue_pv = [&](int i, int j) {  // O of tile i += P V of block j
        if (leader) {
          const int b = j % kAttnKV;
#pragma unroll
          for (int kk = 0; kk < kAttnBK / 16; ++kk) {
            const uint64_t dv = sdesc_sw128_mn(sb + AttnSmem::V + b * AttnSmem::KV_BYTES + kk * 2048);
            tc_mma_f16_tmem_a(tmem + i * kAttnTmemTile + 64, tmem + i * kAttnTmemTile + kk * 8, dv, IDESC_O,
                              (j | kk) != 0);
          }
          if (i == 1) tc_commit(bar_kvempty + 8 * b);
        }
        __syncwarp();
      };
      // Tile 1 starts one softmax block after tile 0 (its first S follows tile 0's
      // first P V), so that each tile's softmax runs while the other tile waits
      // for its P V and next S.
      bool ok = nkb > 0 && wait_all(bar_kvfull, 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
      }
      for (int j = 0; j < nkb && ok; ++j) {
        const bool more = j + 1 < nkb;
        if (!wait_all(bar_pfull, j & 1)) { ok = false; break; }
        tc_fence_after();
        issue_pv(0, j);
        if (!more && leader) tc_commit(bar_ofinal);
        if (j == 0) {
          if (!wait_all(bar_q1, 0)) { ok = false; break; }
          tc_fence_after();
          issue_s(1, 0);
        }
        if (more) {
          if (!wait_all(bar_kvfull + 8 * ((j + 1) % kAttnKV), ((j + 1) / kAttnKV) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (!wait_all(bar_pfull + 8, j & 1)) { ok = false; break; }
        tc_fence_after();
        issue_pv(1, j);
        if (more) issue_s(1, j + 1);
      }
      // single-phase barriers: waiters may arrive any number of phases early
      if (ok && leader) tc_commit(bar_ofinal + 8);
    } else {
      // ---------------- softmax: one query row per thread ----------------
      const int tile = warp >> 2;              // warps 0-3: tile 0, warps 4-7: tile 1
      const int row = tid & 127;               // TMEM lane = row of the tile
      const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const uint32_t tS = tmem + tile * kAttnTmemTile, tO = tS + 64;
      const uint32_t sfull = bar_sfull + 8 * tile, pfull = bar_pfull + 8 * tile;
      bool ok = mbar_wait(tile ? bar_q1 : bar_kvfull, 0);   // the tile's Q rows are in shared memory
      float m = -INFINITY, l = 0.f, gcoef = 0.f;
      if (ok) {
        // score of the global key seeds the running maximum and sum
        const uint8_t* qrow = smem + AttnSmem::Q + tile * kAttnTileQ * 128;
        float sg = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(qrow + swz(row, c)), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) sg = fmaf(f[e], sKg[c * 8 + e], sg);
        }
        m = sg * a.scale_log2;
        l = 1.f;
        gcoef = 1.f;
      }
      for (int j = 0; j < nkb && ok; ++j) {
        if (!mbar_wait(sfull, j & 1)) { ok = false; break; }
        tc_fence_after();
        float sv[kAttnBK];
        tmem_ld32(tS + lane_off, sv);
        tmem_ld32(tS + lane_off + 32, sv + 32);
        tmem_wait_ld();
        const int kbase = j * kAttnBK;
        // row maximum of the raw scores (the scale is positive); keys beyond the
        // window exist only in the last block
        if (kbase + kAttnBK > a.Nw) {
#pragma unroll
          for (int i = 0; i < kAttnBK; ++i)
            if (kbase + i >= a.Nw) sv[i] = -INFINITY;
        }
        // Block maximum first (eight independent partial maxima keep the chains
        // short).  The reference maximum m moves only when a score exceeds it by
        // more than 2^8 (lazy rescale: probabilities stay below 256 and O is rarely
        // touched); then the exponentials are taken once, against m.
        float mp[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          mp[q] = fmax3(sv[q], sv[8 + q], sv[16 + q]);
          mp[q] = fmax3(mp[q], sv[24 + q], sv[32 + q]);
          mp[q] = fmax3(mp[q], sv[40 + q], sv[48 + q]);
          mp[q] = fmaxf(mp[q], sv[56 + q]);
        }
        const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7])) * a.scale_log2;
        const bool grow = mx > m + kAttnRescale;
        const bool warp_grow = __any_sync(0xffffffffu, grow);
        float alpha = 1.f;
        if (grow) {
          alpha = ex2_approx(m - mx);
          l *= alpha;
          gcoef *= alpha;
          m = mx;
        }
        // Pairs of scores through packed f32x2 arithmetic: one FMA per pair forms the
        // exponents x = s * log2(e) / sqrt(hd) - m, four packed partial sums, P back
        // into the S columns as packed bf16 pairs (the A operand of P V).  In a full
        // block one pair in kAttnEmuEvery takes 2^x on the FMA pipe (exp2_fma2), the
        // others on the SFU; the SFU alone would bound the block at twice the tensor
        // time.  The last, partial block keeps every exponential on the SFU, whose
        // 2^-inf = 0 removes its padding keys exactly.
        const uint64_t sc2 = pack_f32x2(a.scale_log2, a.scale_log2);
        const uint64_t nm2 = pack_f32x2(-m, -m);
        uint64_t sp2[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pw[kAttnBK / 2];
        if (kbase + kAttnBK <= a.Nw) {
#pragma unroll
          for (int i = 0; i < kAttnBK; i += 2) {
            const uint64_t x2 = fma_f32x2(pack_f32x2(sv[i], sv[i + 1]), sc2, nm2);
            float e0, e1;
            if ((i >> 1) % kAttnEmuEvery == kAttnEmuEvery - 1) {
              exp2_fma2(x2, e0, e1);
            } else {
              e0 = ex2_approx(lo_f32(x2));
              e1 = ex2_approx(hi_f32(x2));
            }
            sp2[(i >> 1) & 3] = add_f32x2(sp2[(i >> 1) & 3], pack_f32x2(e0, e1));
            pw[i >> 1] = pack_bf16(e0, e1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < kAttnBK; i += 2) {
            const uint64_t x2 = fma_f32x2(pack_f32x2(sv[i], sv[i + 1]), sc2, nm2);
            const float e0 = ex2_approx(lo_f32(x2)), e1 = ex2_approx(hi_f32(x2));
            sp2[(i >> 1) & 3] = add_f32x2(sp2[(i >> 1) & 3], pack_f32x2(e0, e1));
            pw[i >> 1] = pack_bf16(e0, e1);
          }
        }
        const uint64_t s01 = add_f32x2(sp2[0], sp2[1]), s23 = add_f32x2(sp2[2], sp2[3]);
        const uint64_t s0123 = add_f32x2(s01, s23);
        l += lo_f32(s0123) + hi_f32(s0123);
        tmem_st16u(tS + lane_off, pw);
        tmem_st16u(tS + lane_off + 16, pw + 16);
        if (warp_grow && j >= 1) {
          // O holds the sum up to block j-1 (its P V ran before this block's S): rescale the row
#pragma unroll 1
          for (int hh = 0; hh < 4; ++hh) {
            float o[16];
            tmem_ld16(tO + lane_off + hh * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] *= alpha;
            tmem_st16(tO + lane_off + hh * 16, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull);
      }
      if (ok && mbar_wait(bar_ofinal + 8 * tile, 0)) {
        tc_fence_after();
        const int slot = q0 + tile * kAttnTileQ + row;
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kAttnTmemCols);
  }
}

// ---------------------------------------------------------------------------
// the global token's own query row (slot 0) of tile t, head h
// ---------------------------------------------------------------------------
// Warp 8 streams the K/V blocks into the four shared buffers exactly as for a
// window block (no Q); warps w and w + 4 (w < 4) take the blocks of buffer w, w + 4,
// ..., keys 0-31 and 32-63 of each: lane l scores one key against the query (in
// shared memory), the warp's online softmax moves by the maximum over its 32 keys,
// and lane l accumulates channels 2l, 2l + 1 of P V from the shared V rows.  The
// eight warps' states are merged in warp order.
__device__ __forceinline__ void attn_global_block(const CUtensorMap* tm, const AttnArgs& a, int h, int t,
                                                  uint8_t* smem) {
  const bf16* qkv = reinterpret_cast<const bf16*>(a.qkv);
  const size_t ld = static_cast<size_t>(3) * a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_kvfull = sb + AttnSmem::BAR;        // kAttnKV, count 1 (producer's expect_tx) + TMA bytes
  const uint32_t bar_kvempty = bar_kvfull + 8 * kAttnKV; // kAttnKV, count 2 (the two warps that read the block)
  float* sKg = reinterpret_cast<float*>(smem + AttnSmem::KG);
  float* sVg = sKg + 64;
  float* gbuf = reinterpret_cast<float*>(smem + AttnSmem::Q);   // 8 x 66 floats: the warps' states
  float* sQg = gbuf + 8 * 66 + 8;                                // 64 floats: the global query (16-byte aligned)
  const int nkb = (a.Nw + kAttnBK - 1) / kAttnBK;
  constexpr int kWarps = 8;
  if (warp == 8) {
    if (lane == 0) {
      for (int i = 0; i < kAttnKV; ++i) {
        mbar_init(bar_kvfull + 8 * i, 1);
        mbar_init(bar_kvempty + 8 * i, 2);
      }
      fence_barrier_init();
      tma_prefetch_desc(tm);
    }
    __syncwarp();
    asm volatile("bar.arrive 2, %0;" ::"n"(kAttnThreads) : "memory");
    pdl_wait();
    pdl_trigger();
    const AttnLoad c{tm, sb, bar_kvfull, bar_kvempty, 0u, 1, nkb, t, h, lane};
    if (a.load == 2)
      attn_load_grid(a, c);
    else if (a.load == 1)
      attn_load_runs(a, c);
    else
      attn_load_gather(a, c);
  } else {
    pdl_wait();
    pdl_trigger();
    const size_t grow = static_cast<size_t>(attn_row(a, t, 0)) * ld + h * 64;
    if (tid < 64) {
      sQg[tid] = __bfloat162float(qkv[grow + tid]);
      sKg[tid] = __bfloat162float(qkv[grow + a.d + tid]);
      sVg[tid] = __bfloat162float(qkv[grow + 2 * a.d + tid]);
    }
    asm volatile("bar.sync 2, %0;" ::"n"(kAttnThreads) : "memory");
    if (warp < kWarps) {
      float gm = -INFINITY, gl = 0.f, ga0 = 0.f, ga1 = 0.f;
      if (warp == 0) {   // the global key itself
        float sg = 0.f;
#pragma unroll
        for (int c = 0; c < 64; ++c) sg = fmaf(sQg[c], sKg[c], sg);
        gm = sg * a.scale_log2;
        gl = lane == 0 ? 1.f : 0.f;
        ga0 = sVg[2 * lane];
        ga1 = sVg[2 * lane + 1];
      }
      // warps w and w + 4 share the blocks of buffer w % 4, keys 0-31 and 32-63:
      // each waits on every phase of its buffer's barrier, in order
      const int half = warp >> 2, key = half * 32 + lane;
      for (int j = warp & 3; j < nkb; j += kAttnKV) {
        const int b = j % kAttnKV;
        if (!mbar_wait(bar_kvfull + 8 * b, (j / kAttnKV) & 1)) break;
        const uint8_t* kbuf = smem + AttnSmem::K + b * AttnSmem::KV_BYTES;
        const uint8_t* vbuf = smem + AttnSmem::V + b * AttnSmem::KV_BYTES;
        float s0 = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f0[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(kbuf + swz(key, c)), f0);
          const float4 qa = *reinterpret_cast<const float4*>(sQg + 8 * c);
          const float4 qb = *reinterpret_cast<const float4*>(sQg + 8 * c + 4);
          const float q8[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) s0 = fmaf(q8[e], f0[e], s0);
        }
        const int nvalid = min(kAttnBK, a.Nw - j * kAttnBK);
        const float x0 = key < nvalid ? s0 * a.scale_log2 : -INFINITY;
        const float bm = warp_max(x0);
        if (bm != -INFINITY) {           // the second half of a last, short block may hold no key
          const float mnew = fmaxf(gm, bm);
          const float al = ex2_approx(gm - mnew);
          const float p0 = ex2_approx(x0 - mnew);
          gl = fmaf(gl, al, p0);
          ga0 *= al;
          ga1 *= al;
#pragma unroll 8
          for (int k = 0; k < 32; ++k) {
            const float pk = __shfl_sync(0xffffffffu, p0, k);
            const uint32_t off = swz(half * 32 + k, lane >> 2) + (lane & 3) * 4;
            const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vbuf + off));
            ga0 = fmaf(pk, vv.x, ga0);
            ga1 = fmaf(pk, vv.y, ga1);
          }
          gm = mnew;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_kvempty + 8 * b);
      }
      gl = warp_sum(gl);
      if (lane == 0) {
        gbuf[warp * 66] = gm;
        gbuf[warp * 66 + 1] = gl;
      }
      gbuf[warp * 66 + 2 + 2 * lane] = ga0;
      gbuf[warp * 66 + 3 + 2 * lane] = ga1;
    }
  }
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, gbuf[w * 66]);
    float L = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = gbuf[w * 66] == -INFINITY ? 0.f : ex2_approx(gbuf[w * 66] - M);
      L = fmaf(f, gbuf[w * 66 + 1], L);
      o0 = fmaf(f, gbuf[w * 66 + 2 + 2 * lane], o0);
      o1 = fmaf(f, gbuf[w * 66 + 3 + 2 * lane], o1);
    }
    bf16* O = reinterpret_cast<bf16*>(a.O) + static_cast<size_t>(t) * a.N * a.d + h * 64 + 2 * lane;
    *reinterpret_cast<__nv_bfloat162*>(O) = __floats2bfloat162_rn(o0 / L, o1 / L);
  }
}

__global__ void __launch_bounds__(kAttnThreads, kAttnCtasPerSm)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // swizzled tiles need a 1024-byte aligned base: round up inside the launch's slack
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int h = a.head_major ? blockIdx.z : blockIdx.y, t = a.head_major ? blockIdx.y : blockIdx.z;
  if (static_cast<int>(blockIdx.x) == a.nqb)
    attn_global_block(&tm, a, h, t, smem);
  else
    attn_window_block_tc(&tm, a, blockIdx.x, h, t, smem);
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
