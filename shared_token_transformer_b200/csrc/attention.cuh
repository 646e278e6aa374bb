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
// bf16 kernel (hd = 64), 256 threads, 2 CTAs per SM.  Shared layer: grid
// (nqb, T, heads), the head slowest, so that CTAs in flight together work on one
// head of neighbouring tiles, whose overlapping q/k/v rows (one head's slice of
// the whole shared state: a few MB) then come from L2 instead of DRAM.  Per-tile
// layer (no rows shared between tiles): grid (nqb, heads, T), the tile slowest, so
// that the heads of one tile run together and each tile's q/k/v rows (all heads'
// column slices of the same rows) leave DRAM once.
//   blocks qb < nqb: 128 window queries, keys in blocks of 64.
//     warp 4     TMA producer of Q (once) and of K/V blocks into 128-byte-
//                swizzled shared rows: one box of a 3-D map over the grid per
//                block when a block is whole window rows of one frame, else one
//                2-D box per run of consecutive rows, else tile::gather4 loads
//                through the row map (four rows per instruction); four K/V
//                buffers, completion by transaction bytes on one mbarrier each;
//     warp 5     MMA issuer (one lane): S = Q K^T (tcgen05 kind::f16, M = 128,
//                N = 64) into one of three TMEM S buffers, then O += P V with P
//                read from TMEM (A operand) and V from shared memory as an
//                MN-major operand; S of block j+3 reuses the columns of P of
//                block j and is issued after P V of block j (tcgen05.mma runs
//                in issue order);
//     warps 0-3  softmax, one query row per thread (TMEM lane = row): one tcgen05
//                round trip brings the row's 64 scores into registers; online
//                softmax in the exp2 domain with a lazily moved reference maximum
//                (O rescaled in TMEM only when a score exceeds it by 2^8); P goes
//                back over the scores as packed bf16; the global key (slot 0)
//                seeds the running max and sum and is added back at the end with
//                its running coefficient;
//     warps 6-7  in query block 0 only: the global token's own query row (slot 0),
//                an online softmax over the K/V blocks in shared memory (each
//                warp every other block), merged at the end.
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
  int head_major;     // bf16 grid: 1 (nqb, T, heads), head slowest; 0 (nqb, heads, T), tile slowest
};

__device__ __forceinline__ int attn_row(const AttnArgs& a, int t, int s) {
  return a.rowmap ? __ldg(a.rowmap + t * a.N + s) : t * a.N + s;
}

// byte offset of 16-byte chunk `ch` of row `r` in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz(int r, int ch) { return r * 128 + ((ch ^ (r & 7)) << 4); }

constexpr int kAttnThreads = 256;        // 4 softmax, TMA producer, MMA issuer, 2 global-row warps
constexpr int kAttnBQ = 128;             // queries per CTA
constexpr int kAttnBK = 64;              // keys per block
constexpr int kAttnKV = 4;               // K/V buffers
constexpr int kAttnS = 3;                // S / P buffers in TMEM
constexpr float kAttnRescale = 8.0f;     // lazy rescale threshold (log2 units)
#ifndef TS_ATTN_EMU_EVERY
#define TS_ATTN_EMU_EVERY 4
#endif
constexpr int kAttnEmuEvery = TS_ATTN_EMU_EVERY;   // one score pair in this many: 2^x on the FMA pipe

struct AttnSmem {
  static constexpr int Q = 0;                 // 16 KB: 128 rows x 128 B
  static constexpr int K = 16384;                       // kAttnKV x 8 KB: 64 rows x 128 B
  static constexpr int V = K + kAttnKV * 8192;          // kAttnKV x 8 KB
  static constexpr int KG = V + kAttnKV * 8192;         // 64 floats k_g, 64 floats v_g
  static constexpr int GR = KG + 512;         // 2 x 66 floats: partial states of the global query row
  static constexpr int BAR = GR + 1024;       // barriers
  static constexpr int NBAR = 2 * kAttnKV + 2 * kAttnS + 3;
  static constexpr int BYTES = BAR + NBAR * 8 + 8;
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

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
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
  uint32_t sb, bar_kvfull, bar_kvempty;
  int q0, nkb, t, h, lane;
};

__device__ __forceinline__ void attn_load_grid(const AttnArgs& a, const AttnLoad& c) {
  const CUtensorMap* tm = c.tm;
  const uint32_t sb = c.sb, bar_kvfull = c.bar_kvfull, bar_kvempty = c.bar_kvempty;
  const int q0 = c.q0, nkb = c.nkb, t = c.t, h = c.h, lane = c.lane;
  // ---------------- TMA producer, one grid box per 64 slots ----------------
  // A block of 64 window slots is 64 / bx whole window rows of one frame: one
  // box of the 3-D map (channels, grid column, grid row) starting at the row
  // of its first slot.  Blocks past the tile's last slot load block 0 again.
  auto box_at = [&](int slot, int& x, int& y) {
    const int u = attn_row(a, t, slot < a.N ? slot : 1);
    x = u % a.gw;
    y = u / a.gw;
  };
  if (lane == 0) {
    const int xq = h * 64, xk = a.d + h * 64, xv = 2 * a.d + h * 64;
    int x, y;
    mbar_expect_tx(bar_kvfull, 2 * 16384);   // Q rows travel with K/V block 0
    box_at(q0, x, y);
    tma_load_3d(sb + AttnSmem::Q, tm, bar_kvfull, xq, x, y);
    box_at(q0 + 64, x, y);
    tma_load_3d(sb + AttnSmem::Q + 8192, tm, bar_kvfull, xq, x, y);
    int xn, yn;
    box_at(1, xn, yn);
    int armed = 0;
    for (int j = 0; j < nkb; ++j) {
      const int b = j % kAttnKV;
      const int xc = xn, yc = yn;
      if (j + 1 < nkb) box_at(1 + (j + 1) * kAttnBK, xn, yn);
      if (j > 0) {
        if (j >= kAttnKV && !mbar_wait(bar_kvempty + 8 * b, ((j / kAttnKV) - 1) & 1)) break;
        mbar_expect_tx(bar_kvfull + 8 * b, 16384);
      }
      tma_load_3d(sb + AttnSmem::K + b * 8192, tm, bar_kvfull + 8 * b, xk, xc, yc);
      tma_load_3d(sb + AttnSmem::V + b * 8192, tm, bar_kvfull + 8 * b, xv, xc, yc);
      armed = j + 1;
    }
    // no copy may still be landing when the CTA exits (matters only after a timeout)
    for (int j = max(0, armed - kAttnKV); j < armed; ++j) mbar_wait(bar_kvfull + 8 * (j % kAttnKV), (j / kAttnKV) & 1);
  }
}

__device__ __forceinline__ void attn_load_runs(const AttnArgs& a, const AttnLoad& c) {
  const CUtensorMap* tm = c.tm;
  const uint32_t sb = c.sb, bar_kvfull = c.bar_kvfull, bar_kvempty = c.bar_kvempty;
  const int q0 = c.q0, nkb = c.nkb, t = c.t, h = c.h, lane = c.lane;
  // ---------------- TMA producer, runs of consecutive rows ----------------
  // Each run of `run` slots is one tiled box (128 bytes x run rows) of the q/k/v
  // columns of head h.  Runs past the tile's last slot (padding of the last key
  // or query block) load the first run again: their scores are masked and their
  // outputs are not stored.  Lane i looks up the row of run i one block ahead;
  // lane 0 issues the copies.
  const int L = a.run, nrun = kAttnBK / L;
  auto run_row = [&](int slot) { return attn_row(a, t, slot < a.N ? slot : 1); };
  const int xq = h * 64, xk = a.d + h * 64, xv = 2 * a.d + h * 64;
  {
    const int rq = lane < kAttnBQ / L ? run_row(q0 + lane * L) : 0;
    if (lane == 0) mbar_expect_tx(bar_kvfull, 2 * 16384);   // Q rows travel with K/V block 0
    for (int i = 0; i < kAttnBQ / L; ++i) {
      const int r = __shfl_sync(0xffffffffu, rq, i);
      if (lane == 0) tma_load_2d(sb + AttnSmem::Q + i * L * 128, tm, bar_kvfull, xq, r);
    }
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
      if (lane == 0) mbar_expect_tx(bar_kvfull + 8 * b, 16384);
    }
    for (int i = 0; i < nrun; ++i) {
      const int r = __shfl_sync(0xffffffffu, rcur, i);
      if (lane == 0) {
        tma_load_2d(sb + AttnSmem::K + b * 8192 + i * L * 128, tm, bar_kvfull + 8 * b, xk, r);
        tma_load_2d(sb + AttnSmem::V + b * 8192 + i * L * 128, tm, bar_kvfull + 8 * b, xv, r);
      }
    }
    armed = j + 1;
  }
  // no copy may still be landing when the CTA exits (matters only after a timeout)
  if (lane == 0)
    for (int j = max(0, armed - kAttnKV); j < armed; ++j) mbar_wait(bar_kvfull + 8 * (j % kAttnKV), (j / kAttnKV) & 1);
}

__device__ __forceinline__ void attn_load_gather(const AttnArgs& a, const AttnLoad& c) {
  const CUtensorMap* tm = c.tm;
  const uint32_t sb = c.sb, bar_kvfull = c.bar_kvfull, bar_kvempty = c.bar_kvempty;
  const int q0 = c.q0, nkb = c.nkb, t = c.t, h = c.h, lane = c.lane;
  // ---------------- TMA producer, gathered rows ----------------
  // Rows are gathered four at a time (tile::gather4) from the q/k/v columns of
  // head h.  Slots past the tile's last one (padding of the last key or query
  // block) repeat the last slot's row, so every coordinate is in range; their
  // scores are masked and their outputs are not stored.
  auto row_of = [&](int slot) { return attn_row(a, t, min(slot, a.N - 1)); };
  const int xq = h * 64, xk = a.d + h * 64, xv = 2 * a.d + h * 64;
  int vq[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) vq[k] = row_of(q0 + 32 * k + lane);
  int v0 = row_of(1 + lane), v1 = row_of(33 + lane);
  if (lane == 0) mbar_expect_tx(bar_kvfull, 2 * 16384);   // Q rows travel with K/V block 0
#pragma unroll
  for (int g = 0; g < 32; ++g) {
    int r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = __shfl_sync(0xffffffffu, vq[g >> 3], (4 * g + i) & 31);
    if (lane == 0) tma_gather4(sb + AttnSmem::Q + g * 512, tm, bar_kvfull, xq, r[0], r[1], r[2], r[3]);
  }
  int armed = 0;
  for (int j = 0; j < nkb; ++j) {
    const int b = j % kAttnKV;
    if (j > 0) {
      v0 = row_of(1 + j * kAttnBK + lane);
      v1 = row_of(1 + j * kAttnBK + 32 + lane);
      int ok = 1;
      if (lane == 0 && j >= kAttnKV) ok = mbar_wait(bar_kvempty + 8 * b, ((j / kAttnKV) - 1) & 1);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane == 0) mbar_expect_tx(bar_kvfull + 8 * b, 16384);
    }
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      int r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) r[i] = __shfl_sync(0xffffffffu, g < 8 ? v0 : v1, (4 * g + i) & 31);
      if (lane == 0) {
        tma_gather4(sb + AttnSmem::K + b * 8192 + g * 512, tm, bar_kvfull + 8 * b, xk, r[0], r[1], r[2], r[3]);
        tma_gather4(sb + AttnSmem::V + b * 8192 + g * 512, tm, bar_kvfull + 8 * b, xv, r[0], r[1], r[2], r[3]);
      }
    }
    armed = j + 1;
  }
  // no copy may still be landing when the CTA exits (matters only after a timeout)
  if (lane == 0)
    for (int j = max(0, armed - kAttnKV); j < armed; ++j) mbar_wait(bar_kvfull + 8 * (j % kAttnKV), (j / kAttnKV) & 1);
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
  const uint32_t bar_kvempty = bar_kvfull + 8 * kAttnKV; // kAttnKV, count 1 (commit after P V) [+1 global-row warp]
  const uint32_t bar_sfull = bar_kvempty + 8 * kAttnKV;  // kAttnS, count 1 (commit after Q K^T)
  const uint32_t bar_pfull = bar_sfull + 8 * kAttnS;     // kAttnS, count 4 (softmax warps wrote P into TMEM)
  const uint32_t bar_odone = bar_pfull + 8 * kAttnS;     // 2, count 1 (commit after P V)
  const uint32_t bar_ofinal = bar_odone + 16;            // 1, count 1 (commit after the last P V)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + AttnSmem::BAR + AttnSmem::NBAR * 8);
  float* sKg = reinterpret_cast<float*>(smem + AttnSmem::KG);
  float* sVg = sKg + 64;
  const int nkb = (a.Nw + kAttnBK - 1) / kAttnBK;
  const int q0 = 1 + qb * kAttnBQ;  // first slot of this query block
  // The CTA of query block 0 also computes the global token's own query row
  // (slot 0) in warps 6 and 7, which then co-own the K/V buffers they read.
  const bool grow_row = qb == 0;

  uint32_t tmem = 0;
  if (warp == 4) {
    // ---------------- TMA producer ----------------
    // Its copies start as soon as the barriers exist; the other warps learn of
    // the initialisation through a named barrier that this warp only arrives at.
    if (warp == 4 && lane == 0) {
      for (int i = 0; i < kAttnKV; ++i) {
        mbar_init(bar_kvfull + 8 * i, 1);
        mbar_init(bar_kvempty + 8 * i, grow_row ? 2 : 1);
      }
      for (int i = 0; i < kAttnS; ++i) {
        mbar_init(bar_sfull + 8 * i, 1);
        mbar_init(bar_pfull + 8 * i, 4);
      }
      for (int i = 0; i < 2; ++i) mbar_init(bar_odone + 8 * i, 1);
      mbar_init(bar_ofinal, 1);
      fence_barrier_init();
      tma_prefetch_desc(tm);
    }
    __syncwarp();
    asm volatile("bar.arrive 2, %0;" ::"n"(kAttnThreads) : "memory");
    pdl_wait();
    pdl_trigger();
    const AttnLoad c{tm, sb, bar_kvfull, bar_kvempty, q0, nkb, t, h, lane};
    if (a.load == 2)
      attn_load_grid(a, c);
    else if (a.load == 1)
      attn_load_runs(a, c);
    else
      attn_load_gather(a, c);
  } else {
    if (warp == 5) {
      tmem_alloc(smem_u32(tmem_slot), 256);    // S / P buffer k: cols 64k .. 64k + 63 (k < 3), O: 192-255
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
    const uint32_t tO = tmem + 64 * kAttnS;
    if (warp == 5) {
      // ---------------- MMA issuer ----------------
      // S of block j+3 goes into the TMEM columns that hold P of block j; it is
      // issued after P V of block j, and tcgen05.mma runs in issue order.  The whole
      // warp waits on the barriers (lane 0's outcome decides for all); one elected
      // lane issues the MMAs and commits.
      constexpr uint32_t IDESC_S = idesc_make(1u, kAttnBK);             // Q K^T: M 128, N 64
      constexpr uint32_t IDESC_O = idesc_make(1u, 64) | (1u << 16);     // P V: M 128, N 64, B MN-major
      const uint64_t dq = sdesc_sw128(sb + AttnSmem::Q);
      const bool leader = elect_one();
      auto issue_s = [&](int j) -> bool {
        const int b = j % kAttnKV, sbuf = j % kAttnS;
        if (!__shfl_sync(0xffffffffu, mbar_wait(bar_kvfull + 8 * b, (j / kAttnKV) & 1) ? 1 : 0, 0)) return false;
        tc_fence_after();
        if (leader) {
          const uint64_t dk = sdesc_sw128(sb + AttnSmem::K + b * 8192);
#pragma unroll
          for (int k = 0; k < 4; ++k) tc_mma_f16(tmem + sbuf * 64, dq + 2 * k, dk + 2 * k, IDESC_S, k != 0);
          tc_commit(bar_sfull + 8 * sbuf);
        }
        __syncwarp();
        return true;
      };
      bool ok = true;
      for (int j = 0; j < kAttnS && j < nkb && ok; ++j) ok = issue_s(j);
      for (int j = 0; j < nkb && ok; ++j) {
        const int pb = j % kAttnS, b = j % kAttnKV;
        if (!__shfl_sync(0xffffffffu, mbar_wait(bar_pfull + 8 * pb, (j / kAttnS) & 1) ? 1 : 0, 0)) { ok = false; break; }
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t dv = sdesc_sw128_mn(sb + AttnSmem::V + b * 8192 + kk * 2048);
            tc_mma_f16_tmem_a(tO, tmem + pb * 64 + kk * 8, dv, IDESC_O, (j | kk) != 0);
          }
          tc_commit(bar_odone + 8 * (j & 1));
          tc_commit(bar_kvempty + 8 * b);
        }
        __syncwarp();
        if (j + kAttnS < nkb) ok = issue_s(j + kAttnS);
      }
      // single-phase barrier: waiters may arrive any number of phases early
      if (ok && leader) tc_commit(bar_ofinal);
    } else if (warp >= 6) {
      // ---------------- global token's query row (query block 0 only) ----------------
      // Warp 6 + g takes blocks g, g + 2, ...: lane l scores keys l and l + 32 with
      // the full query in registers, then accumulates channels 2l, 2l + 1 of P V.
      // The two warps' online-softmax states are merged at the end.
      if (grow_row) {
        const int g = warp - 6;
        float qf[64];
        {
          const uint4* qr = reinterpret_cast<const uint4*>(qkv + static_cast<size_t>(attn_row(a, t, 0)) * ld + h * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c) bf16x8_to_f32(qr[c], qf + 8 * c);
        }
        float gm = -INFINITY, gl = 0.f, ga0 = 0.f, ga1 = 0.f;
        if (g == 0) {   // the global key itself
          float sg = 0.f;
#pragma unroll
          for (int c = 0; c < 64; ++c) sg = fmaf(qf[c], sKg[c], sg);
          gm = sg * a.scale_log2;
          gl = lane == 0 ? 1.f : 0.f;
          ga0 = sVg[2 * lane];
          ga1 = sVg[2 * lane + 1];
        }
        for (int j = g; j < nkb; j += 2) {
          const int b = j % kAttnKV;
          if (!mbar_wait(bar_kvfull + 8 * b, (j / kAttnKV) & 1)) break;
          const uint8_t* kbuf = smem + AttnSmem::K + b * 8192;
          const uint8_t* vbuf = smem + AttnSmem::V + b * 8192;
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float f0[8], f1[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(kbuf + swz(lane, c)), f0);
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(kbuf + swz(lane + 32, c)), f1);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              s0 = fmaf(qf[8 * c + e], f0[e], s0);
              s1 = fmaf(qf[8 * c + e], f1[e], s1);
            }
          }
          const int nvalid = min(kAttnBK, a.Nw - j * kAttnBK);
          const float x0 = lane < nvalid ? s0 * a.scale_log2 : -INFINITY;
          const float x1 = lane + 32 < nvalid ? s1 * a.scale_log2 : -INFINITY;
          const float mnew = fmaxf(gm, warp_max(fmaxf(x0, x1)));
          const float al = ex2_approx(gm - mnew);
          const float p0 = ex2_approx(x0 - mnew), p1 = ex2_approx(x1 - mnew);
          gl = fmaf(gl, al, p0 + p1);
          ga0 *= al;
          ga1 *= al;
#pragma unroll 8
          for (int k = 0; k < kAttnBK; ++k) {
            const float pk = __shfl_sync(0xffffffffu, k < 32 ? p0 : p1, k & 31);
            const uint32_t off = swz(k, lane >> 2) + (lane & 3) * 4;
            const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vbuf + off));
            ga0 = fmaf(pk, vv.x, ga0);
            ga1 = fmaf(pk, vv.y, ga1);
          }
          gm = mnew;
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_kvempty + 8 * b);
        }
        gl = warp_sum(gl);
        float* gbuf = reinterpret_cast<float*>(smem + AttnSmem::GR);
        if (lane == 0) {
          gbuf[g * 66] = gm;
          gbuf[g * 66 + 1] = gl;
        }
        gbuf[g * 66 + 2 + 2 * lane] = ga0;
        gbuf[g * 66 + 3 + 2 * lane] = ga1;
        asm volatile("bar.sync 1, 64;" ::: "memory");
        if (g == 0) {
          const float M = fmaxf(gbuf[0], gbuf[66]);
          float L = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const float f = gbuf[w * 66] == -INFINITY ? 0.f : ex2_approx(gbuf[w * 66] - M);
            L += f * gbuf[w * 66 + 1];
            o0 += f * gbuf[w * 66 + 2 + 2 * lane];
            o1 += f * gbuf[w * 66 + 3 + 2 * lane];
          }
          bf16* O = reinterpret_cast<bf16*>(a.O) + static_cast<size_t>(t) * a.N * a.d + h * 64 + 2 * lane;
          *reinterpret_cast<__nv_bfloat162*>(O) = __floats2bfloat162_rn(o0 / L, o1 / L);
        }
      }
    } else if (warp < 4) {
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
        const int sbuf = j % kAttnS;
        if (!mbar_wait(bar_sfull + 8 * sbuf, (j / kAttnS) & 1)) { ok = false; break; }
        tc_fence_after();
        float sv[kAttnBK];
        tmem_ld32(tmem + sbuf * 64 + lane_off, sv);
        tmem_ld32(tmem + sbuf * 64 + lane_off + 32, sv + 32);
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
        tmem_st32u(tmem + sbuf * 64 + lane_off, pw);
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
        }
        tmem_wait_st();
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {          // swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) set_status(kStatusDeviceCheck);
    return;
  }
  const int h = a.head_major ? blockIdx.z : blockIdx.y, t = a.head_major ? blockIdx.y : blockIdx.z;
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
