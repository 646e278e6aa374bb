// rowops.cuh -- memory-bound row kernels: LayerNorm, the w-bar blend / merge, the
// tile gather of the stack input, per-row e4m3 quantisation, and the fp32 path's
// QK-RMSNorm + RoPE.  One warp per row, 16-byte vector accesses, fp32 arithmetic.
#pragma once

#include "common.cuh"

namespace ts {

// ---------------------------------------------------------------------------
// element access: bf16 or fp32 rows, 16-byte vectors (8 bf16 / 4 fp32)
// ---------------------------------------------------------------------------
template <typename T>
struct Vec;
template <>
struct Vec<bf16> {
  static constexpr int E = 8;
  __device__ static void load(const bf16* p, float* f) { bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), f); }
  __device__ static void store(bf16* p, const float* f) { *reinterpret_cast<uint4*>(p) = f32_to_bf16x8(f); }
};
template <>
struct Vec<float> {
  static constexpr int E = 4;
  __device__ static void load(const float* p, float* f) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  __device__ static void store(float* p, const float* f) { *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]); }
};

// Write one row held by a warp (NV vectors of E elements per lane, lane-strided) in
// the output format: T (bf16 / fp32), or e4m3 bytes + per-row scale absmax / 448.
template <typename T, int NV, bool Q8>
__device__ __forceinline__ void store_row(const float (&v)[NV][Vec<T>::E], int lane, T* out, uint8_t* q8,
                                          float* qscale, size_t row, int d) {
  constexpr int E = Vec<T>::E;
  if (!Q8) {
#pragma unroll
    for (int i = 0; i < NV; ++i) Vec<T>::store(out + row * d + (i * 32 + lane) * E, v[i]);
  } else {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(v[i][e]));
    amax = warp_max(amax);
    const float s = amax > 0.f ? amax / 448.0f : 1.0f;
    const float inv = 1.0f / s;
    if (lane == 0) qscale[row] = s;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      uint16_t pk[E / 2];
#pragma unroll
      for (int e = 0; e < E; e += 2) pk[e / 2] = f32x2_to_e4m3x2(v[i][e] * inv, v[i][e + 1] * inv);
      uint8_t* dst = q8 + row * d + (i * 32 + lane) * E;
      if (E == 8)
        *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(pk);
      else
        *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(pk);
    }
  }
}

// ---------------------------------------------------------------------------
// LayerNorm (pre-LN block, [TileShare] Tab. S1 Norm1 / Norm2): population variance,
// two passes over the row held in registers.  NV = d / (32 * E) vectors per lane.
// With rms set it is RMSNorm (Tab. S6 "RMSNorm"): no centring and no bias.
// ---------------------------------------------------------------------------
// The first `row_blocks` blocks walk the rows grid-stride (one row per warp at a
// time, the warp's next row loaded before the current one is normalised, so two
// rows per warp are in flight); blocks past them (when rt.cs is set) fill the RoPE
// table that the next QKV GEMM reads.
template <typename T, int NV, bool Q8>
__global__ void __launch_bounds__(256) layernorm_kernel(const T* __restrict__ x, int rows, int d,
                                                        const float* __restrict__ g, const float* __restrict__ b,
                                                        float eps, int rms, T* __restrict__ y, uint8_t* __restrict__ q8,
                                                        float* __restrict__ qscale, const RopeTable rt,
                                                        unsigned row_blocks) {
  pdl_wait();
  pdl_trigger();
  constexpr int E = Vec<T>::E;
  const int lane = threadIdx.x & 31;
  if (blockIdx.x >= row_blocks) {
    rope_table_fill(rt, static_cast<int>((blockIdx.x - row_blocks) * blockDim.x + threadIdx.x));
    return;
  }
  const size_t step = static_cast<size_t>(row_blocks) * (blockDim.x >> 5);
  size_t row = static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  // the next row waits in registers as raw 16-byte vectors
  uint4 nx[NV];
  if (row < static_cast<size_t>(rows)) {
#pragma unroll
    for (int i = 0; i < NV; ++i) nx[i] = *reinterpret_cast<const uint4*>(x + row * d + (i * 32 + lane) * E);
  }
  for (; row < static_cast<size_t>(rows); row += step) {
    float v[NV][E];
#pragma unroll
    for (int i = 0; i < NV; ++i) Vec<T>::load(reinterpret_cast<const T*>(&nx[i]), v[i]);
    if (row + step < static_cast<size_t>(rows)) {
#pragma unroll
      for (int i = 0; i < NV; ++i) nx[i] = *reinterpret_cast<const uint4*>(x + (row + step) * d + (i * 32 + lane) * E);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int e = 0; e < E; ++e) s += v[i][e];
    const float mean = rms ? 0.f : warp_sum(s) / d;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float c = v[i][e] - mean;
        q = fmaf(c, c, q);
      }
    const float rstd = rsqrtf(warp_sum(q) / d + eps);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c0 = (i * 32 + lane) * E;
#pragma unroll
      for (int e = 0; e < E; e += 4) {   // gains and biases as 16-byte vectors
        const float4 gg = __ldg(reinterpret_cast<const float4*>(g + c0 + e));
        const float4 bb = rms ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldg(reinterpret_cast<const float4*>(b + c0 + e));
        v[i][e] = (v[i][e] - mean) * rstd * gg.x + bb.x;
        v[i][e + 1] = (v[i][e + 1] - mean) * rstd * gg.y + bb.y;
        v[i][e + 2] = (v[i][e + 2] - mean) * rstd * gg.z + bb.z;
        v[i][e + 3] = (v[i][e + 3] - mean) * rstd * gg.w + bb.w;
      }
    }
    store_row<T, NV, Q8>(v, lane, y, q8, qscale, row, d);
  }
}

// generic fallback: any d (one warp per row, scalar, two passes over global memory)
template <typename T>
__global__ void __launch_bounds__(256) layernorm_generic_kernel(const T* __restrict__ x, int rows, int d,
                                                                const float* __restrict__ g,
                                                                const float* __restrict__ b, float eps, int rms,
                                                                T* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const size_t row = static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= static_cast<size_t>(rows)) return;
  const T* xr = x + row * d;
  float s = 0.f;
  for (int c = lane; c < d; c += 32) s += static_cast<float>(xr[c]);
  const float mean = rms ? 0.f : warp_sum(s) / d;
  float q = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float t = static_cast<float>(xr[c]) - mean;
    q = fmaf(t, t, q);
  }
  const float rstd = rsqrtf(warp_sum(q) / d + eps);
  for (int c = lane; c < d; c += 32)
    y[row * d + c] = static_cast<T>((static_cast<float>(xr[c]) - mean) * rstd * g[c] + (rms ? 0.f : b[c]));
}

// ---------------------------------------------------------------------------
// Blend / merge ([TileShare] Fig. 2: overlap tokens' attention outputs blended with
// w-bar; Fig. 3b: per-tile states merged).  Row u < U: fp32 sum over the token's
// CSR entries in ascending tile order of wbar * P[ent]; row U + t*R + i: P[t*N + i].  One
// warp writes each output row once; no atomics, so the result is deterministic.
// ---------------------------------------------------------------------------
template <typename T, int NV, bool Q8>
__global__ void __launch_bounds__(256) merge_kernel(const T* __restrict__ P, int rows, int U, int N, int R, int d,
                                                    const int* __restrict__ tok_ptr, const int* __restrict__ tok_ent,
                                                    const float* __restrict__ wbar, T* __restrict__ A,
                                                    uint8_t* __restrict__ q8, float* __restrict__ qscale) {
  pdl_wait();
  pdl_trigger();
  constexpr int E = Vec<T>::E;
  const int lane = threadIdx.x & 31;
  const size_t row = static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= static_cast<size_t>(rows)) return;
  float v[NV][E];
  if (row < static_cast<size_t>(U)) {
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int e = 0; e < E; ++e) v[i][e] = 0.f;
    const int e0 = __ldg(tok_ptr + row), e1 = __ldg(tok_ptr + row + 1);
    for (int e = e0; e < e1; ++e) {
      const float w = __ldg(wbar + e);
      const T* src = P + static_cast<size_t>(__ldg(tok_ent + e)) * d;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        float f[E];
        Vec<T>::load(src + (i * 32 + lane) * E, f);
#pragma unroll
        for (int k = 0; k < E; ++k) v[i][k] = fmaf(w, f[k], v[i][k]);
      }
    }
  } else {
    const size_t reg = row - U;   // register i of tile t: row t*N + i of P
    const T* src = P + ((reg / R) * static_cast<size_t>(N) + reg % R) * d;
#pragma unroll
    for (int i = 0; i < NV; ++i) Vec<T>::load(src + (i * 32 + lane) * E, v[i]);
  }
  store_row<T, NV, Q8>(v, lane, A, q8, qscale, row, d);
}

// The same blend with the tile rows staged in shared memory: each warp owns two
// buffers of `cover` rows (cover = most tiles on one token) and keeps two output
// rows in flight; for each, the lanes read the token's entries (one per lane) and
// issue one bulk copy per entry, so loads in flight hold no registers.  Row
// U + t*R + i is the single entry t*N + i with weight 1.  Sums run in ascending entry order,
// as in merge_kernel.
constexpr int kMergeWarps = 4;
template <typename T, int NV, bool Q8>
__global__ void __launch_bounds__(kMergeWarps * 32) merge_bulk_kernel(
    const T* __restrict__ P, int rows, int U, int N, int R, int d, const int* __restrict__ tok_ptr,
    const int* __restrict__ tok_ent, const float* __restrict__ wbar, int cover, T* __restrict__ A,
    uint8_t* __restrict__ q8, float* __restrict__ qscale) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int E = Vec<T>::E;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const uint32_t rowbytes = static_cast<uint32_t>(d) * sizeof(T);
  uint8_t* wbuf = smem + static_cast<size_t>(wib) * 2 * cover * rowbytes;
  const uint32_t bar = smem_u32(smem + static_cast<size_t>(kMergeWarps) * 2 * cover * rowbytes) + 16 * wib;
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 8, 1);
    fence_barrier_init();
  }
  __syncwarp();
  pdl_wait();
  pdl_trigger();
  // Row metadata runs ahead of the copies so that no dependent L2 round trip sits on
  // a row's path: lane k holds the CSR row pointer and entry count of this warp's
  // row base + k (refreshed every 32 rows), and the entries and weights of a row are
  // loaded one row before its copies are issued.  A register row U + t*R + i is
  // encoded as pointer -1 - (t*R + i), one entry t*N + i of weight 1.
  const int stride = gridDim.x * kMergeWarps;
  const int r0 = blockIdx.x * kMergeWarps + wib;
  int my_e0 = 0, my_n = 0;
  auto load_ptrs = [&](int base) {
    const int r = r0 + (base + lane) * stride;
    my_e0 = 0;
    my_n = 0;
    if (r < rows) {
      if (r < U) {
        my_e0 = __ldg(tok_ptr + r);
        my_n = __ldg(tok_ptr + r + 1) - my_e0;
      } else {
        my_e0 = -1 - (r - U);
        my_n = 1;
      }
    }
  };
  // entries (lane k < n: entry k and its weight) of this warp's i-th row
  auto load_ents = [&](int i, int& ent, float& wl, int& n) {
    const int e0 = __shfl_sync(0xffffffffu, my_e0, i & 31);
    n = __shfl_sync(0xffffffffu, my_n, i & 31);
    ent = 0;
    wl = 0.f;
    if (lane < n) {
      if (e0 >= 0) {
        ent = __ldg(tok_ent + e0 + lane);
        wl = __ldg(wbar + e0 + lane);
      } else {
        const int reg = -1 - e0;
        ent = (reg / R) * N + reg % R;
        wl = 1.f;
      }
    }
  };
  // copies of a row's entries into buffer b
  auto issue = [&](int b, int n, int ent) {
    fence_proxy_async_smem();   // this warp's reads of the buffer precede the copies that overwrite it
    __syncwarp();
    if (lane == 0) mbar_expect_tx(bar + 8 * b, n * rowbytes);
    __syncwarp();
    if (lane < n)
      bulk_load(smem_u32(wbuf + (static_cast<size_t>(b) * cover + lane) * rowbytes), P + static_cast<size_t>(ent) * d,
                rowbytes, bar + 8 * b);
  };
  int row = r0;
  int nc = 0, nn = 0, entc = 0, entn = 0;
  float wc = 0.f, wn = 0.f;
  bool pending_next = false;
  int broke_at = -1;
  load_ptrs(0);
  if (row < rows) {
    load_ents(0, entc, wc, nc);
    issue(0, nc, entc);
  }
  if (row + stride < rows) load_ents(1, entn, wn, nn);
  for (int i = 0; row < rows; ++i, row += stride) {
    pending_next = row + stride < rows;
    if (pending_next) issue((i + 1) & 1, nn, entn);
    int n2 = 0, ent2 = 0;
    float w2 = 0.f;
    if (row + 2 * stride < rows) {
      if (((i + 2) & 31) == 0) load_ptrs(i + 2);
      load_ents(i + 2, ent2, w2, n2);
    }
    if (!mbar_wait(bar + 8 * (i & 1), (i >> 1) & 1)) {
      broke_at = i;
      break;
    }
    pending_next = false;
    const uint8_t* buf = wbuf + static_cast<size_t>(i & 1) * cover * rowbytes;
    float v[NV][E];
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
      for (int e = 0; e < E; ++e) v[k][e] = 0.f;
    for (int k = 0; k < nc; ++k) {
      const float w = __shfl_sync(0xffffffffu, wc, k);
      const T* src = reinterpret_cast<const T*>(buf + static_cast<size_t>(k) * rowbytes);
#pragma unroll
      for (int q = 0; q < NV; ++q) {
        float f[E];
        Vec<T>::load(src + (q * 32 + lane) * E, f);
#pragma unroll
        for (int e = 0; e < E; ++e) v[q][e] = fmaf(w, f[e], v[q][e]);
      }
    }
    store_row<T, NV, Q8>(v, lane, A, q8, qscale, row, d);
    nc = nn;
    wc = wn;
    nn = n2;
    entn = ent2;
    wn = w2;
  }
  // no copy may still be landing when the CTA exits (matters only after a timeout)
  if (broke_at >= 0) {
    mbar_wait(bar + 8 * (broke_at & 1), (broke_at >> 1) & 1);
    if (pending_next) mbar_wait(bar + 8 * ((broke_at + 1) & 1), ((broke_at + 1) >> 1) & 1);
  }
}

// generic fallback of the blend for any d (scalar)
template <typename T>
__global__ void __launch_bounds__(256) merge_generic_kernel(const T* __restrict__ P, int rows, int U, int N, int R, int d,
                                                            const int* __restrict__ tok_ptr,
                                                            const int* __restrict__ tok_ent,
                                                            const float* __restrict__ wbar, T* __restrict__ A) {
  const int lane = threadIdx.x & 31;
  const size_t row = static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= static_cast<size_t>(rows)) return;
  for (int c = lane; c < d; c += 32) {
    float acc = 0.f;
    if (row < static_cast<size_t>(U)) {
      for (int e = tok_ptr[row]; e < tok_ptr[row + 1]; ++e)
        acc = fmaf(wbar[e], static_cast<float>(P[static_cast<size_t>(tok_ent[e]) * d + c]), acc);
    } else {
      const size_t reg = row - U;
      acc = static_cast<float>(P[((reg / R) * static_cast<size_t>(N) + reg % R) * d + c]);
    }
    A[row * d + c] = static_cast<T>(acc);
  }
}

// ---------------------------------------------------------------------------
// Stack input: per-tile copies X[t*N + s] of grid tokens S0 and global tokens G0
// (row map of the shared layout: < U grid token, >= U global token).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint8_t* __restrict__ S0,
                                                          const uint8_t* __restrict__ G0,
                                                          const int* __restrict__ rowmap, int nrows, int U,
                                                          size_t row_bytes, uint8_t* __restrict__ X) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const size_t r = static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= static_cast<size_t>(nrows)) return;
  const int src = __ldg(rowmap + r);
  const uint8_t* s = src < U ? S0 + static_cast<size_t>(src) * row_bytes : G0 + static_cast<size_t>(src - U) * row_bytes;
  for (size_t c = lane * 16; c < row_bytes; c += 32 * 16)
    *reinterpret_cast<uint4*>(X + r * row_bytes + c) = *reinterpret_cast<const uint4*>(s + c);
}

// ---------------------------------------------------------------------------
// Partial sharing ([TileShare] Tab. 1 top): a per-token result R [U + T, d] of a
// shared operation is added to every tile's copy of the token, X[r] += R[rowmap[r]]
// for the T * N per-tile rows (a tile's registers take its register rows of R).  fp32 add, one
// warp per row, 16-byte vectors; every X row is written by one warp.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) scatter_add_rows_kernel(const T* __restrict__ R, const int* __restrict__ rowmap,
                                                               int nrows, int d, T* __restrict__ X) {
  pdl_wait();
  pdl_trigger();
  constexpr int E = Vec<T>::E;
  const int lane = threadIdx.x & 31;
  const size_t r = static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= static_cast<size_t>(nrows)) return;
  const T* src = R + static_cast<size_t>(__ldg(rowmap + r)) * d;
  T* dst = X + r * d;
  for (int c = lane * E; c < d; c += 32 * E) {
    float a[E], b[E];
    Vec<T>::load(dst + c, a);
    Vec<T>::load(src + c, b);
#pragma unroll
    for (int e = 0; e < E; ++e) a[e] += b[e];
    Vec<T>::store(dst + c, a);
  }
}

// ---------------------------------------------------------------------------
// Per-row e4m3 quantisation of a bf16 matrix: scale = absmax / 448 (1 if zero),
// q = e4m3(x / scale), nearest-even, saturating.  cols % 8 == 0.
// ---------------------------------------------------------------------------
// Each lane walks its 16-byte vectors eight at a time (eight loads in flight, so
// the pass is not bound by one load's latency); the second pass reads the row again
// (from L1 / L2) to quantise it.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const bf16* __restrict__ x, int rows, int cols,
                                                            uint8_t* __restrict__ q, float* __restrict__ scale) {
  pdl_wait();
  pdl_trigger();
  constexpr int U = 8;   // vectors in flight per lane
  const int lane = threadIdx.x & 31;
  const size_t row = static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= static_cast<size_t>(rows)) return;
  const bf16* xr = x + row * cols;
  float amax = 0.f;
  for (int c0 = lane * 8; c0 < cols; c0 += 256 * U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + u * 256 < cols) v[u] = *reinterpret_cast<const uint4*>(xr + c0 + u * 256);
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + u * 256 < cols) {
        float f[8];
        bf16x8_to_f32(v[u], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
      }
  }
  amax = warp_max(amax);
  const float s = amax > 0.f ? amax / 448.0f : 1.0f;
  const float inv = 1.0f / s;   // one division per row; x / s becomes x * (1 / s) (within an fp32 ulp)
  if (lane == 0) scale[row] = s;
  for (int c0 = lane * 8; c0 < cols; c0 += 256 * U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + u * 256 < cols) v[u] = *reinterpret_cast<const uint4*>(xr + c0 + u * 256);
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + u * 256 < cols) {
        float f[8];
        bf16x8_to_f32(v[u], f);
        uint16_t pk[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) pk[e / 2] = f32x2_to_e4m3x2(f[e] * inv, f[e + 1] * inv);
        *reinterpret_cast<uint2*>(q + row * cols + c0 + u * 256) = *reinterpret_cast<const uint2*>(pk);
      }
  }
}

// ---------------------------------------------------------------------------
// fp32 path: QK-RMSNorm (gain) then RoPE at the row's coordinates, in place on the
// q and k parts of qkv [rows, 3d].  One thread per (row, head, q|k).
// ---------------------------------------------------------------------------
struct RopeF32 {
  int dims[3];
  float th_hi[32];
  float th_lo[32];
};

__global__ void __launch_bounds__(128) qk_norm_rope_f32_kernel(float* __restrict__ qkv, int rows, int d, int heads,
                                                               const float* __restrict__ q_g,
                                                               const float* __restrict__ k_g, float eps,
                                                               const int4* __restrict__ pos, const RopeF32 rope) {
  const int hd = d / heads;
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<size_t>(rows) * heads * 2) return;
  const int part = static_cast<int>(idx % 2);
  const int h = static_cast<int>((idx / 2) % heads);
  const size_t row = idx / (2 * heads);
  float* v = qkv + row * 3 * d + part * d + h * hd;
  const float* g = part ? k_g : q_g;
  float x[64];
  float ss = 0.f;
  for (int c = 0; c < hd; ++c) {
    x[c] = v[c];
    ss = fmaf(x[c], x[c], ss);
  }
  const float r = rsqrtf(ss / hd + eps);
  for (int c = 0; c < hd; ++c) x[c] = x[c] * r * g[c];
  const int4 p4 = pos[row];
  const float p[3] = {static_cast<float>(p4.x), static_cast<float>(p4.y), static_cast<float>(p4.z)};
  int off = 0, pair = 0;
  for (int a = 0; a < 3; ++a) {
    const int half = rope.dims[a] / 2;
    for (int j = 0; j < half; ++j) {
      float c, s;
      rope_cos_sin(p[a], rope.th_hi[pair + j], rope.th_lo[pair + j], c, s);
      const float xa = x[off + j], xb = x[off + j + half];
      x[off + j] = xa * c - xb * s;
      x[off + j + half] = xa * s + xb * c;
    }
    off += rope.dims[a];
    pair += half;
  }
  for (int c = 0; c < hd; ++c) v[c] = x[c];
}

// ---------------------------------------------------------------------------
// fp32 path: SIMT GEMM Y = A W^T (+ b) with the same epilogues as the tensor-core
// kernel (bias, GELU, residual, SwiGLU).  64 x 64 tiles, K slices of 16, 4 x 4 per
// thread.  EPI 3 (SwiGLU): N is the output width, W has 2N rows (gate rows, then
// up rows); a tile loads 32 gate rows and the 32 matching up rows, so that lane l
// (tx < 8) and lane l + 8 of a warp hold the gate and up sums of the same outputs.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

template <int EPI>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, const float* __restrict__ W,
                                                       const float* __restrict__ bias, float* __restrict__ Y, int M,
                                                       int N, int K) {
  __shared__ float sA[16][64 + 4];
  __shared__ float sW[16][64 + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.x * 64, n0 = blockIdx.y * (EPI == 3 ? 32 : 64);
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i / 16, c = i % 16;
      const int gm = m0 + r, gk = k0 + c;
      int gn = n0 + r;
      bool wok = gn < N;
      if (EPI == 3) {
        gn = n0 + (r & 31);
        wok = gn < N;
        gn += (r >> 5) * N;     // rows 32..63 of the tile: the up rows
      }
      sA[c][r] = (gm < M && gk < K) ? A[static_cast<size_t>(gm) * K + gk] : 0.f;
      sW[c][r] = (wok && gk < K) ? W[static_cast<size_t>(gn) * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sA[kk][ty * 4 + i];
        w[i] = sW[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
  if (EPI == 3) {
    // lanes tx < 8 hold gate columns tx*4 + j, lanes tx + 8 the up columns
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float u = __shfl_down_sync(0xffffffffu, acc[i][j], 8);
        const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
        if (tx < 8 && m < M && n < N) {
          const float gv = acc[i][j] + (bias ? bias[n] : 0.f);
          const float uv = u + (bias ? bias[N + n] : 0.f);
          Y[static_cast<size_t>(m) * N + n] = silu_f(gv) * uv;
        }
      }
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j] + (bias ? bias[n] : 0.f);
      float* y = Y + static_cast<size_t>(m) * N + n;
      if (EPI == 1) v = gelu_erf(v);
      if (EPI == 2) v += *y;
      *y = v;
    }
  }
}

}  // namespace ts
