// attention.cuh -- per-tile dense attention over gathered rows.
//
// [TileShare] Tab. S1 "Attention (dense, per tile)" and Fig. 2: for tile t and head h
// the keys, values and queries are the rows [global token of t, window slots of t];
// O = softmax(q k^T / sqrt(hd)) v with no mask.  In a shared layer the rows come
// from the shared q/k/v through the tile's index map (the "gather"); in a per-tile
// layer they are the tile's own contiguous rows.  q and k arrive already rotated
// (RoPE runs once per row in the QKV epilogue), so this kernel is a plain
// gathered attention.
//
// bf16 kernel (hd = 64), grid (nqb + 1, heads, T), 128 threads:
//   blocks qb < nqb: 64 window queries (4 warps x 16 rows), keys streamed in blocks
//     of 64 window slots through a double-buffered cp.async gather into 128-byte
//     swizzled shared rows; S = Q K^T and O += P V with mma.sync m16n8k16 (bf16 in,
//     fp32 accumulate), online softmax in registers (exp2 domain).  The global key
//     (slot 0) seeds the running max / sum / output before the window keys.
//   block qb == nqb: the global token's own query row (one row attends to N keys),
//     as a split-key reduction over the 128 threads.
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

constexpr int kAttnBQ = 64;
constexpr int kAttnBK = 64;

// window-query block: rows slot = 1 + qb*64 + i
__device__ __forceinline__ void attn_window_block(const AttnArgs& a, int qb, int h, int t, uint8_t* smem) {
  const bf16* qkv = reinterpret_cast<const bf16*>(a.qkv);
  const int ld = 3 * a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;

  uint8_t* sQ = smem;                       // 64 x 128 B
  uint8_t* sK = smem + 8192;                // 2 x 64 x 128 B
  uint8_t* sV = smem + 8192 + 16384;        // 2 x 64 x 128 B
  float* sKg = reinterpret_cast<float*>(smem + 8192 + 32768);   // 64 floats
  float* sVg = sKg + 64;                                        // 64 floats
  const uint32_t uQ = smem_u32(sQ), uK = smem_u32(sK), uV = smem_u32(sV);

  const int q0 = 1 + qb * kAttnBQ;
  // Q gather: 64 rows x 8 chunks, 4 chunks per thread
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid + i * 128;
    const int r = idx >> 3, ch = idx & 7;
    const int slot = q0 + r;
    const bool ok = slot < a.N;
    const bf16* src = qkv + (ok ? static_cast<size_t>(attn_row(a, t, slot)) * ld + h * 64 + ch * 8 : 0);
    cp_async16(uQ + swz(r, ch), src, ok);
  }
  const int nkb = (a.Nw + kAttnBK - 1) / kAttnBK;
  auto load_kv = [&](int kb, int buf) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + i * 128;
      const int r = idx >> 3, ch = idx & 7;
      const int slot = 1 + kb * kAttnBK + r;
      const bool ok = slot < a.N;
      const size_t base = ok ? static_cast<size_t>(attn_row(a, t, slot)) * ld + h * 64 + ch * 8 : 0;
      cp_async16(uK + buf * 8192 + swz(r, ch), qkv + base + (ok ? a.d : 0), ok);
      cp_async16(uV + buf * 8192 + swz(r, ch), qkv + base + (ok ? 2 * a.d : 0), ok);
    }
  };
  load_kv(0, 0);
  cp_async_commit();
  // global key / value (slot 0) as floats
  if (tid < 64) {
    const size_t grow = static_cast<size_t>(attn_row(a, t, 0)) * ld + h * 64 + tid;
    sKg[tid] = __bfloat162float(qkv[grow + a.d]);
    sVg[tid] = __bfloat162float(qkv[grow + 2 * a.d]);
  }

  uint32_t qf[4][4];
  float m_r[2], l_r[2], acc[8][4];

  for (int kb = 0; kb < nkb; ++kb) {
    if (kb + 1 < nkb) load_kv(kb + 1, (kb + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (kb == 0) {
      // Q fragments of this warp's 16 rows
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int r = warp * 16 + (lane & 15);
        const int ch = kk * 2 + (lane >> 4);
        ldmatrix_x4(uQ + swz(r, ch), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
      // seed the online softmax with the global key
      float sg[2] = {0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {       // a0/a2 -> row g, a1/a3 -> row g+8
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {           // columns +0 / +8
            const uint32_t w = qf[kk][half + 2 * hi];
            const __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(&w);
            const int c = kk * 16 + hi * 8 + 2 * tq;
            sg[half] += __bfloat162float(p.x) * sKg[c] + __bfloat162float(p.y) * sKg[c + 1];
          }
        }
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        sg[half] += __shfl_xor_sync(0xffffffffu, sg[half], 1);
        sg[half] += __shfl_xor_sync(0xffffffffu, sg[half], 2);
        m_r[half] = sg[half] * a.scale_log2;
        l_r[half] = (tq == 0) ? 1.f : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = j * 8 + 2 * tq;
        acc[j][0] = sVg[c];
        acc[j][1] = sVg[c + 1];
        acc[j][2] = sVg[c];
        acc[j][3] = sVg[c + 1];
      }
    }
    const uint32_t bK = uK + (kb & 1) * 8192, bV = uV + (kb & 1) * 8192;
    // S = Q K^T over 64 keys (8 n8 tiles)
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        uint32_t b0, b1, b2, b3;
        const int key = j * 8 + ((lane >> 4) << 3) + (lane & 7);
        const int ch = kk * 2 + ((lane >> 3) & 1);
        ldmatrix_x4(bK + swz(key, ch), b0, b1, b2, b3);
        mma_bf16_16816(s[j], qf[kk], b0, b1);
        mma_bf16_16816(s[j + 1], qf[kk], b2, b3);
      }
    }
    // mask keys beyond the window, then online softmax (two rows per thread)
    const int kbase = kb * kAttnBK;
    float mx[2] = {m_r[0], m_r[1]};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kbase + j * 8 + 2 * tq + (e & 1);
        s[j][e] = (key < a.Nw) ? s[j][e] * a.scale_log2 : -INFINITY;
        mx[e >> 1] = fmaxf(mx[e >> 1], s[j][e]);
      }
    }
    float alpha[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      mx[half] = fmaxf(mx[half], __shfl_xor_sync(0xffffffffu, mx[half], 1));
      mx[half] = fmaxf(mx[half], __shfl_xor_sync(0xffffffffu, mx[half], 2));
      alpha[half] = exp2f(m_r[half] - mx[half]);
      m_r[half] = mx[half];
      l_r[half] *= alpha[half];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[j][e] - m_r[e >> 1]);
        s[j][e] = p;
        l_r[e >> 1] += p;
        acc[j][e] *= alpha[e >> 1];
      }
    }
    // O += P V over 4 chunks of 16 keys
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kc][0], s[2 * kc][1]);
      pa[1] = pack_bf16(s[2 * kc][2], s[2 * kc][3]);
      pa[2] = pack_bf16(s[2 * kc + 1][0], s[2 * kc + 1][1]);
      pa[3] = pack_bf16(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
      for (int n = 0; n < 8; n += 2) {
        uint32_t b0, b1, b2, b3;
        const int mi = lane >> 3;
        const int key = kc * 16 + ((mi & 1) << 3) + (lane & 7);
        const int ch = n + (mi >> 1);
        ldmatrix_x4_trans(bV + swz(key, ch), b0, b1, b2, b3);
        mma_bf16_16816(acc[n], pa, b0, b1);
        mma_bf16_16816(acc[n + 1], pa, b2, b3);
      }
    }
    __syncthreads();
  }
  // normalise and store
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    l_r[half] += __shfl_xor_sync(0xffffffffu, l_r[half], 1);
    l_r[half] += __shfl_xor_sync(0xffffffffu, l_r[half], 2);
  }
  bf16* O = reinterpret_cast<bf16*>(a.O);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int slot = q0 + warp * 16 + g + half * 8;
    if (slot < a.N) {
      const float inv = 1.f / l_r[half];
      bf16* dst = O + (static_cast<size_t>(t) * a.N + slot) * a.d + h * 64;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        *reinterpret_cast<uint32_t*>(dst + j * 8 + 2 * tq) =
            pack_bf16(acc[j][2 * half] * inv, acc[j][2 * half + 1] * inv);
      }
    }
  }
}

// the global token's query (slot 0): 128 threads split the N keys
__device__ __forceinline__ void attn_global_row(const AttnArgs& a, int h, int t, uint8_t* smem) {
  const bf16* qkv = reinterpret_cast<const bf16*>(a.qkv);
  const int ld = 3 * a.d;
  const int tid = threadIdx.x;
  float* sq = reinterpret_cast<float*>(smem);            // 64
  float* sm = sq + 64;                                   // 128 maxima
  float* sl = sm + 128;                                  // 128 sums
  float* sacc = sl + 128;                                // 128 x 65
  if (tid < 64) sq[tid] = __bfloat162float(qkv[static_cast<size_t>(attn_row(a, t, 0)) * ld + h * 64 + tid]);
  __syncthreads();
  float m = -INFINITY, l = 0.f, acc[64];
#pragma unroll
  for (int c = 0; c < 64; ++c) acc[c] = 0.f;
  for (int s = tid; s < a.N; s += 128) {
    const bf16* kr = qkv + static_cast<size_t>(attn_row(a, t, s)) * ld + a.d + h * 64;
    float dot = 0.f;
#pragma unroll
    for (int c = 0; c < 64; c += 8) {
      float f[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(kr + c), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(f[e], sq[c + e], dot);
    }
    const float sc = dot * a.scale_log2;
    const float mn = fmaxf(m, sc);
    const float al = exp2f(m - mn), p = exp2f(sc - mn);
    l = l * al + p;
    const bf16* vr = kr + a.d;
#pragma unroll
    for (int c = 0; c < 64; c += 8) {
      float f[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(vr + c), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[c + e] = acc[c + e] * al + p * f[e];
    }
    m = mn;
  }
  sm[tid] = m;
  __syncthreads();
  float M = -INFINITY;
  for (int i = 0; i < 128; ++i) M = fmaxf(M, sm[i]);
  const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
  sl[tid] = l * f;
#pragma unroll
  for (int c = 0; c < 64; ++c) sacc[tid * 65 + c] = acc[c] * f;
  __syncthreads();
  if (tid < 64) {
    float L = 0.f, o = 0.f;
    for (int i = 0; i < 128; ++i) {
      L += sl[i];
      o += sacc[i * 65 + tid];
    }
    bf16* O = reinterpret_cast<bf16*>(a.O);
    O[static_cast<size_t>(t) * a.N * a.d + h * 64 + tid] = __float2bfloat16(o / L);
  }
}

__global__ void __launch_bounds__(128) attn_bf16_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int nqb = gridDim.x - 1;
  const int qb = blockIdx.x, h = blockIdx.y, t = blockIdx.z;
  if (qb < nqb)
    attn_window_block(a, qb, h, t, smem);
  else
    attn_global_row(a, h, t, smem);
}

constexpr int kAttnBf16Smem = 8192 + 32768 + 512;                 // window block
constexpr int kAttnBf16SmemGlobal = (64 + 128 + 128 + 128 * 65) * 4;  // global row
constexpr int kAttnBf16SmemMax = kAttnBf16SmemGlobal > kAttnBf16Smem ? kAttnBf16SmemGlobal : kAttnBf16Smem;

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
