// tileshare.cu -- libtileshare.so: the C ABI declared in include/tileshare.h and
// include/tileshare_ops.h, the host-side launchers and the layer orchestration.
//
// One translation unit: the kernels live in the included .cuh files.
//
// [TileShare] = "TileShare: Training-Free Acceleration of Overlapping Tiled ViT
// Decoding" (arXiv 2610.32233).  Data flow of one shared layer (Fig. 2, Tab. S1):
//   S --LN1--> xn --QKV GEMM + QK-RMSNorm + RoPE--> qkv --gathered attention--> O
//     --w-bar blend--> A --out-proj GEMM (+= S)--> S --LN2--> xn --up GEMM + GELU--> h
//     --down GEMM (+= S)--> S
// A per-tile layer is the same on X [T*N, d] with contiguous rows and no blend.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "../../include/tileshare.h"
#include "../../include/tileshare_ops.h"
#include "attention.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "plan.inl"
#include "rowops.cuh"

using ts::bf16;

// ============================================================================
// errors
// ============================================================================
static thread_local std::string g_last_error;

static ts_status fail(ts_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
static ts_status fail(ts_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define TS_CUDA_CHECK(expr)                                                                        \
  do {                                                                                             \
    cudaError_t e_ = (expr);                                                                       \
    if (e_ != cudaSuccess) return fail(TS_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_));       \
  } while (0)

#define TS_TRY(expr)               \
  do {                             \
    ts_status s_ = (expr);         \
    if (s_ != TS_OK) return s_;    \
  } while (0)

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static ts_status launched(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TS_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return TS_OK;
}

// ============================================================================
// kernel trace and launch counter
//   Each launcher calls trace_pre(stream) right before its kernel launch and
//   trace_post(stream, what) right after; the caller describes the launch's
//   algorithmic work in g_work (kernel class, FLOPs, HBM bytes).
// ============================================================================
struct Work {
  const char* name;
  double flops;
  double bytes;
};
static thread_local Work g_work = {"kernel", 0.0, 0.0};
static thread_local int g_slot = -1;
static std::atomic<long long> g_launches{0};

struct TraceRec {
  int cls, slot;
  double flops, bytes;
};
static struct {
  bool on = false;
  int cap = 0, used = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<std::string> names;
  std::vector<long long> count;
  std::vector<TraceRec> recs;
} g_trace;

static void set_work(const char* name, double flops, double bytes) { g_work = {name, flops, bytes}; }

static void trace_pre(cudaStream_t st) {
  g_slot = -1;
  if (g_trace.on && g_trace.used < g_trace.cap) {
    g_slot = g_trace.used++;
    cudaEventRecord(g_trace.ev[2 * g_slot], st);
  }
}

static ts_status trace_post(cudaStream_t st, const char* what) {
  ++g_launches;
  TS_TRY(launched(what));
  if (g_trace.on) {
    int cls = -1;
    for (size_t i = 0; i < g_trace.names.size(); ++i)
      if (g_trace.names[i] == g_work.name) cls = static_cast<int>(i);
    if (cls < 0) {
      cls = static_cast<int>(g_trace.names.size());
      g_trace.names.push_back(g_work.name);
      g_trace.count.push_back(0);
    }
    g_trace.count[cls]++;
    if (g_slot >= 0) {
      cudaEventRecord(g_trace.ev[2 * g_slot + 1], st);
      g_trace.recs.push_back({cls, g_slot, g_work.flops, g_work.bytes});
    }
  }
  g_slot = -1;
  return TS_OK;
}

// ============================================================================
// tensor maps (driver entry point fetched through the runtime, no -lcuda)
// ============================================================================
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static ts_status encode_fn(EncodeTiledFn* out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
      return fail(TS_ERR_CUDA, "cuTensorMapEncodeTiled not available");
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  *out = fn;
  return TS_OK;
}

// 2-D K-major operand [rows, K] (element size esz), box of 128 bytes x box_rows,
// 128-byte swizzle, out-of-bounds rows read as zero.
static ts_status make_tmap(CUtensorMap* map, const void* base, int rows, int K, int esz, int box_rows) {
  EncodeTiledFn enc;
  TS_TRY(encode_fn(&enc));
  const CUtensorMapDataType dt = esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * esz};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return TS_OK;
}

// 3-D bf16 map over the grid rows of a [F*H*W, cols] matrix: (column, grid x,
// grid row f*H + y), box of 128 bytes x bx x by, 128-byte swizzle.
static ts_status make_tmap_grid(CUtensorMap* map, const void* base, int cols, int W, int R, int bx, int by) {
  EncodeTiledFn enc;
  TS_TRY(encode_fn(&enc));
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(R)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, static_cast<cuuint64_t>(cols) * 2 * W};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(bx), static_cast<cuuint32_t>(by)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TS_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", static_cast<int>(r));
  return TS_OK;
}

// ============================================================================
// launches with programmatic dependent launch (PDL)
//   Kernels launched this way call pdl_wait() before touching activations, so
//   their prologue (barrier init, TMEM allocation, descriptor prefetch) overlaps
//   the tail of the previous kernel in the stream.
// ============================================================================
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // one shared-memory carve-out for every hot kernel, so that consecutive kernels
  // never wait for the SM to re-partition L1 and shared memory
  static thread_local const void* seen[64];
  static thread_local int nseen = 0;
  const void* key = reinterpret_cast<const void*>(kern);
  bool known = false;
  for (int i = 0; i < nseen; ++i) known |= seen[i] == key;
  if (!known) {
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (nseen < 64) seen[nseen++] = key;
  }
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The same launch as clusters of two CTAs (two-SM MMA pairs); grid.x is even.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl_pair(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                   Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ============================================================================
// model checks and RoPE tables
// ============================================================================
static int esize(ts_dtype dt) { return dt == TS_F32 ? 4 : 2; }

static ts_status check_model(const ts_model_desc* m) {
  if (!m) return fail(TS_ERR_INVALID_ARG, "model is NULL");
  if (m->d <= 0 || m->heads <= 0 || m->mlp <= 0 || m->d % m->heads)
    return fail(TS_ERR_INVALID_ARG, "bad model sizes d=%d heads=%d mlp=%d", m->d, m->heads, m->mlp);
  if (m->dtype != TS_F32 && m->dtype != TS_BF16 && m->dtype != TS_FP8_E4M3)
    return fail(TS_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(m->dtype));
  const int hd = m->d / m->heads;
  int sum = 0;
  for (int a = 0; a < 3; ++a) {
    if (m->rope_dims[a] < 0 || (m->rope_dims[a] & 1)) return fail(TS_ERR_INVALID_ARG, "rope_dims must be even and >= 0");
    sum += m->rope_dims[a];
  }
  if (sum != hd) return fail(TS_ERR_INVALID_ARG, "rope_dims sum %d != head dim %d", sum, hd);
  if (m->block != TS_BLOCK_LN_GELU && m->block != TS_BLOCK_RMS_SWIGLU)
    return fail(TS_ERR_INVALID_ARG, "unknown block flavour %d", static_cast<int>(m->block));
  if (!(m->eps_ln > 0.f) || !(m->eps_qk > 0.f) || !(m->rope_base > 0.f))
    return fail(TS_ERR_INVALID_ARG, "eps and rope_base must be positive");
  if (m->dtype == TS_F32) {
    if (hd != 16 && hd != 32 && hd != 64) return fail(TS_ERR_UNSUPPORTED, "fp32 path supports head dim 16, 32, 64");
    if (m->d % 4 || m->mlp % 4) return fail(TS_ERR_UNSUPPORTED, "fp32 path needs d, mlp multiples of 4");
  } else {
    if (hd != 64) return fail(TS_ERR_UNSUPPORTED, "bf16/e4m3 path supports head dim 64 only");
    if (m->d % 256 || m->d > 2048) return fail(TS_ERR_UNSUPPORTED, "bf16/e4m3 path needs d %% 256 == 0, d <= 2048");
    if (m->mlp % 256) return fail(TS_ERR_UNSUPPORTED, "bf16/e4m3 path needs mlp %% 256 == 0");
    const int* r = m->rope_dims;
    const bool s2 = r[0] == 0 && r[1] == 32 && r[2] == 32;
    const bool s3 = r[0] == 16 && r[1] == 24 && r[2] == 24;
    if (!s2 && !s3) return fail(TS_ERR_UNSUPPORTED, "bf16/e4m3 path supports rope_dims (0,32,32) or (16,24,24)");
  }
  return TS_OK;
}

template <typename Tab>
static void fill_theta(const ts_model_desc* m, Tab* hi, Tab* lo) {
  int pair = 0;
  for (int a = 0; a < 3; ++a) {
    const int D = m->rope_dims[a];
    for (int j = 0; j < D / 2; ++j, ++pair) {
      const double th = std::pow(static_cast<double>(m->rope_base), -2.0 * j / D);
      hi[pair] = static_cast<float>(th);
      lo[pair] = static_cast<float>(th - static_cast<double>(hi[pair]));
    }
  }
}

static ts_status check_plan(ts_plan_t p) {
  if (!p) return fail(TS_ERR_INVALID_ARG, "plan is NULL");
  int dev = -1;
  TS_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev != p->device) return fail(TS_ERR_INVALID_ARG, "current device %d differs from the plan's device %d", dev, p->device);
  return TS_OK;
}

static ts_status check_weights(const ts_model_desc* m, const ts_layer_weights* w) {
  if (!w) return fail(TS_ERR_INVALID_ARG, "weights are NULL");
  const bool rms = m->block == TS_BLOCK_RMS_SWIGLU;
  const void* ptrs[] = {w->ln1_g, rms ? w->ln1_g : w->ln1_b, w->w_qkv, w->b_qkv, w->q_g, w->k_g, w->w_o, w->b_o,
                        w->ln2_g, rms ? w->ln2_g : w->ln2_b, w->w_1,   w->b_1,   w->w_2, w->b_2};
  for (const void* p : ptrs) {
    if (!p) return fail(TS_ERR_INVALID_ARG, "a weight pointer is NULL");
    if (!aligned16(p)) return fail(TS_ERR_INVALID_ARG, "weight pointers must be 16-byte aligned");
  }
  if (m->dtype == TS_FP8_E4M3) {
    const void* s[] = {w->s_qkv, w->s_o, w->s_1, w->s_2};
    for (const void* p : s)
      if (!p || !aligned16(p)) return fail(TS_ERR_INVALID_ARG, "e4m3 weights need 16-byte aligned scales s_*");
  }
  return TS_OK;
}

// ============================================================================
// workspace layout
// ============================================================================
struct Workspace {
  void* xn;      // [Mx, d]   normalised rows
  void* qkv;     // [Mx, 3d]
  void* o;       // [T*N, d]  attention output
  void* a;       // [U+T, d]  blended attention output
  void* h;       // [Mx, f]   MLP hidden
  uint8_t* q8;   // [Mx, max(d, f)] e4m3 GEMM operand
  float* qs;     // [Mx]      its per-row scales
  void* X;       // [T*N, d]  per-tile state (stack)
  void* S;       // [U+T, d]  shared state (stack)
  float2* rope;  // RoPE cos/sin table (rope_table_entries)
  void* sm;      // [U+T, d]  partial sharing: merged per-tile state, then a per-token result
  size_t bytes;
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// entries of the RoPE table of a plan and model: per axis, grid extent x pairs
static size_t rope_table_entries(const ts_plan_s* p, const ts_model_desc* m) {
  size_t n = 0;
  for (int a = 0; a < 3; ++a) n += static_cast<size_t>(p->grid[a]) * (m->rope_dims[a] / 2);
  return n;
}

static ts::RopeTable make_rope_table(const ts_plan_s* p, const ts_model_desc* m, float2* cs) {
  ts::RopeTable rt{};
  rt.cs = cs;
  int off = 0;
  for (int a = 0; a < 3; ++a) {
    rt.G[a] = p->grid[a];
    rt.half[a] = m->rope_dims[a] / 2;
    rt.off[a] = off;
    off += rt.G[a] * rt.half[a];
  }
  rt.total = off;
  rt.base = m->rope_base;
  return rt;
}

// Regions of the caller workspace (256-byte aligned, in this order).  With
// shared_only the regions cover one shared layer alone (rows U + T*R; no stack
// states, no partial-sharing buffer): the scratch of ts_block_shared_noalloc.
static Workspace layout(const ts_plan_s* p, const ts_model_desc* m, bool stack, char* base, bool shared_only = false) {
  const size_t Mt = static_cast<size_t>(p->T) * p->N, Ms = static_cast<size_t>(p->U) + p->G;
  const size_t Mx = shared_only ? Ms : std::max(Mt, Ms);
  const size_t e = esize(m->dtype), d = m->d, f = m->mlp;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* r = base ? base + off : nullptr;
    off += align256(bytes);
    return r;
  };
  Workspace w{};
  w.xn = take(Mx * d * e);
  w.qkv = take(Mx * 3 * d * e);
  w.o = take(Mt * d * e);
  w.a = take(Ms * d * e);
  w.h = take(Mx * f * e);
  if (m->dtype == TS_FP8_E4M3) {
    w.q8 = reinterpret_cast<uint8_t*>(take(Mx * std::max(d, f)));
    w.qs = reinterpret_cast<float*>(take(Mx * 4));
  }
  if (stack && !shared_only) {
    w.X = take(Mt * d * e);
    w.S = take(Ms * d * e);
  }
  w.rope = reinterpret_cast<float2*>(take(rope_table_entries(p, m) * sizeof(float2)));
  if (!shared_only) w.sm = take(Ms * d * e);
  w.bytes = off;
  return w;
}

// ============================================================================
// launchers
// ============================================================================
static int g_num_sms = 0;
static int num_sms() {
  if (!g_num_sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

static inline unsigned rows_grid(size_t rows) { return static_cast<unsigned>((rows + 7) / 8); }

template <typename T, bool Q8>
static ts_status launch_layernorm_vec(const void* x, int rows, int d, const float* g, const float* b, float eps, int rms,
                                      void* y, uint8_t* q8, float* qs, const ts::RopeTable& rt, cudaStream_t st) {
  const unsigned fill_blocks = rt.cs ? static_cast<unsigned>((rt.total + 255) / 256) : 0u;
  constexpr int E = ts::Vec<T>::E;
  const int nv = d / (32 * E);
  const T* xx = static_cast<const T*>(x);
  T* yy = static_cast<T*>(y);
  trace_pre(st);
  // row blocks: as many as are resident at once (all of them walk the rows grid-stride)
#define TS_LN_CASE(NV)                                                                                      \
  case NV: {                                                                                                \
    auto kern = ts::layernorm_kernel<T, NV, Q8>;                                                            \
    static int occ = 0;                                                                                     \
    if (occ <= 0) {                                                                                         \
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 256, 0) != cudaSuccess || occ < 1) occ = 1; \
    }                                                                                                       \
    const unsigned row_blocks = std::min<unsigned>(rows_grid(rows), static_cast<unsigned>(occ * num_sms())); \
    launch_pdl(kern, dim3(row_blocks + fill_blocks), dim3(256), 0, st, xx, rows, d, g, b, eps, rms, yy, q8, qs, rt, \
               row_blocks);                                                                                 \
    break;                                                                                                  \
  }
  switch (nv) {
    TS_LN_CASE(1) TS_LN_CASE(2) TS_LN_CASE(3) TS_LN_CASE(4) TS_LN_CASE(5) TS_LN_CASE(6) TS_LN_CASE(7) TS_LN_CASE(8)
    default: return fail(TS_ERR_UNSUPPORTED, "layernorm width %d", d);
  }
#undef TS_LN_CASE
  return trace_post(st, "layernorm");
}

// y = Norm(x): LayerNorm, or RMSNorm for TS_BLOCK_RMS_SWIGLU (b unused); for e4m3
// writes q8/qs instead of y.
static ts_status run_layernorm(const ts_model_desc* m, const void* x, int rows, const float* g, const float* b,
                               void* y, uint8_t* q8, float* qs, cudaStream_t st,
                               const ts::RopeTable& rt = ts::RopeTable{}) {
  if (rows == 0) return TS_OK;
  const int d = m->d;
  const int rms = m->block == TS_BLOCK_RMS_SWIGLU;
  const double e = esize(m->dtype);
  set_work("layernorm", 0.0, static_cast<double>(rows) * d * (e + (q8 ? 1.0 : e)) + (q8 ? 4.0 * rows : 0.0));
  if (m->dtype == TS_F32) {
    if (d % 128 == 0 && d <= 1024)
      return launch_layernorm_vec<float, false>(x, rows, d, g, b, m->eps_ln, rms, y, nullptr, nullptr, ts::RopeTable{}, st);
    trace_pre(st);
    ts::layernorm_generic_kernel<float><<<rows_grid(rows), 256, 0, st>>>(static_cast<const float*>(x), rows, d, g, b,
                                                                        m->eps_ln, rms, static_cast<float*>(y));
    return trace_post(st, "layernorm_generic");
  }
  if (q8) return launch_layernorm_vec<bf16, true>(x, rows, d, g, b, m->eps_ln, rms, nullptr, q8, qs, rt, st);
  return launch_layernorm_vec<bf16, false>(x, rows, d, g, b, m->eps_ln, rms, y, nullptr, nullptr, rt, st);
}

template <typename T, bool Q8>
static ts_status launch_merge_vec(const ts_plan_s* p, const void* P, int rows, int d, void* A, uint8_t* q8,
                                  float* qs, cudaStream_t st) {
  constexpr int E = ts::Vec<T>::E;
  const int nv = d / (32 * E);
  const T* pp = static_cast<const T*>(P);
  T* aa = static_cast<T*>(A);
  // Staged variant: every warp holds two buffers of max_cover rows in shared memory.
  const size_t smem = static_cast<size_t>(ts::kMergeWarps) * 2 * p->max_cover * d * sizeof(T) + 16 * ts::kMergeWarps;
  const int per_sm = static_cast<int>(std::min<size_t>(8, (227u * 1024u) / std::max<size_t>(smem, 1)));
  if (per_sm >= 1) {
    trace_pre(st);
    const unsigned grid = static_cast<unsigned>(
        std::min<size_t>((static_cast<size_t>(rows) + ts::kMergeWarps - 1) / ts::kMergeWarps,
                         static_cast<size_t>(per_sm) * num_sms()));
#define TS_MB_CASE(NV)                                                                                        \
  case NV: {                                                                                                  \
    auto kern = ts::merge_bulk_kernel<T, NV, Q8>;                                                             \
    static int configured[64] = {0};                                                                          \
    int dev = 0;                                                                                              \
    cudaGetDevice(&dev);                                                                                      \
    if (dev < 64 && !configured[dev]) {                                                                       \
      TS_CUDA_CHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));     \
      configured[dev] = 1;                                                                                    \
    }                                                                                                         \
    launch_pdl(kern, dim3(grid), dim3(32 * ts::kMergeWarps), smem, st, pp, rows, p->U, p->N, p->R, d,          \
               static_cast<const int*>(p->d_tok_ptr), static_cast<const int*>(p->d_tok_ent),                   \
               static_cast<const float*>(p->d_wbar), p->max_cover, aa, q8, qs);                              \
    break;                                                                                                    \
  }
    switch (nv) {
      TS_MB_CASE(1) TS_MB_CASE(2) TS_MB_CASE(3) TS_MB_CASE(4) TS_MB_CASE(5) TS_MB_CASE(6) TS_MB_CASE(7) TS_MB_CASE(8)
      default: return fail(TS_ERR_UNSUPPORTED, "merge width %d", d);
    }
#undef TS_MB_CASE
    return trace_post(st, "merge");
  }
  trace_pre(st);
#define TS_MG_CASE(NV)                                                                                    \
  case NV:                                                                                                \
    launch_pdl(ts::merge_kernel<T, NV, Q8>, dim3(rows_grid(rows)), dim3(256), 0, st, pp, rows, p->U, p->N,    \
               p->R, d,                                                                                     \
               static_cast<const int*>(p->d_tok_ptr), static_cast<const int*>(p->d_tok_ent),               \
               static_cast<const float*>(p->d_wbar), aa, q8, qs);                                           \
    break;
  switch (nv) {
    TS_MG_CASE(1) TS_MG_CASE(2) TS_MG_CASE(3) TS_MG_CASE(4) TS_MG_CASE(5) TS_MG_CASE(6) TS_MG_CASE(7) TS_MG_CASE(8)
    default: return fail(TS_ERR_UNSUPPORTED, "merge width %d", d);
  }
#undef TS_MG_CASE
  return trace_post(st, "merge");
}

static ts_status run_merge(const char* name, const ts_plan_s* p, const ts_model_desc* m, const void* P, int rows,
                           void* A, uint8_t* q8, float* qs, cudaStream_t st) {
  if (rows == 0) return TS_OK;
  const int d = m->d;
  {
    // reads every (tile, slot) entry of the rows written once, writes each row once
    const double e = esize(m->dtype);
    const double reads = static_cast<double>(p->nnz) * d * e + (rows > p->U ? static_cast<double>(rows - p->U) * d * e : 0.0);
    const double writes = static_cast<double>(rows) * d * (q8 ? 1.0 : e) + (q8 ? 4.0 * rows : 0.0);
    set_work(name, 0.0, reads + writes);
  }
  if (m->dtype == TS_F32) {
    if (d % 128 == 0 && d <= 1024) return launch_merge_vec<float, false>(p, P, rows, d, A, nullptr, nullptr, st);
    trace_pre(st);
    ts::merge_generic_kernel<float><<<rows_grid(rows), 256, 0, st>>>(static_cast<const float*>(P), rows, p->U, p->N, p->R, d,
                                                                    p->d_tok_ptr, p->d_tok_ent, p->d_wbar,
                                                                    static_cast<float*>(A));
    return trace_post(st, "merge_generic");
  }
  if (q8) return launch_merge_vec<bf16, true>(p, P, rows, d, nullptr, q8, qs, st);
  return launch_merge_vec<bf16, false>(p, P, rows, d, A, nullptr, nullptr, st);
}

static ts_status run_quantize(const void* x, int rows, int cols, uint8_t* q, float* s, cudaStream_t st) {
  if (rows == 0) return TS_OK;
  set_work("quantize_e4m3", 0.0, static_cast<double>(rows) * cols * 3.0 + 4.0 * rows);
  trace_pre(st);
  launch_pdl(ts::quantize_rows_kernel, dim3(rows_grid(rows)), dim3(256), 0, st, static_cast<const bf16*>(x), rows, cols,
             q, s);
  return trace_post(st, "quantize_rows");
}

// ---------------------------------------------------------------------------
// tensor-core GEMM
// ---------------------------------------------------------------------------


template <int BN, int STAGES, int EPI, bool FP8, int R0, int R1, int R2, int CG = 1>
static ts_status launch_gemm_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                                const ts::GemmArgs& args, cudaStream_t st) {
  using SM = ts::GemmSmem<BN, STAGES, CG>;
  auto kern = ts::gemm_tc_kernel<BN, STAGES, EPI, FP8, R0, R1, R2, CG>;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    TS_CUDA_CHECK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::LAUNCH_BYTES));
    configured[dev] = 1;
  }
  const int tiles = ((args.M + 128 * CG - 1) / (128 * CG)) * (args.N / BN);
  trace_pre(st);
  if (CG == 2) {
    // one pair per two SMs, both CTAs of a pair walking the same tiles
    dim3 grid(2 * std::min(tiles, num_sms() / 2));
    launch_pdl_pair(kern, grid, dim3(ts::kGemmThreads), SM::LAUNCH_BYTES, st, ta, tb, td, args);
  } else {
    dim3 grid(std::min(tiles, num_sms()));
    launch_pdl(kern, grid, dim3(ts::kGemmThreads), SM::LAUNCH_BYTES, st, ta, tb, td, args);
  }
  return trace_post(st, "gemm_tc");
}

template <int EPI, bool FP8, int R0, int R1, int R2>
static ts_status dispatch_gemm_bn(int bn, bool pair, const CUtensorMap& ta, const CUtensorMap& tb,
                                  const CUtensorMap& td, const ts::GemmArgs& args, cudaStream_t st) {
  switch (bn) {
    case 256:
      if (pair) return launch_gemm_tc<256, 6, EPI, FP8, R0, R1, R2, 2>(ta, tb, td, args, st);
      return launch_gemm_tc<256, 4, EPI, FP8, R0, R1, R2>(ta, tb, td, args, st);
    case 128: return launch_gemm_tc<128, 6, EPI, FP8, R0, R1, R2>(ta, tb, td, args, st);
    default:
      if constexpr (EPI == ts::EPI_SWIGLU)   // SwiGLU tiles are at least 128 wide
        return launch_gemm_tc<128, 6, EPI, FP8, R0, R1, R2>(ta, tb, td, args, st);
      else
        return launch_gemm_tc<64, 8, EPI, FP8, R0, R1, R2>(ta, tb, td, args, st);
  }
}

// Two-SM pairs (256-row tiles) for GEMMs of at least this many rows with 256-wide
// tiles; TS_GEMM_PAIR=0 in the environment turns them off (for comparisons).
static constexpr int kGemmPairMinRows = 2048;
static bool gemm_pairs_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("TS_GEMM_PAIR");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Output tile width for the persistent GEMM: the persistent CTAs walk the tiles
// round-robin, so the busiest CTA handles ceil(tiles / SMs) tiles.  Cost model:
// that count times (BN + 48), 48 columns standing for the fixed per-tile work
// (pipeline fill, epilogue tail); ties go to the wider tile.
static int pick_bn(int M, int N) {
  // tuning override: TS_GEMM_BN=64|128|256 forces the tile width where it divides N
  static const int forced = [] {
    const char* e = std::getenv("TS_GEMM_BN");
    return e ? std::atoi(e) : 0;
  }();
  if ((forced == 64 || forced == 128 || forced == 256) && N % forced == 0) return forced;
  const int mt = (M + 127) / 128;
  const int sms = num_sms();
  int best = 64;
  long best_cost = -1;
  for (int bn : {256, 128, 64}) {
    if (N % bn) continue;
    const long tiles = static_cast<long>(mt) * (N / bn);
    const long cost = ((tiles + sms - 1) / sms) * (bn + 48);
    if (best_cost < 0 || cost < best_cost) {
      best = bn;
      best_cost = cost;
    }
  }
  return best;
}

// Y[M, N] = A[M, K] W[N, K]^T with epilogue; A bf16 (or e4m3 + a_scale), W bf16 (or e4m3 + w_scale).
// EPI_SWIGLU: N is the output width and W, bias, w_scale have 2N rows (gate, then up).
static ts_status run_gemm_tc(const char* name, const ts_model_desc* m, int epi, const void* A, const float* a_scale,
                             const void* W, const float* w_scale, int M, int N, int K, const float* bias, bf16* out,
                             const ts_layer_weights* qk, const int* pos, cudaStream_t st,
                             const ts::RopeTable& rt = ts::RopeTable{}) {
  if (M == 0) return TS_OK;
  const bool fp8 = m->dtype == TS_FP8_E4M3;
  const bool glu = epi == ts::EPI_SWIGLU;
  const int NA = glu ? 2 * N : N;   // accumulator columns = rows of W
  {
    const double ea = fp8 ? 1.0 : 2.0;
    const double bytes = static_cast<double>(M) * K * ea + static_cast<double>(NA) * K * ea +
                         static_cast<double>(M) * N * 2.0 * (epi == ts::EPI_RESID ? 2.0 : 1.0);
    set_work(name, 2.0 * M * static_cast<double>(NA) * K, bytes);
  }
  if (K % (fp8 ? 128 : 64) || N % 64) return fail(TS_ERR_UNSUPPORTED, "GEMM sizes K=%d N=%d not tiled", K, N);
  int bn = pick_bn(M, NA);
  if (glu && bn < 128) bn = 128;    // NA = 2N is a multiple of 128
  // 256-wide tiles of tall GEMMs run as two-SM pairs of 256 x 256 tiles
  const bool pair = bn == 256 && M >= kGemmPairMinRows && gemm_pairs_enabled();
  CUtensorMap ta, tb, td;
  TS_TRY(make_tmap(&ta, A, M, K, fp8 ? 1 : 2, 128));
  TS_TRY(make_tmap(&tb, W, NA, K, fp8 ? 1 : 2, (glu || pair) ? bn / 2 : bn));
  TS_TRY(make_tmap(&td, out, M, N, 2, 32));   // output (and residual): 32 x 64 chunks of the epilogue warps
  ts::GemmArgs g{};
  g.M = M;
  g.N = NA;
  g.K = K;
  g.bias = bias;
  g.out = out;
  g.ldo = N;
  g.a_scale = a_scale;
  g.w_scale = w_scale;
  g.d = m->d;
  g.eps_qk = m->eps_qk;
  if (epi == ts::EPI_QKV) {
    g.q_g = qk->q_g;
    g.k_g = qk->k_g;
    g.pos = reinterpret_cast<const int4*>(pos);
    g.rope_cs = rt.cs;
    for (int a = 0; a < 3; ++a) g.rope_off[a] = rt.off[a];
  }
  const bool r3 = m->rope_dims[0] == 16;
#define TS_GEMM_EPI(E, R0, R1, R2) \
  (fp8 ? dispatch_gemm_bn<E, true, R0, R1, R2>(bn, pair, ta, tb, td, g, st)     \
       : dispatch_gemm_bn<E, false, R0, R1, R2>(bn, pair, ta, tb, td, g, st))
  switch (epi) {
    case ts::EPI_BIAS: return TS_GEMM_EPI(ts::EPI_BIAS, 0, 32, 32);
    case ts::EPI_GELU: return TS_GEMM_EPI(ts::EPI_GELU, 0, 32, 32);
    case ts::EPI_RESID: return TS_GEMM_EPI(ts::EPI_RESID, 0, 32, 32);
    case ts::EPI_QKV: return r3 ? TS_GEMM_EPI(ts::EPI_QKV, 16, 24, 24) : TS_GEMM_EPI(ts::EPI_QKV, 0, 32, 32);
    case ts::EPI_SWIGLU: return TS_GEMM_EPI(ts::EPI_SWIGLU, 0, 32, 32);
  }
#undef TS_GEMM_EPI
  return fail(TS_ERR_INVALID_ARG, "unknown epilogue");
}

// fp32 SIMT GEMM (EPI_SWIGLU: N is the output width, W has 2N rows)
static ts_status run_gemm_f32(const char* name, int epi, const float* A, const float* W, int M, int N, int K,
                              const float* bias, float* Y, cudaStream_t st) {
  if (M == 0) return TS_OK;
  const int NA = epi == ts::EPI_SWIGLU ? 2 * N : N;
  set_work(name, 2.0 * M * static_cast<double>(NA) * K,
           4.0 * (static_cast<double>(M) * K + static_cast<double>(NA) * K + M * static_cast<double>(N) * (epi == ts::EPI_RESID ? 2 : 1)));
  dim3 grid((M + 63) / 64, (N + 63) / 64);
  trace_pre(st);
  switch (epi) {
    case ts::EPI_SWIGLU:
      grid.y = (N + 31) / 32;
      ts::gemm_f32_kernel<3><<<grid, 256, 0, st>>>(A, W, bias, Y, M, N, K);
      break;
    case ts::EPI_GELU: ts::gemm_f32_kernel<1><<<grid, 256, 0, st>>>(A, W, bias, Y, M, N, K); break;
    case ts::EPI_RESID: ts::gemm_f32_kernel<2><<<grid, 256, 0, st>>>(A, W, bias, Y, M, N, K); break;
    default: ts::gemm_f32_kernel<0><<<grid, 256, 0, st>>>(A, W, bias, Y, M, N, K); break;
  }
  return trace_post(st, "gemm_f32");
}

// ---------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------
static ts_status run_attention(const ts_plan_s* p, const ts_model_desc* m, bool shared, const void* qkv, void* O,
                               cudaStream_t st) {
  const int hd = m->d / m->heads;
  ts::AttnArgs a{};
  a.qkv = qkv;
  a.rowmap = shared ? p->d_rowmap : nullptr;
  a.O = O;
  a.N = p->N;
  a.Nw = p->N - 1;    // slots after slot 0 (the tile's first register, handled apart)
  a.d = m->d;
  a.heads = m->heads;
  a.T = p->T;
  a.scale = 1.0f / std::sqrt(static_cast<float>(hd));
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(hd)));
  {
    const double e = esize(m->dtype), rows = static_cast<double>(p->T) * p->N;
    set_work("attention", 4.0 * p->T * static_cast<double>(p->N) * p->N * m->d, rows * 3.0 * m->d * e + rows * m->d * e);
  }
  trace_pre(st);
  if (m->dtype == TS_F32) {
    dim3 grid((p->N + 63) / 64, m->heads, p->T);
    switch (hd) {
      case 16: ts::attn_f32_kernel<16><<<grid, 64, 0, st>>>(a); break;
      case 32: ts::attn_f32_kernel<32><<<grid, 64, 0, st>>>(a); break;
      default: ts::attn_f32_kernel<64><<<grid, 64, 0, st>>>(a); break;
    }
    return trace_post(st, "attn_f32");
  }
  const int nqb = (p->N - 1 + ts::kAttnBQ - 1) / ts::kAttnBQ;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    TS_CUDA_CHECK(cudaFuncSetAttribute(ts::attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       ts::AttnSmem::LAUNCH_BYTES));
    // four CTAs per SM need the largest shared-memory carveout
    TS_CUDA_CHECK(cudaFuncSetAttribute(ts::attn_bf16_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       cudaSharedmemCarveoutMaxShared));
    configured[dev] = 1;
  }
  // Loads: a block of 32 window slots that is whole window rows of one frame (or
  // a part of one row) is one box of a 3-D map over the grid; otherwise runs of
  // consecutive rows are 2-D boxes of `run` rows (the per-tile layout is one run
  // per block), else four-row gathers through a map with one-row boxes.
  const int wx = p->win[2], wy = p->win[1];
  const int bk = ts::kAttnBK;
  const bool grid_box = p->R == 1 && (wx <= bk ? (bk % wx == 0 && (wy * wx) % bk == 0) : wx % bk == 0);
  CUtensorMap tm;
  if (shared && grid_box) {
    a.load = 2;
    a.gw = p->grid[2];
    const int bx = std::min(wx, bk);
    TS_TRY(make_tmap_grid(&tm, qkv, 3 * m->d, p->grid[2], p->grid[0] * p->grid[1], bx, bk / bx));
  } else {
    a.run = shared ? std::min(p->run, bk) : bk;   // runs of 64 consecutive rows are runs of 32 as well
    a.load = a.run > 0 ? 1 : 0;
    TS_TRY(make_tmap(&tm, qkv, shared ? p->U + p->G : p->T * p->N, 3 * m->d, 2, a.run > 0 ? a.run : 1));
  }
  a.head_major = shared ? 1 : 0;
  a.nqb = nqb;
  // block x = nqb of each tile and head computes the global token's query row
  dim3 grid = shared ? dim3(nqb + 1, p->T, m->heads)    // head slowest: neighbouring tiles of one head share L2
                     : dim3(nqb + 1, m->heads, p->T);   // tile slowest: a tile's rows are read once for all heads
  launch_pdl(ts::attn_bf16_kernel, grid, dim3(ts::kAttnThreads), ts::AttnSmem::LAUNCH_BYTES, st, tm, a);
  return trace_post(st, "attn_bf16");
}

// ---------------------------------------------------------------------------
// QKV step: LN1 + QKV GEMM + QK-RMSNorm + RoPE
// ---------------------------------------------------------------------------
static ts_status run_qkv(const ts_plan_s* p, const ts_model_desc* m, const ts_layer_weights* w, bool shared,
                         const void* state, void* qkv, const Workspace& ws, cudaStream_t st) {
  const int rows = shared ? p->U + p->G : p->T * p->N;
  const int* pos = shared ? p->d_pos_shared : p->d_pos_tiled;
  const int d = m->d;
  if (m->dtype == TS_F32) {
    TS_TRY(run_layernorm(m, state, rows, w->ln1_g, w->ln1_b, ws.xn, nullptr, nullptr, st));
    TS_TRY(run_gemm_f32("gemm_qkv", ts::EPI_BIAS, static_cast<const float*>(ws.xn), static_cast<const float*>(w->w_qkv), rows,
                        3 * d, d, w->b_qkv, static_cast<float*>(qkv), st));
    ts::RopeF32 r{};
    for (int a = 0; a < 3; ++a) r.dims[a] = m->rope_dims[a];
    fill_theta(m, r.th_hi, r.th_lo);
    const size_t n = static_cast<size_t>(rows) * m->heads * 2;
    set_work("qk_norm_rope", 0.0, 2.0 * rows * 2.0 * d * 4.0);
    trace_pre(st);
    ts::qk_norm_rope_f32_kernel<<<static_cast<unsigned>((n + 127) / 128), 128, 0, st>>>(
        static_cast<float*>(qkv), rows, d, m->heads, w->q_g, w->k_g, m->eps_qk, reinterpret_cast<const int4*>(pos), r);
    return trace_post(st, "qk_norm_rope_f32");
  }
  // LN1 also fills the RoPE table that the QKV epilogue reads
  const ts::RopeTable rt = make_rope_table(p, m, ws.rope);
  if (m->dtype == TS_FP8_E4M3) {
    TS_TRY(run_layernorm(m, state, rows, w->ln1_g, w->ln1_b, nullptr, ws.q8, ws.qs, st, rt));
    return run_gemm_tc("gemm_qkv", m, ts::EPI_QKV, ws.q8, ws.qs, w->w_qkv, w->s_qkv, rows, 3 * d, d, w->b_qkv,
                       static_cast<bf16*>(qkv), w, pos, st, rt);
  }
  TS_TRY(run_layernorm(m, state, rows, w->ln1_g, w->ln1_b, ws.xn, nullptr, nullptr, st, rt));
  return run_gemm_tc("gemm_qkv", m, ts::EPI_QKV, ws.xn, nullptr, w->w_qkv, nullptr, rows, 3 * d, d, w->b_qkv,
                     static_cast<bf16*>(qkv), w, pos, st, rt);
}

// out-proj (+= state) from attention/blend output `att` [rows, d]
static ts_status run_out_proj(const ts_model_desc* m, const ts_layer_weights* w, const void* att, bool att_quantised,
                              int rows, void* state, const Workspace& ws, cudaStream_t st) {
  const int d = m->d;
  if (m->dtype == TS_F32)
    return run_gemm_f32("gemm_out", ts::EPI_RESID, static_cast<const float*>(att), static_cast<const float*>(w->w_o), rows, d, d,
                        w->b_o, static_cast<float*>(state), st);
  if (m->dtype == TS_FP8_E4M3) {
    if (!att_quantised) TS_TRY(run_quantize(att, rows, d, ws.q8, ws.qs, st));
    return run_gemm_tc("gemm_out", m, ts::EPI_RESID, ws.q8, ws.qs, w->w_o, w->s_o, rows, d, d, w->b_o, static_cast<bf16*>(state),
                       nullptr, nullptr, st);
  }
  return run_gemm_tc("gemm_out", m, ts::EPI_RESID, att, nullptr, w->w_o, nullptr, rows, d, d, w->b_o, static_cast<bf16*>(state),
                     nullptr, nullptr, st);
}

// out (+)= W2 act(W1 Norm2(in) + b1) + b2 with act GELU, or SwiGLU for
// TS_BLOCK_RMS_SWIGLU (W1 [2f, d]); resid: out is the residual stream (in place
// when out == in), else out is written.
static ts_status run_mlp_any(const ts_model_desc* m, const ts_layer_weights* w, int rows, const void* in, void* out,
                             bool resid, const Workspace& ws, cudaStream_t st) {
  const int d = m->d, f = m->mlp;
  const int up = m->block == TS_BLOCK_RMS_SWIGLU ? ts::EPI_SWIGLU : ts::EPI_GELU;
  const int down = resid ? ts::EPI_RESID : ts::EPI_BIAS;
  if (m->dtype == TS_F32) {
    TS_TRY(run_layernorm(m, in, rows, w->ln2_g, w->ln2_b, ws.xn, nullptr, nullptr, st));
    TS_TRY(run_gemm_f32("gemm_up", up, static_cast<const float*>(ws.xn), static_cast<const float*>(w->w_1), rows, f, d,
                        w->b_1, static_cast<float*>(ws.h), st));
    return run_gemm_f32("gemm_down", down, static_cast<const float*>(ws.h), static_cast<const float*>(w->w_2), rows, d, f,
                        w->b_2, static_cast<float*>(out), st);
  }
  if (m->dtype == TS_FP8_E4M3) {
    TS_TRY(run_layernorm(m, in, rows, w->ln2_g, w->ln2_b, nullptr, ws.q8, ws.qs, st));
    TS_TRY(run_gemm_tc("gemm_up", m, up, ws.q8, ws.qs, w->w_1, w->s_1, rows, f, d, w->b_1, static_cast<bf16*>(ws.h),
                       nullptr, nullptr, st));
    TS_TRY(run_quantize(ws.h, rows, f, ws.q8, ws.qs, st));
    return run_gemm_tc("gemm_down", m, down, ws.q8, ws.qs, w->w_2, w->s_2, rows, d, f, w->b_2, static_cast<bf16*>(out),
                       nullptr, nullptr, st);
  }
  TS_TRY(run_layernorm(m, in, rows, w->ln2_g, w->ln2_b, ws.xn, nullptr, nullptr, st));
  TS_TRY(run_gemm_tc("gemm_up", m, up, ws.xn, nullptr, w->w_1, nullptr, rows, f, d, w->b_1, static_cast<bf16*>(ws.h),
                     nullptr, nullptr, st));
  return run_gemm_tc("gemm_down", m, down, ws.h, nullptr, w->w_2, nullptr, rows, d, f, w->b_2, static_cast<bf16*>(out),
                     nullptr, nullptr, st);
}

// state += MLP(state)
static ts_status run_mlp(const ts_model_desc* m, const ts_layer_weights* w, int rows, void* state, const Workspace& ws,
                         cudaStream_t st) {
  return run_mlp_any(m, w, rows, state, state, true, ws, st);
}

// per-tile copies of the stack input (grid tokens S0, global tokens G0)
static ts_status run_gather(const ts_plan_s* p, const ts_model_desc* m, const void* S0, const void* G0, void* X,
                            cudaStream_t st) {
  const int nrows = p->T * p->N;
  const size_t rb = static_cast<size_t>(m->d) * esize(m->dtype);
  set_work("gather", 0.0, 2.0 * nrows * static_cast<double>(rb));
  trace_pre(st);
  launch_pdl(ts::gather_rows_kernel, dim3(rows_grid(nrows)), dim3(256), 0, st, static_cast<const uint8_t*>(S0),
             static_cast<const uint8_t*>(G0), static_cast<const int*>(p->d_rowmap), nrows, p->U, rb,
             static_cast<uint8_t*>(X));
  return trace_post(st, "gather_rows");
}

// X[r] += R[rowmap[r]] over the T * N per-tile rows (partial sharing)
static ts_status run_scatter_add(const ts_plan_s* p, const ts_model_desc* m, const void* R, void* X, cudaStream_t st) {
  const int nrows = p->T * p->N;
  const int d = m->d;
  const double e = esize(m->dtype);
  set_work("scatter_add", 0.0, 3.0 * nrows * static_cast<double>(d) * e);
  trace_pre(st);
  if (m->dtype == TS_F32)
    launch_pdl(ts::scatter_add_rows_kernel<float>, dim3(rows_grid(nrows)), dim3(256), 0, st,
               static_cast<const float*>(R), static_cast<const int*>(p->d_rowmap), nrows, d, static_cast<float*>(X));
  else
    launch_pdl(ts::scatter_add_rows_kernel<bf16>, dim3(rows_grid(nrows)), dim3(256), 0, st,
               static_cast<const bf16*>(R), static_cast<const int*>(p->d_rowmap), nrows, d, static_cast<bf16*>(X));
  return trace_post(st, "scatter_add");
}

// out = att W_o^T + b_o (no residual): the out-projection of a shared operation
static ts_status run_out_bias(const ts_model_desc* m, const ts_layer_weights* w, const void* att, bool att_quantised,
                              int rows, void* out, const Workspace& ws, cudaStream_t st) {
  const int d = m->d;
  if (m->dtype == TS_F32)
    return run_gemm_f32("gemm_out", ts::EPI_BIAS, static_cast<const float*>(att), static_cast<const float*>(w->w_o), rows, d, d,
                        w->b_o, static_cast<float*>(out), st);
  if (m->dtype == TS_FP8_E4M3) {
    if (!att_quantised) TS_TRY(run_quantize(att, rows, d, ws.q8, ws.qs, st));
    return run_gemm_tc("gemm_out", m, ts::EPI_BIAS, ws.q8, ws.qs, w->w_o, w->s_o, rows, d, d, w->b_o, static_cast<bf16*>(out),
                       nullptr, nullptr, st);
  }
  return run_gemm_tc("gemm_out", m, ts::EPI_BIAS, att, nullptr, w->w_o, nullptr, rows, d, d, w->b_o, static_cast<bf16*>(out),
                     nullptr, nullptr, st);
}

// out = MLP(in) (no residual): the MLP of a shared operation
static ts_status run_mlp_out(const ts_model_desc* m, const ts_layer_weights* w, int rows, const void* in, void* out,
                             const Workspace& ws, cudaStream_t st) {
  return run_mlp_any(m, w, rows, in, out, false, ws, st);
}

// ============================================================================
// layers
// ============================================================================
static ts_status layer_tiled(const ts_plan_s* p, const ts_model_desc* m, const ts_layer_weights* w, void* X,
                             const Workspace& ws, cudaStream_t st) {
  const int rows = p->T * p->N;
  TS_TRY(run_qkv(p, m, w, false, X, ws.qkv, ws, st));
  TS_TRY(run_attention(p, m, false, ws.qkv, ws.o, st));
  TS_TRY(run_out_proj(m, w, ws.o, false, rows, X, ws, st));
  return run_mlp(m, w, rows, X, ws, st);
}

static ts_status layer_shared(const ts_plan_s* p, const ts_model_desc* m, const ts_layer_weights* w, void* S,
                              const Workspace& ws, cudaStream_t st) {
  const int rows = p->U + p->G;
  TS_TRY(run_qkv(p, m, w, true, S, ws.qkv, ws, st));
  TS_TRY(run_attention(p, m, true, ws.qkv, ws.o, st));
  const bool q = m->dtype == TS_FP8_E4M3;
  TS_TRY(run_merge("blend", p, m, ws.o, rows, q ? nullptr : ws.a, q ? ws.q8 : nullptr, q ? ws.qs : nullptr, st));
  TS_TRY(run_out_proj(m, w, ws.a, q, rows, S, ws, st));
  return run_mlp(m, w, rows, S, ws, st);
}

// Partial sharing ([TileShare] Tab. 1 top): per-tile residual streams X, the
// operations in `ops` once per token on the merged inputs, their results used by
// (QKV) or added to (out-projection, MLP) every tile's copy of the token.
static ts_status layer_partial(const ts_plan_s* p, const ts_model_desc* m, const ts_layer_weights* w, unsigned ops,
                               void* X, const Workspace& ws, cudaStream_t st) {
  const int rows_t = p->T * p->N, rows_s = p->U + p->G;
  const bool q8 = m->dtype == TS_FP8_E4M3;
  if (ops & TS_SHARE_QKV) {
    TS_TRY(run_merge("merge", p, m, X, rows_s, ws.sm, nullptr, nullptr, st));
    TS_TRY(run_qkv(p, m, w, true, ws.sm, ws.qkv, ws, st));
    TS_TRY(run_attention(p, m, true, ws.qkv, ws.o, st));
  } else {
    TS_TRY(run_qkv(p, m, w, false, X, ws.qkv, ws, st));
    TS_TRY(run_attention(p, m, false, ws.qkv, ws.o, st));
  }
  if (ops & TS_SHARE_OUT) {
    TS_TRY(run_merge("blend", p, m, ws.o, rows_s, q8 ? nullptr : ws.a, q8 ? ws.q8 : nullptr, q8 ? ws.qs : nullptr, st));
    TS_TRY(run_out_bias(m, w, ws.a, q8, rows_s, ws.sm, ws, st));
    TS_TRY(run_scatter_add(p, m, ws.sm, X, st));
  } else {
    TS_TRY(run_out_proj(m, w, ws.o, false, rows_t, X, ws, st));
  }
  if (ops & TS_SHARE_MLP) {
    TS_TRY(run_merge("merge", p, m, X, rows_s, ws.sm, nullptr, nullptr, st));
    TS_TRY(run_mlp_out(m, w, rows_s, ws.sm, ws.a, ws, st));
    return run_scatter_add(p, m, ws.a, X, st);
  }
  return run_mlp(m, w, rows_t, X, ws, st);
}

static ts_status check_ws(const ts_plan_s* p, const ts_model_desc* m, bool stack, void* ws, size_t ws_bytes,
                          Workspace* out) {
  const Workspace need = layout(p, m, stack, nullptr);
  if (!ws) return fail(TS_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned16(ws)) return fail(TS_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (ws_bytes < need.bytes) return fail(TS_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need.bytes);
  *out = layout(p, m, stack, static_cast<char*>(ws));
  return TS_OK;
}

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

ts_status ts_gather_tiles(ts_plan_t p, const ts_model_desc* m, const void* S0, const void* G0, void* X,
                          void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  if (!S0 || !G0 || !X || !aligned16(S0) || !aligned16(G0) || !aligned16(X))
    return fail(TS_ERR_INVALID_ARG, "S0, G0, X must be 16-byte aligned device pointers");
  return run_gather(p, m, S0, G0, X, static_cast<cudaStream_t>(stream));
}

ts_status ts_trace_begin(int max_launches) {
  if (max_launches < 0) return fail(TS_ERR_INVALID_ARG, "max_launches < 0");
  if (g_trace.on) return fail(TS_ERR_INVALID_ARG, "trace already running");
  for (cudaEvent_t e : g_trace.ev) cudaEventDestroy(e);
  g_trace.ev.assign(2 * static_cast<size_t>(max_launches), nullptr);
  for (auto& e : g_trace.ev) TS_CUDA_CHECK(cudaEventCreate(&e));
  g_trace.cap = max_launches;
  g_trace.used = 0;
  g_trace.names.clear();
  g_trace.count.clear();
  g_trace.recs.clear();
  g_trace.on = true;
  return TS_OK;
}

ts_status ts_trace_end(ts_trace_entry* entries, int capacity, int* count) {
  if (!g_trace.on) return fail(TS_ERR_INVALID_ARG, "no trace running");
  g_trace.on = false;
  const size_t n = g_trace.names.size();
  std::vector<ts_trace_entry> out(n);
  for (size_t i = 0; i < n; ++i) {
    std::memset(&out[i], 0, sizeof(ts_trace_entry));
    std::strncpy(out[i].name, g_trace.names[i].c_str(), sizeof(out[i].name) - 1);
    out[i].launches = static_cast<int>(g_trace.count[i]);
  }
  for (const TraceRec& r : g_trace.recs) {
    TS_CUDA_CHECK(cudaEventSynchronize(g_trace.ev[2 * r.slot + 1]));
    float ms = 0.f;
    TS_CUDA_CHECK(cudaEventElapsedTime(&ms, g_trace.ev[2 * r.slot], g_trace.ev[2 * r.slot + 1]));
    ts_trace_entry& e = out[r.cls];
    e.timed += 1;
    e.ms += ms;
    e.flops += r.flops;
    e.bytes += r.bytes;
  }
  if (count) *count = static_cast<int>(n);
  if (entries)
    for (size_t i = 0; i < n && static_cast<int>(i) < capacity; ++i) entries[i] = out[i];
  return TS_OK;
}

long long ts_launch_count(void) { return g_launches.load(); }

const char* ts_status_string(ts_status s) {
  switch (s) {
    case TS_OK: return "ok";
    case TS_ERR_INVALID_ARG: return "invalid argument";
    case TS_ERR_UNSUPPORTED: return "unsupported";
    case TS_ERR_WORKSPACE: return "workspace too small";
    case TS_ERR_CUDA: return "CUDA error";
    case TS_ERR_DEVICE_CHECK: return "device-side check failed";
    case TS_ERR_TIMEOUT: return "device-side wait timed out";
    case TS_ERR_ALLOC: return "allocation failed";
  }
  return "unknown status";
}

const char* ts_last_error(void) { return g_last_error.c_str(); }

static ts_status plan_build_host(const int grid[3], const int win[3], const int stride[3], ts_blend_rule rule,
                                 int registers, ts_plan_s** out) {
  if (!grid || !win || !stride || !out) return fail(TS_ERR_INVALID_ARG, "NULL argument");
  *out = nullptr;
  if (registers < 1 || registers > 64) return fail(TS_ERR_INVALID_ARG, "registers per tile must lie in [1, 64]");
  if (rule != TS_BLEND_LINEAR_RAMP && rule != TS_BLEND_HARD_STITCH)
    return fail(TS_ERR_INVALID_ARG, "unknown blend rule %d", static_cast<int>(rule));
  for (int a = 0; a < 3; ++a) {
    if (grid[a] < 1 || win[a] < 1 || win[a] > grid[a] || stride[a] < 1 || stride[a] > win[a])
      return fail(TS_ERR_INVALID_ARG, "axis %d: need 1 <= win <= grid and 1 <= stride <= win", a);
  }
  if (static_cast<double>(grid[0]) * grid[1] * grid[2] > (1 << 28)) return fail(TS_ERR_UNSUPPORTED, "grid too large");
  if (static_cast<double>(win[0]) * win[1] * win[2] > (1 << 24)) return fail(TS_ERR_UNSUPPORTED, "window too large");
  ts_plan_s* P = new (std::nothrow) ts_plan_s();
  if (!P) return fail(TS_ERR_ALLOC, "host allocation failed");
  for (int a = 0; a < 3; ++a) {
    P->grid[a] = grid[a];
    P->win[a] = win[a];
    P->stride[a] = stride[a];
  }
  P->device = -1;
  P->rule = rule == TS_BLEND_HARD_STITCH ? 1 : 0;
  P->R = registers;
  if (!tsplan::build(*P)) {
    delete P;
    return fail(TS_ERR_INVALID_ARG, "tiling leaves a token uncovered");
  }
  if (static_cast<double>(P->T) * P->N > 2.0e9) {
    delete P;
    return fail(TS_ERR_UNSUPPORTED, "too many tile rows");
  }
  *out = P;
  return TS_OK;
}

ts_status ts_plan_create_host(const int grid[3], const int win[3], const int stride[3], ts_blend_rule rule,
                              ts_plan_t* out) {
  return plan_build_host(grid, win, stride, rule, 1, out);
}

ts_status ts_plan_create_host_registers(const int grid[3], const int win[3], const int stride[3], ts_blend_rule rule,
                                        int registers, ts_plan_t* out) {
  return plan_build_host(grid, win, stride, rule, registers, out);
}

ts_status ts_plan_create(const int grid[3], const int win[3], const int stride[3], ts_blend_rule rule,
                         ts_plan_t* out) {
  return ts_plan_create_registers(grid, win, stride, rule, 1, out);
}

ts_status ts_plan_create_registers(const int grid[3], const int win[3], const int stride[3], ts_blend_rule rule,
                                   int registers, ts_plan_t* out) {
  ts_plan_s* P = nullptr;
  TS_TRY(plan_build_host(grid, win, stride, rule, registers, &P));
  cudaError_t e = cudaGetDevice(&P->device);
  auto upload = [&](auto** dst, const auto& vec) -> bool {
    using E = typename std::decay<decltype(vec)>::type::value_type;
    if (e != cudaSuccess) return false;
    const size_t bytes = std::max<size_t>(vec.size(), 1) * sizeof(E);
    e = cudaMalloc(reinterpret_cast<void**>(dst), bytes);
    if (e != cudaSuccess) return false;
    if (!vec.empty()) e = cudaMemcpy(*dst, vec.data(), vec.size() * sizeof(E), cudaMemcpyHostToDevice);
    return e == cudaSuccess;
  };
  const bool ok = upload(&P->d_tok_ptr, P->tok_ptr) && upload(&P->d_tok_ent, P->tok_ent) &&
                  upload(&P->d_wbar, P->wbar) && upload(&P->d_rowmap, P->rowmap) &&
                  upload(&P->d_pos_shared, P->pos_shared) && upload(&P->d_pos_tiled, P->pos_tiled);
  if (!ok) {
    if (P->device < 0) P->device = 0;
    ts_plan_destroy(P);
    return fail(e == cudaErrorMemoryAllocation ? TS_ERR_ALLOC : TS_ERR_CUDA, "plan upload failed: %s",
                cudaGetErrorString(e));
  }
  *out = P;
  return TS_OK;
}

ts_status ts_plan_info(ts_plan_t p, ts_plan_desc* out) {
  if (!p || !out) return fail(TS_ERR_INVALID_ARG, "NULL argument");
  for (int a = 0; a < 3; ++a) {
    out->grid[a] = p->grid[a];
    out->win[a] = p->win[a];
    out->stride[a] = p->stride[a];
  }
  out->T = p->T;
  out->U = p->U;
  out->Nw = p->Nw;
  out->N = p->N;
  out->nnz = p->nnz;
  out->max_cover = p->max_cover;
  out->device = p->device;
  out->run = p->run;
  out->R = p->R;
  out->origins = p->origins.data();
  out->tile_tok = p->tile_tok.data();
  out->slot_pos = p->slot_pos.data();
  out->tok_ptr = p->tok_ptr.data();
  out->tok_ent = p->tok_ent.data();
  out->wbar = p->wbar.data();
  return TS_OK;
}

void ts_plan_destroy(ts_plan_t p) {
  if (!p) return;
  if (p->device < 0) {
    delete p;
    return;
  }
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(p->device);
  cudaFree(p->d_tok_ptr);
  cudaFree(p->d_tok_ent);
  cudaFree(p->d_wbar);
  cudaFree(p->d_rowmap);
  cudaFree(p->d_pos_shared);
  cudaFree(p->d_pos_tiled);
  if (prev >= 0) cudaSetDevice(prev);
  delete p;
}

ts_status ts_workspace_size(ts_plan_t p, const ts_model_desc* m, int L, int k, size_t* bytes) {
  if (!p || !bytes) return fail(TS_ERR_INVALID_ARG, "NULL argument");
  TS_TRY(check_model(m));
  if (L < 0 || k < 0 || k > L) return fail(TS_ERR_INVALID_ARG, "need L >= 0 and 0 <= k <= L");
  *bytes = layout(p, m, L > 0, nullptr).bytes;
  return TS_OK;
}

ts_status ts_block_tiled(ts_plan_t p, const ts_model_desc* m, const ts_layer_weights* w, void* X, void* ws,
                         size_t ws_bytes, void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  TS_TRY(check_weights(m, w));
  if (!X || !aligned16(X)) return fail(TS_ERR_INVALID_ARG, "X must be a 16-byte aligned device pointer");
  Workspace W;
  TS_TRY(check_ws(p, m, false, ws, ws_bytes, &W));
  return layer_tiled(p, m, w, X, W, static_cast<cudaStream_t>(stream));
}

ts_status ts_block_shared(ts_plan_t p, const ts_model_desc* m, const ts_layer_weights* w, void* S, void* ws,
                          size_t ws_bytes, void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  TS_TRY(check_weights(m, w));
  if (!S || !aligned16(S)) return fail(TS_ERR_INVALID_ARG, "S must be a 16-byte aligned device pointer");
  Workspace W;
  TS_TRY(check_ws(p, m, false, ws, ws_bytes, &W));
  return layer_shared(p, m, w, S, W, static_cast<cudaStream_t>(stream));
}

ts_status ts_block_partial(ts_plan_t p, const ts_model_desc* m, const ts_layer_weights* w, unsigned shared_ops,
                           void* X, void* ws, size_t ws_bytes, void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  TS_TRY(check_weights(m, w));
  if (shared_ops & ~static_cast<unsigned>(TS_SHARE_QKV | TS_SHARE_OUT | TS_SHARE_MLP))
    return fail(TS_ERR_INVALID_ARG, "unknown shared operations 0x%x", shared_ops);
  if (!X || !aligned16(X)) return fail(TS_ERR_INVALID_ARG, "X must be a 16-byte aligned device pointer");
  Workspace W;
  TS_TRY(check_ws(p, m, false, ws, ws_bytes, &W));
  return layer_partial(p, m, w, shared_ops, X, W, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Shared layer with its scratch in a static device array (no allocation).
// ---------------------------------------------------------------------------
}  // extern "C"

static __device__ __align__(256) unsigned char g_noalloc_scratch[TS_NOALLOC_SCRATCH_BYTES];

// Device address of the static scratch in the current CUDA context.  The address
// belongs to a context (the module holding the array is loaded per context), so it
// is cached under the driver's unique context ID, which a process never reuses:
// a non-primary context, or a primary context recreated after a device reset,
// gets its own lookup.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static std::mutex g_noalloc_mu;
struct NoallocEntry {
  unsigned long long ctx_id;
  void* ptr;
};
static std::vector<NoallocEntry> g_noalloc_cache;

static ts_status current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess || !a ||
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess || !b)
      return fail(TS_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId not available");
    get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return fail(TS_ERR_CUDA, "no current CUDA context");
  if (get_id(ctx, id) != CUDA_SUCCESS) return fail(TS_ERR_CUDA, "cuCtxGetId failed");
  return TS_OK;
}

static ts_status noalloc_scratch(void** out) {
  int dev = -1;
  TS_CUDA_CHECK(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long id = 0;
  // A thread with no current context yet gets the device's primary context from
  // the runtime at the symbol lookup below; it is looked up (and cached) then.
  if (current_context_id(&id) == TS_OK) {
    for (const NoallocEntry& e : g_noalloc_cache)
      if (e.ctx_id == id) {
        *out = e.ptr;
        return TS_OK;
      }
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p)
    return fail(TS_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed on device %d: %s", dev,
                cudaGetErrorString(e));
  TS_TRY(current_context_id(&id));
  g_noalloc_cache.push_back({id, p});
  *out = p;
  return TS_OK;
}

extern "C" {

ts_status ts_block_shared_noalloc(ts_plan_t p, const ts_model_desc* m, const ts_layer_weights* w, void* S,
                                  void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  TS_TRY(check_weights(m, w));
  if (!S || !aligned16(S)) return fail(TS_ERR_INVALID_ARG, "S must be a 16-byte aligned device pointer");
  const size_t need = layout(p, m, false, nullptr, true).bytes;
  if (need > TS_NOALLOC_SCRATCH_BYTES)
    return fail(TS_ERR_WORKSPACE,
                "ts_block_shared_noalloc: this plan and model need %zu bytes of scratch, the static array holds %u; "
                "use ts_block_shared with a workspace",
                need, TS_NOALLOC_SCRATCH_BYTES);
  void* base = nullptr;
  TS_TRY(noalloc_scratch(&base));
  const Workspace W = layout(p, m, false, static_cast<char*>(base), true);
  // layer_shared reads the regions xn, qkv, o, a, h, rope (and q8, qs for e4m3)
  // and no others (not X, S or sm, which the shared-only layout leaves null)
  if (!W.xn || !W.qkv || !W.o || !W.a || !W.h || !W.rope || (m->dtype == TS_FP8_E4M3 && (!W.q8 || !W.qs)))
    return fail(TS_ERR_WORKSPACE, "ts_block_shared_noalloc: scratch layout incomplete");
  return layer_shared(p, m, w, S, W, static_cast<cudaStream_t>(stream));
}

ts_status ts_decode_stack(ts_plan_t p, const ts_model_desc* m, const ts_layer_weights* w, int L, int k, const void* S0,
                          const void* G0, void* out, void* ws, size_t ws_bytes, void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  if (!w) return fail(TS_ERR_INVALID_ARG, "weights are NULL");
  if (L < 1 || k < 0 || k > L) return fail(TS_ERR_INVALID_ARG, "need L >= 1 and 0 <= k <= L");
  for (int l = 0; l < L; ++l) TS_TRY(check_weights(m, w + l));
  if (!S0 || !G0 || !out || !aligned16(S0) || !aligned16(G0) || !aligned16(out))
    return fail(TS_ERR_INVALID_ARG, "S0, G0, out must be 16-byte aligned device pointers");
  Workspace W;
  TS_TRY(check_ws(p, m, true, ws, ws_bytes, &W));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t rb = static_cast<size_t>(m->d) * esize(m->dtype);
  if (k > 0) {
    TS_TRY(run_gather(p, m, S0, G0, W.X, st));
    for (int l = 0; l < k; ++l) TS_TRY(layer_tiled(p, m, w + l, W.X, W, st));
    if (k == L) return run_merge("merge", p, m, W.X, p->U, out, nullptr, nullptr, st);
    TS_TRY(run_merge("merge", p, m, W.X, p->U + p->G, W.S, nullptr, nullptr, st));
  } else {
    TS_CUDA_CHECK(cudaMemcpyAsync(W.S, S0, rb * p->U, cudaMemcpyDeviceToDevice, st));
    TS_CUDA_CHECK(cudaMemcpyAsync(static_cast<char*>(W.S) + rb * p->U, G0, rb * p->G, cudaMemcpyDeviceToDevice, st));
  }
  for (int l = k; l < L; ++l) TS_TRY(layer_shared(p, m, w + l, W.S, W, st));
  TS_CUDA_CHECK(cudaMemcpyAsync(out, W.S, rb * p->U, cudaMemcpyDeviceToDevice, st));
  return TS_OK;
}

ts_status ts_quantize_rows_e4m3(const void* x, int rows, int cols, void* q, float* scale, void* stream) {
  if (!x || !q || !scale) return fail(TS_ERR_INVALID_ARG, "NULL argument");
  if (rows < 0 || cols <= 0 || cols % 8) return fail(TS_ERR_INVALID_ARG, "need rows >= 0, cols %% 8 == 0");
  if (!aligned16(x) || !aligned16(q) || !aligned16(scale)) return fail(TS_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  return run_quantize(x, rows, cols, static_cast<uint8_t*>(q), scale, static_cast<cudaStream_t>(stream));
}

ts_status ts_device_status(void) {
  int v = 0;
  TS_CUDA_CHECK(cudaDeviceSynchronize());
  TS_CUDA_CHECK(cudaMemcpyFromSymbol(&v, ts::g_status, sizeof(int)));
  const int zero = 0;
  TS_CUDA_CHECK(cudaMemcpyToSymbol(ts::g_status, &zero, sizeof(int)));
  if (v == 0) return TS_OK;
  return fail(static_cast<ts_status>(v), "device status %d", v);
}

ts_status ts_selftest_bounded_wait(long long limit_ns, int* done, void* stream) {
  if (!done || limit_ns <= 0 || limit_ns > 1000000000LL)
    return fail(TS_ERR_INVALID_ARG, "need done != NULL and 0 < limit_ns <= 1e9");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ts::wait_selftest_kernel<<<1, 1, 0, st>>>(static_cast<uint64_t>(limit_ns), done);
  TS_CUDA_CHECK(cudaGetLastError());
  return TS_OK;
}

// ---------------------------------------------------------------------------
// op-level entry points (include/tileshare_ops.h)
// ---------------------------------------------------------------------------
ts_status ts_op_layernorm(const ts_model_desc* m, const void* x, int rows, const float* g, const float* b, void* y,
                          void* stream) {
  TS_TRY(check_model(m));
  const bool rms = m->block == TS_BLOCK_RMS_SWIGLU;
  if (!x || !y || !g || (!b && !rms) || rows < 0) return fail(TS_ERR_INVALID_ARG, "bad argument");
  if (!aligned16(x) || !aligned16(y) || !aligned16(g) || (b && !aligned16(b))) return fail(TS_ERR_INVALID_ARG, "alignment");
  return run_layernorm(m, x, rows, g, b, y, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

ts_status ts_op_linear(const ts_model_desc* m, const void* x, int rows, int K, const void* W, const float* w_scale,
                       int N, const float* bias, ts_epilogue epi, void* y, void* scratch, void* stream) {
  TS_TRY(check_model(m));
  if (!x || !W || !y || !bias || rows < 0 || K <= 0 || N <= 0) return fail(TS_ERR_INVALID_ARG, "bad argument");
  if (!aligned16(x) || !aligned16(W) || !aligned16(y) || !aligned16(bias)) return fail(TS_ERR_INVALID_ARG, "alignment");
  if (epi != TS_EPI_BIAS && epi != TS_EPI_BIAS_GELU && epi != TS_EPI_BIAS_RESID && epi != TS_EPI_BIAS_SWIGLU)
    return fail(TS_ERR_INVALID_ARG, "unknown epilogue");
  const int e = epi == TS_EPI_BIAS        ? ts::EPI_BIAS
                : epi == TS_EPI_BIAS_GELU ? ts::EPI_GELU
                : epi == TS_EPI_BIAS_RESID ? ts::EPI_RESID
                                           : ts::EPI_SWIGLU;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (m->dtype == TS_F32)
    return run_gemm_f32("linear", e, static_cast<const float*>(x), static_cast<const float*>(W), rows, N, K, bias,
                        static_cast<float*>(y), st);
  if (m->dtype == TS_FP8_E4M3) {
    if (!scratch || !aligned16(scratch) || !w_scale) return fail(TS_ERR_INVALID_ARG, "e4m3 linear needs scratch and w_scale");
    uint8_t* q8 = static_cast<uint8_t*>(scratch);
    float* qs = reinterpret_cast<float*>(q8 + align256(static_cast<size_t>(rows) * K));
    TS_TRY(run_quantize(x, rows, K, q8, qs, st));
    return run_gemm_tc("linear", m, e, q8, qs, W, w_scale, rows, N, K, bias, static_cast<bf16*>(y), nullptr, nullptr, st);
  }
  return run_gemm_tc("linear", m, e, x, nullptr, W, nullptr, rows, N, K, bias, static_cast<bf16*>(y), nullptr, nullptr, st);
}

ts_status ts_op_qkv(ts_plan_t p, const ts_model_desc* m, const ts_layer_weights* w, ts_rows_mode mode,
                    const void* state, void* qkv, void* scratch, void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  TS_TRY(check_weights(m, w));
  if (!state || !qkv || !scratch || !aligned16(state) || !aligned16(qkv) || !aligned16(scratch))
    return fail(TS_ERR_INVALID_ARG, "bad argument");
  const bool shared = mode == TS_ROWS_SHARED;
  const size_t rows = shared ? p->U + p->G : static_cast<size_t>(p->T) * p->N;
  Workspace ws{};
  ws.xn = scratch;
  ws.q8 = static_cast<uint8_t*>(scratch) + align256(rows * m->d * esize(m->dtype));
  ws.qs = reinterpret_cast<float*>(ws.q8 + align256(rows * m->d));
  ws.rope = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(ws.qs) + align256(rows * 4));
  return run_qkv(p, m, w, shared, state, qkv, ws, static_cast<cudaStream_t>(stream));
}

ts_status ts_op_attention(ts_plan_t p, const ts_model_desc* m, ts_rows_mode mode, const void* qkv, void* O,
                          void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  if (!qkv || !O || !aligned16(qkv) || !aligned16(O)) return fail(TS_ERR_INVALID_ARG, "bad argument");
  return run_attention(p, m, mode == TS_ROWS_SHARED, qkv, O, static_cast<cudaStream_t>(stream));
}

ts_status ts_op_merge(ts_plan_t p, const ts_model_desc* m, const void* P, int rows, void* A, void* stream) {
  TS_TRY(check_plan(p));
  TS_TRY(check_model(m));
  if (!P || !A || !aligned16(P) || !aligned16(A)) return fail(TS_ERR_INVALID_ARG, "bad argument");
  if (rows != p->U && rows != p->U + p->G) return fail(TS_ERR_INVALID_ARG, "rows must be U or U + T*R");
  return run_merge("merge", p, m, P, rows, A, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
