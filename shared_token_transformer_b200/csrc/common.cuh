// common.cuh -- device helpers shared by the kernels of libtileshare.so (sm_100a).
//
// Thin wrappers over the PTX of the Blackwell asynchronous pipeline: mbarriers,
// TMA bulk tensor loads, tcgen05 MMA / TMEM, plus a device status word that bounded
// waits and device-side checks write instead of trapping.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace ts {

typedef __nv_bfloat16 bf16;

// Status word of the library on each device (0 = fine, else a ts_status code).
// Kernels never trap: a failed bounded wait or device check writes it and returns.
__device__ int g_status;

enum : int { kStatusDeviceCheck = 5, kStatusTimeout = 6 };

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

// Longest a pipeline wait may spin before the kernel gives up (ns of %globaltimer).
constexpr uint64_t kWaitLimitNs = 4000000000ull;

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel in the stream still runs.
// pdl_wait() blocks until that kernel has completed and its writes are visible;
// every such kernel calls it before touching activations (reads or writes).
// pdl_trigger() lets the next kernel begin its own prologue.  Both are no-ops
// for ordinary launches.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; gives up after
// limit_ns (kWaitLimitNs in the kernels), writes kStatusTimeout and returns false.
__device__ __noinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit_ns) {
      set_status(kStatusTimeout);
      return false;
    }
  }
}
// Fast path inline (one potentially blocking try_wait); the bounded loop is a call.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
#ifndef TS_MBAR_NOFAST
  if (mbar_try_wait(bar, parity)) return true;
#endif
  return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// Self-test of the bounded wait: one thread initialises an mbarrier that nothing
// arrives at and waits for it with a short limit; the wait must give up, write
// kStatusTimeout and let the kernel return.  `done` receives 1 (returned) and the
// wait's result.
__global__ void wait_selftest_kernel(uint64_t limit_ns, int* done) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  const bool ok = mbar_wait_for(b, 0, limit_ns);
  done[0] = 1;
  done[1] = ok ? 1 : 0;
}

// ----------------------------------------------------------------------------
// TMA (bulk tensor copies, no multicast)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled load of the box at (x = inner element index, y = row) into shared
// memory; completion is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Contiguous copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from global into shared memory; completion is signalled on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// 3-D tiled load of the box at (x = inner element index, y, z).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA, commit, loads
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// ----------------------------------------------------------------------------
// two-SM MMA pairs (tcgen05 cta_group::2): a cluster of two CTAs, the even one
// (rank 0) issuing the MMAs for both.  No TMA load here uses cluster multicast.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Arrive once on an mbarrier of another CTA of the cluster (address from cluster_map).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Tiled 2-D load by either CTA of a pair into its own shared memory, whose
// transaction bytes complete on `leader_bar`, the mbarrier of the even CTA.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* map, uint32_t leader_bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
      : "memory");
}
// Arrive once on `bar` in both CTAs of the pair when the MMAs issued so far are done.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  const uint16_t both = 0x3;
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
               "h"(both)
               : "memory");
}
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_mma_f8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D(tmem) (+)= A(smem desc) * B(smem desc)^T, bf16/f16 operands, fp32 accumulate.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Same with 8-bit float operands (e4m3 / e5m2), fp32 accumulate.
__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (lane quarter = warp % 4).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand tile stored with the
// 128-byte swizzle (rows of 128 bytes, 8-row atoms of 1024 bytes, atoms 1024-byte
// aligned): start address >> 4 in bits 0-13, leading byte offset (unused for this
// layout) 16 bytes, stride byte offset 1024 (between 8-row atoms) in bits 32-45,
// descriptor version 1 in bits 46-47, layout type 2 (128-byte swizzle) in bits
// 61-63.  Advancing the start address by 32 bytes steps K by 32 bytes inside the
// atom.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor: fp32 accumulator, A and B K-major, M = m (128, or 256
// for a two-SM pair), N = n.  a/b format: bf16 = 1 for kind::f16, e4m3 = 0 for
// kind::f8f6f4.
__host__ __device__ constexpr uint32_t idesc_make(uint32_t ab_format, int n, int m = 128) {
  return (1u << 4)                                // D format: f32
         | (ab_format << 7) | (ab_format << 10)   // A, B format
         | (static_cast<uint32_t>(n >> 3) << 17)  // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);    // M / 16
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ----------------------------------------------------------------------------
// small numeric helpers
// ----------------------------------------------------------------------------
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
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t splat_f32x2(float v) { return pack_f32x2(v, v); }

// Exact-erf GELU, 0.5 x (1 + erf(x / sqrt 2)).  erf by Abramowitz & Stegun,
// Handbook of Mathematical Functions, formula 7.1.26 (|error| <= 1.5e-7 for
// z >= 0, odd extension), evaluated with the approximate reciprocal and base-2
// exponential: about 2e-7 absolute on erf, far below the bf16 output rounding
// and the fp32 path's 1e-5 layer tolerance.
__device__ __forceinline__ float gelu_erf(float x) {
  const float z = fabsf(x) * 0.70710678118654752f;
  const float t = __fdividef(1.0f, fmaf(0.3275911f, z, 1.0f));
  float p = fmaf(1.061405429f, t, -1.453152027f);
  p = fmaf(p, t, 1.421413741f);
  p = fmaf(p, t, -0.284496736f);
  p = fmaf(p, t, 0.254829592f);
  const float e = ex2_approx(-1.4426950408889634f * z * z);
  const float erf_z = fmaf(-p * t, e, 1.0f);
  return 0.5f * x * (1.0f + copysignf(erf_z, x));
}
// gelu_erf of a pair of values (low = first) in packed f32x2 arithmetic: the same
// formula and the same two SFU operations per value, half the FMA-pipe
// instructions.  The bf16 GEMM epilogue, bound by its issue slots, uses it.
__device__ __forceinline__ uint64_t gelu_erf2(uint64_t x2) {
  const float x0 = lo_f32(x2), x1 = hi_f32(x2);
  const uint64_t z = mul_f32x2(pack_f32x2(fabsf(x0), fabsf(x1)), splat_f32x2(0.70710678118654752f));
  const uint64_t den = fma_f32x2(splat_f32x2(0.3275911f), z, splat_f32x2(1.0f));
  const uint64_t t = pack_f32x2(__fdividef(1.0f, lo_f32(den)), __fdividef(1.0f, hi_f32(den)));
  uint64_t p = fma_f32x2(splat_f32x2(1.061405429f), t, splat_f32x2(-1.453152027f));
  p = fma_f32x2(p, t, splat_f32x2(1.421413741f));
  p = fma_f32x2(p, t, splat_f32x2(-0.284496736f));
  p = fma_f32x2(p, t, splat_f32x2(0.254829592f));
  const uint64_t ea = mul_f32x2(mul_f32x2(z, z), splat_f32x2(-1.4426950408889634f));
  const uint64_t e = pack_f32x2(ex2_approx(lo_f32(ea)), ex2_approx(hi_f32(ea)));
  const uint64_t erf = fma_f32x2(mul_f32x2(p, t), pack_f32x2(-lo_f32(e), -hi_f32(e)), splat_f32x2(1.0f));
  const uint64_t s = pack_f32x2(copysignf(lo_f32(erf), x0), copysignf(hi_f32(erf), x1));
  return mul_f32x2(mul_f32x2(x2, splat_f32x2(0.5f)), add_f32x2(s, splat_f32x2(1.0f)));
}
// The same GELU with erf by Abramowitz & Stegun formula 7.1.28: for z >= 0,
// erf z = 1 - (1 + a1 z + a2 z^2 + ... + a6 z^6)^-16 with |error| <= 3e-7 (odd
// extension).  One approximate reciprocal and four squarings: a single SFU
// operation per value where 7.1.26 needs two.  Evaluated in fp32 it stays within
// 6e-7 of exact-erf GELU relative to max(1, |GELU|).  On a pair of values (low =
// first) in packed f32x2 arithmetic; the e4m3 GEMMs use it, since at twice the
// bf16 MMA rate their GELU epilogue is bound by the SFU and the issue slots.
__device__ __forceinline__ uint64_t gelu_erf_one_sfu2(uint64_t x2) {
  const float x0 = lo_f32(x2), x1 = hi_f32(x2);
  const uint64_t z = mul_f32x2(pack_f32x2(fabsf(x0), fabsf(x1)), splat_f32x2(0.70710678118654752f));
  uint64_t p = fma_f32x2(splat_f32x2(0.0000430638f), z, splat_f32x2(0.0002765672f));
  p = fma_f32x2(p, z, splat_f32x2(0.0001520143f));
  p = fma_f32x2(p, z, splat_f32x2(0.0092705272f));
  p = fma_f32x2(p, z, splat_f32x2(0.0422820123f));
  p = fma_f32x2(p, z, splat_f32x2(0.0705230784f));
  p = fma_f32x2(p, z, splat_f32x2(1.0f));
  uint64_t r = pack_f32x2(__fdividef(1.0f, lo_f32(p)), __fdividef(1.0f, hi_f32(p)));
  r = mul_f32x2(r, r);
  r = mul_f32x2(r, r);
  r = mul_f32x2(r, r);
  r = mul_f32x2(r, r);
  const uint64_t erf = add_f32x2(splat_f32x2(1.0f), pack_f32x2(-lo_f32(r), -hi_f32(r)));
  const uint64_t s = pack_f32x2(copysignf(lo_f32(erf), x0), copysignf(hi_f32(erf), x1));
  return mul_f32x2(mul_f32x2(x2, splat_f32x2(0.5f)), add_f32x2(s, splat_f32x2(1.0f)));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 8 bf16 <-> 8 floats through one 16-byte word
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 p = __bfloat1622float2(h[i]);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
  }
}
__device__ __forceinline__ uint4 f32_to_bf16x8(const float* f) {
  uint4 u;
  u.x = pack_bf16(f[0], f[1]);
  u.y = pack_bf16(f[2], f[3]);
  u.z = pack_bf16(f[4], f[5]);
  u.w = pack_bf16(f[6], f[7]);
  return u;
}

// Cosine / sine table of the RoPE angles of one plan and model: for axis a,
// coordinate p < G[a] and pair j < half[a], entry off[a] + p * half[a] + j holds
// (cos, sin) of p * base^(-j / half[a]), computed in double and rounded to float.
struct RopeTable {
  float2* cs;
  int G[3];
  int half[3];
  int off[3];
  int total;
  float base;
};

__device__ __forceinline__ void rope_table_fill(const RopeTable& rt, int e) {
  if (e >= rt.total) return;
  const int a = e >= rt.off[2] ? 2 : (e >= rt.off[1] ? 1 : 0);
  const int r = e - rt.off[a];
  const int p = r / rt.half[a], j = r % rt.half[a];
  const double theta = exp(-log(static_cast<double>(rt.base)) * j / rt.half[a]);
  double sn, cs;
  sincos(static_cast<double>(p) * theta, &sn, &cs);
  rt.cs[e] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
}

// two floats -> two e4m3 bytes, nearest-even, saturating at +-448
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float a, float b) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// Rotation angle pos * theta with theta given as a float pair (hi + lo): the
// product is split into a rounded part and its exact error so that the cosine
// and sine keep full float accuracy for coordinates in the hundreds.
__device__ __forceinline__ void rope_cos_sin(float pos, float th_hi, float th_lo, float& c, float& s) {
  const float a = pos * th_hi;
  const float err = fmaf(pos, th_hi, -a) + pos * th_lo;
  float sa, ca;
  sincosf(a, &sa, &ca);
  c = ca - err * sa;
  s = sa + err * ca;
}

}  // namespace ts
