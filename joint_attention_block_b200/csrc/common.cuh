// Device helpers shared by the sm_100a kernels: bf16 packing, mbarriers with
// bounded waits, TMA tiled loads, tcgen05 (TMEM alloc, MMA, commit, ld/st) and
// the shared-memory matrix descriptors the tensor cores read.
//
// Every wait here is bounded by wall time (%globaltimer).  A wait that runs out
// records where it gave up in the library's device error word and returns
// false; callers then leave their loops, drain what they issued and free TMEM,
// so a stuck pipeline ends the kernel with an error status instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

#define JAB_DEVICE __device__ __forceinline__

namespace jab {

// ------------------------------------------------------------------ misc

// Programmatic dependent launch (see launch_pdl): wait for the previous kernel on the stream,
// then let the next one launch.
JAB_DEVICE void pdl_wait_then_release() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

JAB_DEVICE uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

JAB_DEVICE uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Record an error code (first one wins) in the library's device error word.
// Bits 0..11: which wait; bits 12..15: CTA rank in its cluster; bits 16..31: k-block
// or loop index where it gave up (see where_code()).
JAB_DEVICE void record_error(uint32_t* err, uint32_t code) {
  if (err != nullptr) atomicCAS(err, 0u, code);
}

JAB_DEVICE uint32_t where_code(uint32_t where, uint32_t rank, uint32_t index) {
  return (where & 0xFFFu) | ((rank & 0xFu) << 12) | ((index < 0xFFFFu ? index : 0xFFFFu) << 16);
}

JAB_DEVICE float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
JAB_DEVICE float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Two fp32 -> packed bf16x2 (round to nearest even), lo in the low half.
JAB_DEVICE uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 -> packed f16x2 (round to nearest even, saturating to +-65504), lo in the low half.
JAB_DEVICE uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

JAB_DEVICE float f16_lo(uint32_t v) {
  float f;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(f) : "r"(v));
  return f;
}
JAB_DEVICE float f16_hi(uint32_t v) {
  float f;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(f) : "r"(v));
  return f;
}

template <int F>
JAB_DEVICE uint32_t pack2(float lo, float hi) {
  if constexpr (F == FMT_F16) return pack_f16x2(lo, hi);
  else return pack_bf16x2(lo, hi);
}
template <int F>
JAB_DEVICE float unpack_lo(uint32_t v) {
  if constexpr (F == FMT_F16) return f16_lo(v);
  else return bf16_lo(v);
}
template <int F>
JAB_DEVICE float unpack_hi(uint32_t v) {
  if constexpr (F == FMT_F16) return f16_hi(v);
  else return bf16_hi(v);
}

// Load 8 consecutive activations of format F (16-bit: one 16-byte vector; f32: two).
template <int F>
JAB_DEVICE void load8(const void* base, int64_t idx8, float (&v)[8]) {
  if constexpr (F == FMT_F32) {
    const float4 a = reinterpret_cast<const float4*>(base)[2 * idx8];
    const float4 b = reinterpret_cast<const float4*>(base)[2 * idx8 + 1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 a = reinterpret_cast<const uint4*>(base)[idx8];
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&a);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = unpack_lo<F>(w[k]);
      v[2 * k + 1] = unpack_hi<F>(w[k]);
    }
  }
}

// Store 8 consecutive values in format F.
template <int F>
JAB_DEVICE void store8(void* base, int64_t idx8, const float (&v)[8]) {
  if constexpr (F == FMT_F32) {
    reinterpret_cast<float4*>(base)[2 * idx8] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(base)[2 * idx8 + 1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 o;
    o.x = pack2<F>(v[0], v[1]);
    o.y = pack2<F>(v[2], v[3]);
    o.z = pack2<F>(v[4], v[5]);
    o.w = pack2<F>(v[6], v[7]);
    reinterpret_cast<uint4*>(base)[idx8] = o;
  }
}

// Packed fp32 pair arithmetic (sm_100 f32x2 forms): one instruction for two lanes of work.
JAB_DEVICE float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
JAB_DEVICE float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

JAB_DEVICE float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

JAB_DEVICE float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

JAB_DEVICE float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU, exact form, on a pair of values: x Phi(x) with Phi the standard normal CDF, through
// x Phi(x) = max(x, 0) - |x| Phi(-|x|) and Abramowitz & Stegun, Handbook of Mathematical
// Functions, formula 7.1.26: erfc(z) = (a1 t + ... + a5 t^5) exp(-z^2) + e(z), t = 1 / (1 + p z),
// |e(z)| <= 1.5e-7 for z >= 0, z = |x| / sqrt 2 (the coefficients below are halved so that the
// sum is Phi(-|x|)).  The reciprocal t and exp2 run on the MUFU unit (rcp.approx and
// ex2.approx, about one fp32 ulp each), the polynomial and the rest on the FMA pipe in packed
// pairs; taking t by three Newton steps on the FMA pipe instead measured 1 % slower in the MLP
// up-projection, whose epilogue is otherwise FMA-issue-bound.  Branch-free; huge |x| gives x
// (x >= 0) or 0 (x < 0).
JAB_DEVICE float2 gelu_erf_pair(float2 x) {
  constexpr float kp = 0.3275911f * 0.7071067811865476f;
  constexpr float a1 = 0.5f * 0.254829592f, a2 = 0.5f * -0.284496736f, a3 = 0.5f * 1.421413741f,
                  a4 = 0.5f * -1.453152027f, a5 = 0.5f * 1.061405429f;
  const float2 nax = make_float2(__uint_as_float(__float_as_uint(x.x) | 0x80000000u),
                                 __uint_as_float(__float_as_uint(x.y) | 0x80000000u));  // -|x|
  const float2 nd = fma2(nax, make_float2(kp, kp), make_float2(-1.f, -1.f));           // -(1 + p z)
  const float2 y = make_float2(-rcp_approx(nd.x), -rcp_approx(nd.y));  // t = 1 / (1 + p z)
  float2 q = fma2(make_float2(a5, a5), y, make_float2(a4, a4));
  q = fma2(q, y, make_float2(a3, a3));
  q = fma2(q, y, make_float2(a2, a2));
  q = fma2(q, y, make_float2(a1, a1));
  q = mul2(q, y);
  const float2 xx = mul2(mul2(x, make_float2(-0.7213475204444817f, -0.7213475204444817f)), x);  // -x^2 log2(e) / 2
  const float2 e = make_float2(ex2_approx(xx.x), ex2_approx(xx.y));                     // exp(-x^2 / 2)
  return fma2(mul2(nax, e), q, make_float2(fmaxf(x.x, 0.f), fmaxf(x.y, 0.f)));
}

// e4m3 bytes -> bf16, exactly, for all finite codes.
//
// Each byte b is widened to a 16-bit lane whose high byte repeats b's sign
// (prmt sign-replicate mode); shifting the lane left by 4 and masking
// 0x87F0 leaves the sign at bit 15 and the 7 exponent+mantissa bits at bits
// 4..10, which as a bf16 is exactly value(b) * 2^-120 (e4m3 subnormals become
// bf16 subnormals with the same ratio).  A bf16 multiply by 2^120 then gives
// value(b).  The two NaN codes (0x7F, 0xFF) come out as +-480; FP8 weight
// files carry no NaN.
JAB_DEVICE void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  uint32_t a, b;
  asm("prmt.b32 %0, %1, 0, 0x9180;" : "=r"(a) : "r"(w));
  asm("prmt.b32 %0, %1, 0, 0xB3A2;" : "=r"(b) : "r"(w));
  a = (a << 4) & 0x87F087F0u;
  b = (b << 4) & 0x87F087F0u;
  const uint32_t two120 = 0x7B807B80u;  // bf16x2 (2^120, 2^120)
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(two120));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(two120));
}

// e4m3 -> f16 with the hardware pair conversion (exact: e4m3 is a subset of f16).
// Measured on B200: ~46 elements/clk/SM, against ~28 for an integer widening like the bf16
// one above (shift by 7, mask 0xBF80, multiply by 2^8 in f16).
JAB_DEVICE void e4m3x4_to_f16x4_cvt(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

template <bool F16>
JAB_DEVICE void e4m3x4_to_16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  if constexpr (F16) e4m3x4_to_f16x4_cvt(w, lo, hi);
  else e4m3x4_to_bf16x4(w, lo, hi);
}

// ------------------------------------------------------------------ mbarrier

JAB_DEVICE void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

JAB_DEVICE void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

JAB_DEVICE void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

JAB_DEVICE void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

JAB_DEVICE bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up after the
// guard's wall-time limit, or, unless `drain` is set, as soon as another role of
// the CTA has aborted.  Drains (waits for copies / MMAs this CTA issued) ignore
// the abort flag so that nothing is left in flight when the CTA exits.
JAB_DEVICE bool mbar_wait(uint64_t* bar, uint32_t parity, const KernelGuard& g, volatile uint32_t* abort_flag,
                          uint32_t where, bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (((++spins) & 63u) == 0) {
      if (!drain && *abort_flag) return false;
      if (!drain && g.err != nullptr && *reinterpret_cast<volatile uint32_t*>(g.err) != 0u) {
        *abort_flag = 1u;  // another CTA already failed: give up at once
        return false;
      }
      if (global_timer_ns() - t0 > g.timeout_ns) {
        *abort_flag = 1u;
        record_error(g.err, where);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------ CTA pairs (clusters of 2)

JAB_DEVICE uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory object in CTA `rank` of the cluster.
JAB_DEVICE uint32_t mapa_shared(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}

// Arrive on an mbarrier given by its shared::cluster address (possibly in the peer
// CTA), with the default (CTA-scope release) semantics: a cluster-scope release
// would make the thread wait for all of its outstanding memory operations.
JAB_DEVICE void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

JAB_DEVICE void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (given by its shared::cluster address).
JAB_DEVICE void tma_load_2d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster_addr, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}

// The 3D form of tma_load_2d_pair.
JAB_DEVICE void tma_load_3d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster_addr, int32_t x, int32_t y,
                                 int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster_addr), "r"(x), "r"(y), "r"(z)
      : "memory");
}

JAB_DEVICE void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

JAB_DEVICE void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Pair MMA issued by the leader CTA with both operands in shared memory: D (M=256
// over both CTAs' TMEM) (+)= A (128 rows in each CTA) * B (N/2 rows in each CTA)^T.
// Both descriptors give the same shared-memory offsets in the two CTAs.
JAB_DEVICE void mma_f16kind_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Pair MMA issued by the leader CTA with A read from tensor memory: D (M=256 over both
// CTAs' TMEM) (+)= A (128 rows in each CTA's TMEM at the same address) * B (N/2 rows in
// each CTA's shared memory)^T.
JAB_DEVICE void mma_f16kind_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the mbarrier at this shared-memory offset in every CTA of `cta_mask`
// once all pair MMAs issued so far by this thread are done.
JAB_DEVICE void mma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// ------------------------------------------------------------------ proxies / fences

JAB_DEVICE void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

JAB_DEVICE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
JAB_DEVICE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ------------------------------------------------------------------ TMA

JAB_DEVICE void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// Bring the box at (x, y) of a tensor map into L2 ahead of its load (no shared memory, no barrier).
JAB_DEVICE void tma_prefetch_l2_2d(const CUtensorMap* m, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y)
               : "memory");
}

JAB_DEVICE void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

JAB_DEVICE void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

JAB_DEVICE void tma_store_3d(const CUtensorMap* m, const void* src, int32_t x, int32_t y, int32_t z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
// The same store with an L2 cache-policy hint (see l2_evict_first_policy).
JAB_DEVICE void tma_store_3d_hint(const CUtensorMap* m, const void* src, int32_t x, int32_t y, int32_t z,
                                  uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group.L2::cache_hint [%0, {%2, %3, %4}], [%1], %5;" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}
// L2 policy marking lines as the first to evict: for output streams larger than L2 that
// would otherwise push out operands the same kernel still re-reads.
JAB_DEVICE uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
JAB_DEVICE void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed bulk groups still read shared memory.
template <int N>
JAB_DEVICE void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ tcgen05

// Allocate `ncols` TMEM columns (power of two >= 32); the whole warp calls it.
JAB_DEVICE void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

JAB_DEVICE void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// K-major (or MN-major) shared-memory matrix descriptor with 128-byte swizzle.
// start/lbo/sbo are byte quantities; bits 46..47 hold the fixed version 1.
JAB_DEVICE uint64_t smem_desc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;  // 128-byte swizzle
  return d;
}

// The same with 64-byte swizzle (rows of 64 bytes; the pattern repeats every 512 bytes).
JAB_DEVICE uint64_t smem_desc_sw64(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 4ull << 61;  // 64-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16 with fp32 accumulation; A and B are both
// bf16 (f16 = false) or both f16 (f16 = true).
__host__ __device__ constexpr uint32_t idesc_f16kind(int M, int N, bool f16, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                      // D format f32
         | (f16 ? 0u : (1u << 7))                       // A: 0 = f16, 1 = bf16
         | (f16 ? 0u : (1u << 10))                      // B: 0 = f16, 1 = bf16
         | (a_mn_major ? (1u << 15) : 0u) | (b_mn_major ? (1u << 16) : 0u) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
JAB_DEVICE void mma_f16kind_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A (M x 16, 16-bit, one row per TMEM lane, two
// elements per 32-bit column) is read from tensor memory.
JAB_DEVICE void mma_f16kind_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
JAB_DEVICE void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base + i), columns col..col+31.
JAB_DEVICE void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

JAB_DEVICE void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns.
JAB_DEVICE void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

JAB_DEVICE void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
JAB_DEVICE void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Wait for this thread's TMEM loads, then pass `r` through an empty asm so that no use of
// the loaded registers can be scheduled above the wait (they are written asynchronously).
JAB_DEVICE void tmem_ld_wait_regs(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
  asm volatile("" : "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

JAB_DEVICE uint32_t warp_id() { return threadIdx.x >> 5; }
JAB_DEVICE uint32_t lane_id() { return threadIdx.x & 31u; }

}  // namespace jab
