// Device-side building blocks shared by the KroQuant kernels (sm_100a).
//
//  * TMA / mbarrier wrappers (inline PTX) with bounded waits;
//  * bf16 -> fp32 widening;
//  * the Kronecker butterfly: T = A_1 (x) ... (x) A_5 applied to one 32-element
//    block held in registers as 16 float2 pairs (x[2k], x[2k+1]);
//  * the MXFP4 block encoder (amax, E8M0 byte, E2M1 nibbles).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kq {

// ---------------------------------------------------------------------------
// bounded waiting
// ---------------------------------------------------------------------------
// A wait that runs longer than this gives up (about one second).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async proxy (TMA) and the CTA.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of the barrier; false if it did not complete within
// limit_ns (default kWaitLimitNs).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2-D tiled TMA load global -> shared, completion signalled on `bar`.
// No cluster multicast: every CTA loads its own tiles of this GPU's memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Asynchronous 4-byte global -> shared copy (cp.async); all copies a thread
// issued are awaited with cp_async_wait_all().
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// 3-D tiled TMA load global -> shared (coordinates innermost first).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, int c0, int c1, int c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// L2 prefetch of a 3-D tile (no shared memory, no completion signal).
__device__ __forceinline__ void tma_prefetch_l2_3d(const void* tmap, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

// L2 prefetch of the 128-byte line holding p (a hint: changes no memory).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p) : "memory");
}

// Programmatic dependent launch (PTX griddepcontrol).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait_predecessor() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
// Two bf16 packed in a 32-bit word (element 2k low, 2k+1 high) -> exact fp32.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// ---------------------------------------------------------------------------
// Kronecker butterfly
// ---------------------------------------------------------------------------
// One 2x2 factor [[c.x, c.y], [c.z, c.w]] per Kronecker position; factor m
// acts on bit (4 - m) of the element index.  v[k] holds elements (2k, 2k+1),
// so index bits 1..4 are bits 0..3 of k and factors 0..3 pair whole float2s
// (packed f32x2 FMA); factor 4 acts on bit 0, inside each float2.
__device__ __forceinline__ void butterfly32(float2 (&v)[16], const float4 (&A)[5]) {
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int h = 1 << (3 - m);
    const float2 a00 = make_float2(A[m].x, A[m].x);
    const float2 a01 = make_float2(A[m].y, A[m].y);
    const float2 a10 = make_float2(A[m].z, A[m].z);
    const float2 a11 = make_float2(A[m].w, A[m].w);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k & h) continue;
      const float2 lo = v[k], hi = v[k + h];
      v[k] = __ffma2_rn(a01, hi, __fmul2_rn(a00, lo));
      v[k + h] = __ffma2_rn(a11, hi, __fmul2_rn(a10, lo));
    }
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float x0 = v[k].x, x1 = v[k].y;
    v[k].x = __fmaf_rn(A[4].y, x1, __fmul_rn(A[4].x, x0));
    v[k].y = __fmaf_rn(A[4].w, x1, __fmul_rn(A[4].z, x0));
  }
}

// Factor (A00, A01, A10, A11) of A = L U, L = [[1,0],[a,1]], U = [[u,b],[0,1/u]].
// The factor is defined (and invertible) only for u != 0 and finite a, b, u.
__device__ __forceinline__ bool lu_params_bad(float a, float b, float u) {
  return u == 0.0f || !isfinite(a) || !isfinite(b) || !isfinite(u);
}

__device__ __forceinline__ float4 lu_factor(float a, float b, float u) {
  const float inv_u = 1.0f / u;
  return make_float4(u, b, __fmul_rn(a, u), __fmaf_rn(a, b, inv_u));
}

// Transposed inverse of that factor: A^{-1} = [[ab+1/u, -b], [-au, u]], so
// A^{-T} = [[ab+1/u, -au], [-b, u]].  Applying (x)_m A_m^{-T} to a weight-row
// block w computes (w T^{-1}).
__device__ __forceinline__ float4 lu_factor_inv_t(float a, float b, float u) {
  const float inv_u = 1.0f / u;
  return make_float4(__fmaf_rn(a, b, inv_u), -__fmul_rn(a, u), -b, u);
}

// ---------------------------------------------------------------------------
// MXFP4 encoding of one 32-element block
// ---------------------------------------------------------------------------
// max(|a|, |b|) and max(|a|, |b|, |c|), NaN-propagating (a NaN anywhere gives NaN).
__device__ __forceinline__ float absmax2(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(fabsf(a)), "f"(fabsf(b)));
  return r;
}

__device__ __forceinline__ float absmax3(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
  return r;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Largest magnitude of 32 values: a 3-input max tree of 16 instructions.
__device__ __forceinline__ float block_absmax(const float2 (&v)[16]) {
  const float* f = reinterpret_cast<const float*>(v);
  float m[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) m[i] = absmax3(f[3 * i], f[3 * i + 1], f[3 * i + 2]);
  m[10] = absmax2(f[30], f[31]);
  const float q0 = max3(m[0], m[1], m[2]), q1 = max3(m[3], m[4], m[5]);
  const float q2 = max3(m[6], m[7], m[8]), q3 = max3(m[9], m[10], q0);
  return max3(q1, q2, q3);
}

// E8M0 byte of a block with largest magnitude `amax` (NaN if any element is
// NaN): floor(log2 amax) - 2 + 127 read from the exponent field, clamped at 0;
// NaN / Inf give 0xFF.
__device__ __forceinline__ uint32_t e8m0_byte(float amax) {
  const uint32_t E = __float_as_uint(amax) >> 23;
  if (E == 255u) return 255u;
  return E > 2u ? E - 2u : 0u;
}

// 2^(127 - byte) for byte in [0, 252] (all scale bytes of finite fp32 blocks).
__device__ __forceinline__ float inv_scale_from_byte(uint32_t byte) {
  const uint32_t b = byte > 252u ? 252u : byte;
  return __uint_as_float((254u - b) << 23);
}

// Four pairs -> 8 E2M1 nibbles in one word; element 2i of the pair list lands
// in nibble 2i (low nibble first).  Each pair goes through the PTX conversion
// cvt.rn.satfinite.e2m1x2.f32 (round to nearest even, saturating to +-6),
// whose first source lands in the upper nibble of the byte, so a pair (x, y)
// is passed as (y, x).  The four bytes are packed by a vector mov (byte 0
// first): ptxas then keeps them in byte lanes instead of widening each one to
// a word and shifting it into place.
__device__ __forceinline__ uint32_t e2m1x8(float2 p0, float2 p1, float2 p2, float2 p3) {
  uint32_t w;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(w)
      : "f"(p0.x), "f"(p0.y), "f"(p1.x), "f"(p1.y), "f"(p2.x), "f"(p2.y), "f"(p3.x), "f"(p3.y));
  return w;
}

// Encode 32 values: returns the scale byte and writes 16 code bytes to `out`.
__device__ __forceinline__ uint32_t mxfp4_encode32(const float2 (&v)[16], uint4& out) {
  const uint32_t byte = e8m0_byte(block_absmax(v));
  const float sc = inv_scale_from_byte(byte);
  const float2 sc2 = make_float2(sc, sc);
  float2 r[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) r[k] = __fmul2_rn(v[k], sc2);
  out.x = e2m1x8(r[0], r[1], r[2], r[3]);
  out.y = e2m1x8(r[4], r[5], r[6], r[7]);
  out.z = e2m1x8(r[8], r[9], r[10], r[11]);
  out.w = e2m1x8(r[12], r[13], r[14], r[15]);
  return byte;
}

}  // namespace kq
