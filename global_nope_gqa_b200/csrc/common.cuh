// common.cuh -- small device helpers shared by the attention-core kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "beam_attn.h"

namespace beam {

constexpr int kHq = 48;      // query heads
constexpr int kHkv = 8;      // KV heads
constexpr int kGroup = 6;    // query heads per KV head
constexpr int kD = 128;      // head axis
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void set_status(int32_t *status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Round two floats to bf16 (nearest, ties to even) and pack: lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Scalable-softmax factor a(p) = (1 + p/base)^expo for the one-based position p.
__device__ __forceinline__ float ssmax_factor(int64_t p, float base, float expo) {
  return exp2f(expo * log2f(1.0f + (float)p / base));
}

// ---- cp.async (16-byte, L2 only) -------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void *gptr, bool valid) {
  int src_bytes = valid ? 16 : 0;  // 0: nothing is read, the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr), "l"(gptr),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- warp-level MMA (m16n8k16, bf16 in, fp32 accumulate) -------------------
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Byte offset of 16-byte chunk `c` (0..15) of row `r` in a tile of 256-byte rows,
// XOR-swizzled so that eight consecutive rows at one chunk hit distinct banks.
__device__ __forceinline__ uint32_t swz256(int r, int c) {
  return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4));
}

// Two E4M3 codes (low byte first) -> fp16x2 (low half first); exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xFFFFu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Eight E4M3 codes (low byte first) -> their eight values as bf16, exactly (an E4M3 value
// has 4 significant bits and an exponent within bf16's range): the unscaled values an
// FP8 cache row holds, in the form the bf16 tensor-core kernels read.
__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(const uint2 codes) {
  const uint32_t pairs[4] = {codes.x & 0xFFFFu, codes.x >> 16, codes.y & 0xFFFFu, codes.y >> 16};
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t h = e4m3x2_to_f16x2(pairs[i]);
    w[i] = pack_bf16(__half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu))),
                     __half2float(__ushort_as_half((unsigned short)(h >> 16))));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// The nearest E4M3 code of a double, ties to the even code, magnitudes from 448 up
// saturating to 448 (OCP E4M3: sign, 4 exponent bits with bias 7, 3 fraction bits,
// subnormals m * 2^-9, no infinities; S.1111.111 is NaN and never produced).  Written from
// that definition in integer arithmetic on the double's 53-bit significand, so the one
// rounding sees every bit of its input.
__device__ __forceinline__ uint32_t e4m3_rne(double q) {
  const uint64_t bits = (uint64_t)__double_as_longlong(q);
  const uint32_t sign = (uint32_t)(bits >> 63) << 7;
  const uint64_t mag = bits & 0x7FFFFFFFFFFFFFFFull;
  if (mag >= 0x407C000000000000ull) return sign | 0x7Eu;   // |q| >= 448 = 1.75 * 2^8
  const int e = (int)(mag >> 52) - 1023;                    // |q| in [2^e, 2^(e + 1))
  if (e < -21) return sign;                                 // below 2^-11: rounds to zero
  const uint64_t sig = (1ull << 52) | (mag & ((1ull << 52) - 1));
  if (e >= -6) {   // a normal code: keep 3 fraction bits
    uint64_t m = sig >> 49;                                 // 8 .. 15
    const uint64_t rem = sig & ((1ull << 49) - 1), half = 1ull << 48;
    if (rem > half || (rem == half && (m & 1))) ++m;
    int ee = e;
    if (m == 16) { m = 8; ++ee; }                           // cannot pass 448 (checked above)
    return sign | ((uint32_t)(ee + 7) << 3) | (uint32_t)(m - 8);
  }
  // a subnormal code: |q| in units of 2^-9 (8 is the smallest normal, code 0x08)
  const int shift = 43 - e;                                 // 50 .. 64
  uint64_t m = shift >= 64 ? 0 : sig >> shift;
  const uint64_t rem = shift >= 64 ? sig : sig & ((1ull << shift) - 1);
  const uint64_t half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (m & 1))) ++m;
  return sign | (uint32_t)m;
}

// Eight fp32 values -> eight cache codes E4M3(x / scale) (nearest, ties to even, saturating
// at +-448), in order: the quotient of the value and the cache's scale, formed in fp64
// (IEEE division, exact to 53 bits), not the product with a rounded reciprocal, so a code
// is the nearest code of the quotient at any finite positive scale.
__device__ __forceinline__ uint2 f32x8_to_e4m3_div(const float (&x)[8], float scale) {
  const double s = (double)scale;
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) c[i] = e4m3_rne((double)x[i] / s);
  return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24),
                    c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

// Eight fp32 values -> eight E4M3 codes (value * mul, nearest, saturating), in order.  Used
// with power-of-two factors (the decode query's two-term split), where the product is exact.
__device__ __forceinline__ uint2 f32x8_to_e4m3(const float (&x)[8], float inv_scale) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = __nv_cvt_float2_to_fp8x2(make_float2(x[2 * i] * inv_scale, x[2 * i + 1] * inv_scale),
                                    __NV_SATFINITE, __NV_E4M3);
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization
// may start while the kernel before it in the stream is still running; pdl_wait() returns
// once that kernel has completed and its memory writes are visible (at once for a kernel
// launched without the attribute).  pdl_trigger() lets the next kernel's CTAs be scheduled
// as soon as every CTA of this one has issued it or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// 2^x on the special-function unit (flushes subnormal results to zero; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace beam
