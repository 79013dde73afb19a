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

// x / scale rounded to fp32 by round-to-odd: the quotient is formed by IEEE fp64 division
// (correctly rounded), truncated to fp32, and the last significand bit is set when the
// truncation dropped anything.  Rounding that fp32 value once more to nearest at 4
// significant bits (E4M3) gives the nearest E4M3 value of the fp64 quotient -- no double
// rounding -- because 24 >= 4 + 2 (round-to-odd: S. Boldo, G. Melquiond, "Emulation of
// FMA and correctly rounded sums: proved algorithms using rounding to odd", IEEE Trans.
// Computers 57(4), 2008).  Magnitudes past the fp32 range truncate to FLT_MAX, which the
// saturating conversion maps to 448 like any other value past 448.
__device__ __forceinline__ float div_to_f32_odd(float x, double scale) {
  const double q = (double)x / scale;
  float f = __double2float_rz(q);
  if ((double)f != q) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f;
}

// Eight fp32 values -> eight cache codes E4M3(x / scale) (nearest, ties to even, saturating
// at +-448), in order: the quotient of the value and the cache's scale, not of the value
// and a rounded reciprocal, so a code matches the nearest code of the exact quotient at any
// finite positive scale.
__device__ __forceinline__ uint2 f32x8_to_e4m3_div(const float (&x)[8], float scale) {
  const double s = (double)scale;
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = __nv_cvt_float2_to_fp8x2(
        make_float2(div_to_f32_odd(x[2 * i], s), div_to_f32_odd(x[2 * i + 1], s)),
        __NV_SATFINITE, __NV_E4M3);
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
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

// 2^x on the special-function unit (flushes subnormal results to zero; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace beam
