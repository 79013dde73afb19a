// decode8.cuh -- split-K decode attention over an FP8 E4M3 KV cache, then the gate.
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax", section "KV memory": an
// FP8 cache halves the bytes a decode step streams (18 KiB per token over the nine
// global layers instead of 36 KiB).  The cache holds E4M3 codes of K^ / k_scale and
// V / v_scale (one float scale per cache tensor of a layer); the attention is the same as
// in decode.cuh.
//
// Same grid and split as the BF16 kernel: (split, KV head, sequence), 128 threads; each
// CTA prepares its group's six queries, the owner of the new token's slot writes the new
// key and value as codes, and the CTA streams its run of slots through a 4-stage cp.async
// ring of 64-slot tiles (64 x 128 bytes for K and for V; 16-byte chunks XOR-swizzled by
// row).  S = Q K^T runs on E4M3 MMAs (m16n8k32, fp32 accumulation) straight on the key
// codes, the six heads as M rows: each query row is split into two E4M3 terms,
// 16 q = hi + lo with lo = E4M3(16 q - hi), which keeps about 8 significant bits (bf16
// keeps 8), and both terms go into the same accumulator.  The output is formed transposed,
// O^T = V^T P^T, on fp16 m16n8k16 MMAs with d as M (eight 16-row tiles) and the heads as
// N (8 columns, 6 used), so no MMA row is padding: every E4M3 value is exact in fp16, so
// the value codes are widened to fp16 in registers, and P is fp16 (two E4M3 terms would
// not hold the small probabilities of a long context).  The score accumulator of a lane
// (head lane / 4, keys 2c + {0, 1} of an 8-key block, c = lane % 4) is exactly the P^T
// operand fragment the second MMA wants, so P never leaves registers.  k_scale / 16 joins
// the score scale, v_scale the partial output.
//
// Operand layout.  A dot product over d may visit d in any order as long as both
// operands use the same one, and a result row may sit anywhere as long as it is written
// back to its own d, so the fragments are laid out for wide shared-memory loads:
//   S = Q K^T: in k-step ks (of 4), MMA k-slot 4c + j (16 + 4c + j) of lane c = lane % 4 is
//     d = 32 c + 8 ks + j (+ 4), j < 4, so a lane reads its 32 bytes of a key row with two
//     16-byte loads and takes two words per k-step;
//   O^T = V^T P^T: row r of tile mt is d = 16 r + mt (r < 8) or 16 (r - 8) + 8 + mt, so a
//     lane holding rows g = lane / 4 and g + 8 reads 16 contiguous bytes (d = 16 g ..
//     16 g + 15) of each of its four key rows and pairs bytes of two keys with a byte
//     permute.
#pragma once

#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "decode.cuh"
#include "prologue.cuh"

namespace beam {

constexpr int kDec8Tile = 64;                           // slots per tile
constexpr int kDec8Stages = 4;
constexpr int kDec8TileBytes = kDec8Tile * kD;          // 8 KiB of codes
constexpr int kDec8Smem = kDec8Stages * 2 * kDec8TileBytes;   // 64 KiB: three CTAs per SM

struct Decode8Args {
  DecodeArgs base;          // caches are the code arrays (k_cache / v_cache as bytes)
  float k_scale, v_scale;   // value = code * scale; code = E4M3(value / scale)
};

__device__ __forceinline__ uint32_t swz128(int row, int chunk) {  // byte offset in a tile
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a2,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

constexpr float kDec8QScale = 16.0f;  // queries are split as E4M3 terms of 16 q

// Four E4M3 codes (bytes 0..3 of w) -> two fp16x2: (byte 0, byte 1) and (byte 2, byte 3),
// the lower byte in the lower half; exact.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
  asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %2;\n cvt.rn.f16x2.e4m3x2 %0, a;\n"
      " cvt.rn.f16x2.e4m3x2 %1, b;\n}\n"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// kCluster = false (global cache): partials to the workspace, merged by
// decode_combine_kernel.  kCluster = true (local ring): the splits of a (sequence, KV
// head) form one cluster; the ranks merge their shares of the outputs through
// distributed shared memory and gate them.
template <bool kCluster>
__global__ void __launch_bounds__(kDecThreads) decode8_attn_kernel(const Decode8Args A) {
  const DecodeArgs &a = A.base;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(16) uint8_t q_hi[kGroup * kD];   // E4M3 codes of 16 q
  __shared__ __align__(16) uint8_t q_lo[kGroup * kD];   // E4M3 codes of 16 q - hi
  const int s_idx = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  // launched with programmatic serialization (see decode_attn_kernel)
  pdl_wait();
  pdl_trigger();
  const int64_t t = a.pos[b];
  const int64_t n_vis = decode_visible(a, t);
  if (n_vis == 0) {   // a position outside the cache: nothing is written
    if (threadIdx.x == 0 && s_idx == 0) set_status(a.status, BEAM_ERR_CAPACITY);
    return;
  }
  const int64_t key_lo = (int64_t)s_idx * a.split;
  if (!kCluster && key_lo >= n_vis) return;
  const int64_t key_hi = min(n_vis, key_lo + a.split);
  const int n_keys = key_hi > key_lo ? (int)(key_hi - key_lo) : 0;
  const int n_tiles = (n_keys + kDec8Tile - 1) / kDec8Tile;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t head_off = (size_t)b * a.stride_seq + (size_t)g * a.stride_head;
  uint8_t *kbase = reinterpret_cast<uint8_t *>(a.k_cache) + head_off;
  uint8_t *vbase = reinterpret_cast<uint8_t *>(a.v_cache) + head_off;

  // Thread tid moves chunk tid % 8 of rows tid / 8 + 16 it, it < 4: its swizzle is the same
  // in every row it moves, so the four copies differ by constant offsets.
  const int ld_r = tid >> 3;
  const uint32_t ld_soff = swz128(ld_r, tid & 7);
  const uint8_t *ld_k = kbase + (size_t)(key_lo + ld_r) * kD + (tid & 7) * 16;
  const uint8_t *ld_v = vbase + (size_t)(key_lo + ld_r) * kD + (tid & 7) * 16;
  auto load_tile = [&](int tile, int stage) {
    const uint32_t ks = smem_u32(smem + stage * 2 * kDec8TileBytes) + ld_soff;
    const uint32_t vs = ks + kDec8TileBytes;
    const size_t goff = (size_t)tile * kDec8TileBytes;
    const int rows_left = n_keys - tile * kDec8Tile - ld_r;   // this thread's rows: 0, 16, 32, 48
    if (rows_left > 48) {
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        cp_async16(ks + it * 2048, ld_k + goff + it * 2048, true);
        cp_async16(vs + it * 2048, ld_v + goff + it * 2048, true);
      }
    } else {
      // rows past the run read as zeros (source size 0) and point at the run's first row,
      // which exists (the run is never empty)
      const uint8_t *k_first = kbase + (size_t)key_lo * kD + (tid & 7) * 16;
      const uint8_t *v_first = vbase + (size_t)key_lo * kD + (tid & 7) * 16;
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const bool valid = 16 * it < rows_left;
        cp_async16(ks + it * 2048, valid ? ld_k + goff + it * 2048 : k_first, valid);
        cp_async16(vs + it * 2048, valid ? ld_v + goff + it * 2048 : v_first, valid);
      }
    }
  };
#pragma unroll
  for (int st = 0; st < kDec8Stages - 1; ++st) {
    if (st < n_tiles) load_tile(st, st);
    cp_async_commit();
  }

  int patch_tile = -1, patch_row = 0;  // prefetched tile and row of the new slot
  uint2 patch_val = make_uint2(0u, 0u);
  // cluster: rank r gates outputs [r, r + 1) * 768 / n of the group (idx = 128 hh + d):
  // this thread's are idx0 + 128 k.  The first two gate values are fetched now (all a rank
  // of a 3- or 4-CTA cluster needs), any others at the merge.
  const int merge_n = kGroup * kD / gridDim.x, idx0 = s_idx * merge_n + tid;
  auto gate_at = [&](int idx) {
    const int h = g * kGroup + idx / kD;
    return __uint_as_float((uint32_t)a.gate[((size_t)b * kHq + h) * kD + idx % kD] << 16) +
           a.gate_bias[h];
  };
  float gate_k[2] = {0.f, 0.f};
  {
    if (kCluster) {
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (k * kDecThreads + tid < merge_n) gate_k[k] = gate_at(idx0 + k * kDecThreads);
    }
    // rows: 6 queries, the new key, the new value; a half-warp per row
    const int half = lane >> 4, l16 = lane & 15, row = warp * 2 + half;
    const unsigned half_mask = 0xFFFFu << (half * 16);
    const bool rope = a.kind == BEAM_LOCAL;
    float cs[8], sn[8];
    if (rope) rope_angles(a.inv_freq, t, l16 & 7, cs, sn);
    float w[8];
    load_weights8(row < kGroup ? a.qw : a.kw, l16, w);
    const uint16_t *src = row < kGroup ? a.q_raw + ((size_t)b * kHq + g * kGroup + row) * kD
                                       : (row == kGroup ? a.k_raw : a.v_raw) +
                                             ((size_t)b * kHkv + g) * kD;
    const uint4 raw = *reinterpret_cast<const uint4 *>(src + l16 * 8);
    float x[8];
    if (row == kGroup + 1) {
      x[0] = bf16_lo(raw.x); x[1] = bf16_hi(raw.x); x[2] = bf16_lo(raw.y); x[3] = bf16_hi(raw.y);
      x[4] = bf16_lo(raw.z); x[5] = bf16_hi(raw.z); x[6] = bf16_lo(raw.w); x[7] = bf16_hi(raw.w);
    } else {
      norm_rope_f32(raw, w, rope, cs, sn, l16, half_mask, a.eps, x);
    }
    const int64_t slot = a.kind == BEAM_LOCAL ? t % a.window : t;
    if (row < kGroup) {
      const uint2 hi = f32x8_to_e4m3(x, kDec8QScale);
      const uint32_t hw[4] = {hi.x & 0xFFFFu, hi.x >> 16, hi.y & 0xFFFFu, hi.y >> 16};
      float r[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {   // residual 16 q - hi, exact in fp32
        const uint32_t h2 = e4m3x2_to_f16x2(hw[e]);
        r[2 * e] = fmaf(x[2 * e], kDec8QScale, -__half2float(__ushort_as_half(h2 & 0xFFFFu)));
        r[2 * e + 1] = fmaf(x[2 * e + 1], kDec8QScale, -__half2float(__ushort_as_half(h2 >> 16)));
      }
      *reinterpret_cast<uint2 *>(q_hi + row * kD + l16 * 8) = hi;
      *reinterpret_cast<uint2 *>(q_lo + row * kD + l16 * 8) = f32x8_to_e4m3(r, 1.0f);
    } else if (slot / a.split == s_idx) {
      const uint2 codes = f32x8_to_e4m3_div(x, row == kGroup ? A.k_scale : A.v_scale);
      uint8_t *cache = row == kGroup ? kbase : vbase;
      *reinterpret_cast<uint2 *>(cache + (size_t)slot * kD + l16 * 8) = codes;
      const int rel = (int)(slot - key_lo);
      if (rel / kDec8Tile < kDec8Stages - 1) {
        patch_tile = rel / kDec8Tile;
        patch_row = rel % kDec8Tile;
        patch_val = codes;
      } else {
        __threadfence();  // a later tile streams this row (cp.async.cg reads L2)
      }
    }
    __syncthreads();  // the queries are in shared memory
  }

  float factor = a.scale_log2 * A.k_scale * (1.0f / kDec8QScale);
  if (a.kind == BEAM_GLOBAL) factor *= ssmax_factor(t + 1, a.ssmax_base, a.ssmax_exp);

  // Query fragments (E4M3 hi and lo terms): row h = lane/4 (< 6 valid); k-step ks holds
  // d = 32c + 8ks + 0..3 (register a0) and + 4..7 (a2).
  const int c4 = lane & 3, h = lane >> 2;
  uint4 qh[2], ql[2];   // 32 bytes of the row at d = 32c: words 2ks, 2ks + 1 of k-step ks
  {
    const int hr = h < kGroup ? h : 0;
    qh[0] = *reinterpret_cast<const uint4 *>(q_hi + hr * kD + c4 * 32);
    qh[1] = *reinterpret_cast<const uint4 *>(q_hi + hr * kD + c4 * 32 + 16);
    ql[0] = *reinterpret_cast<const uint4 *>(q_lo + hr * kD + c4 * 32);
    ql[1] = *reinterpret_cast<const uint4 *>(q_lo + hr * kD + c4 * 32 + 16);
    if (h >= kGroup) qh[0] = qh[1] = ql[0] = ql[1] = make_uint4(0u, 0u, 0u, 0u);
  }
  const uint32_t qhw[8] = {qh[0].x, qh[0].y, qh[0].z, qh[0].w, qh[1].x, qh[1].y, qh[1].z, qh[1].w};
  const uint32_t qlw[8] = {ql[0].x, ql[0].y, ql[0].z, ql[0].w, ql[1].x, ql[1].y, ql[1].z, ql[1].w};

  float m_run = -INFINITY;
  float l_run = 0.f;
  float o[8][4];   // O^T tiles: rows d = 16 g + mt (c0, c1) and 16 g + 8 + mt (c2, c3)
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

  const bool any_patch = __syncthreads_or(patch_tile >= 0);
  for (int tile = 0; tile < n_tiles; ++tile) {
    cp_async_wait<kDec8Stages - 2>();
    __syncthreads();
    if (any_patch && tile < kDec8Stages - 1) {
      if (patch_tile == tile) {   // lane l16 of the key / value half-warp: 8 codes at d = 8 l16
        uint8_t *ks = smem + (tile % kDec8Stages) * 2 * kDec8TileBytes;
        uint8_t *dst = (warp * 2 + (lane >> 4) == kGroup) ? ks : ks + kDec8TileBytes;
        const int l16 = lane & 15;
        *reinterpret_cast<uint2 *>(dst + swz128(patch_row, l16 >> 1) + (l16 & 1) * 8) = patch_val;
      }
      __syncthreads();
    }
    {
      const int nt = tile + kDec8Stages - 1;
      if (nt < n_tiles) load_tile(nt, nt % kDec8Stages);
      cp_async_commit();
    }
    const uint8_t *ks = smem + (tile % kDec8Stages) * 2 * kDec8TileBytes;
    const uint8_t *vs = ks + kDec8TileBytes;
    const int wrow = warp * 16;  // this warp's 16 slots of the tile

    // S[head][key] for keys wrow + 8 nb + lane/4
    float s[2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
      s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
      const int r = wrow + nb * 8 + h;
      const uint4 k0 = *reinterpret_cast<const uint4 *>(ks + swz128(r, 2 * c4));
      const uint4 k1 = *reinterpret_cast<const uint4 *>(ks + swz128(r, 2 * c4 + 1));
      const uint32_t kw8[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};  // as codes
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        mma_e4m3_16832(s[nb], qhw[2 * ks], qhw[2 * ks + 1], kw8[2 * ks], kw8[2 * ks + 1]);
        mma_e4m3_16832(s[nb], qlw[2 * ks], qlw[2 * ks + 1], kw8[2 * ks], kw8[2 * ks + 1]);
      }
    }
    // scale, mask the ragged end (last tile only), online softmax for head lane/4
    float mx = -INFINITY;
    if ((tile + 1) * kDec8Tile > n_keys) {
      const int key0 = tile * kDec8Tile + wrow + c4 * 2;
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kk = key0 + nb * 8 + e;
          s[nb][e] = kk < n_keys ? s[nb][e] * factor : -INFINITY;
          mx = fmaxf(mx, s[nb][e]);
        }
    } else {
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[nb][e] *= factor;
          mx = fmaxf(mx, s[nb][e]);
        }
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const bool grew = m_new > m_run;
    const float corr = ex2_approx(m_run - m_use);
    m_run = m_new;
    float p[2][2];
    float psum = 0.f;
#pragma unroll
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        p[nb][e] = ex2_approx(s[nb][e] - m_use);
        psum += p[nb][e];
      }
    l_run = l_run * corr + psum;
    if (__any_sync(0xffffffffu, grew)) {  // O^T columns of heads 2c, 2c + 1: their corrections
      const float corr0 = __shfl_sync(0xffffffffu, corr, (2 * c4) * 4);
      const float corr1 = __shfl_sync(0xffffffffu, corr, (2 * c4 + 1) * 4);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[mt][0] *= corr0; o[mt][1] *= corr1; o[mt][2] *= corr0; o[mt][3] *= corr1;
      }
    }

    // O^T[d][head] += V^T[d][key] P^T[key][head]: keys wrow + 2c + {0,1} (+ 8); the lane's
    // rows are d = 16 g + mt and 16 g + 8 + mt (g = lane / 4)
    const uint32_t pb0 = pack_f16(p[0][0], p[0][1]), pb1 = pack_f16(p[1][0], p[1][1]);
    const int r0 = wrow + c4 * 2;
    const uint4 va = *reinterpret_cast<const uint4 *>(vs + swz128(r0, h));
    const uint4 vb = *reinterpret_cast<const uint4 *>(vs + swz128(r0 + 1, h));
    const uint4 vc = *reinterpret_cast<const uint4 *>(vs + swz128(r0 + 8, h));
    const uint4 vd = *reinterpret_cast<const uint4 *>(vs + swz128(r0 + 9, h));
    const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
    const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      // byte j of word q is d = 16 g + 4q + j, of word q + 2 is d = 16 g + 8 + 4q + j:
      // pair the bytes of keys (r0, r0 + 1) and (r0 + 8, r0 + 9), widen the pairs
      uint32_t x01[4], y01[4], x23[4], y23[4];   // [j]: the pair at byte j
      e4m3x4_to_f16x2x2(prmt(wa[q], wb[q], 0x5140u), x01[0], x01[1]);
      e4m3x4_to_f16x2x2(prmt(wa[q], wb[q], 0x7362u), x01[2], x01[3]);
      e4m3x4_to_f16x2x2(prmt(wa[q + 2], wb[q + 2], 0x5140u), y01[0], y01[1]);
      e4m3x4_to_f16x2x2(prmt(wa[q + 2], wb[q + 2], 0x7362u), y01[2], y01[3]);
      e4m3x4_to_f16x2x2(prmt(wc[q], wd[q], 0x5140u), x23[0], x23[1]);
      e4m3x4_to_f16x2x2(prmt(wc[q], wd[q], 0x7362u), x23[2], x23[3]);
      e4m3x4_to_f16x2x2(prmt(wc[q + 2], wd[q + 2], 0x5140u), y23[0], y23[1]);
      e4m3x4_to_f16x2x2(prmt(wc[q + 2], wd[q + 2], 0x7362u), y23[2], y23[3]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t afr[4] = {x01[j], y01[j], x23[j], y23[j]};
        mma_f16_16816(o[4 * q + j], afr, pb0, pb1);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // Merge the four warps.
  float *sm_o = reinterpret_cast<float *>(smem);                 // [4 warps][6][128]
  float *sm_m = sm_o + 4 * kGroup * kD;                          // [4][6]
  float *sm_l = sm_m + 4 * kGroup;                               // [4][6]
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  if (2 * c4 < kGroup) {   // heads 2c, 2c + 1 (lanes with c = 3 hold the padding columns)
    float *o0 = sm_o + (warp * kGroup + 2 * c4) * kD + 16 * h;
    float *o1 = o0 + kD;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      o0[mt] = o[mt][0];
      o1[mt] = o[mt][1];
      o0[8 + mt] = o[mt][2];
      o1[8 + mt] = o[mt][3];
    }
  }
  if (h < kGroup) {
    if (c4 == 0) {
      sm_m[warp * kGroup + h] = m_run;
      sm_l[warp * kGroup + h] = l_run;
    }
  }
  __syncthreads();
  const size_t part = ((size_t)b * kHkv + g) * a.n_split_max + s_idx;
  for (int idx = tid; idx < kGroup * kD; idx += kDecThreads) {
    const int hh = idx / kD, d = idx - hh * kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w * kGroup + hh]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float sc = exp2f(sm_m[w * kGroup + hh] - Mu);
      acc += sc * sm_o[(w * kGroup + hh) * kD + d];
      L += sc * sm_l[w * kGroup + hh];
    }
    acc *= A.v_scale;
    if (kCluster) {
      float *cl = reinterpret_cast<float *>(smem + 16384);  // this CTA's partial
      cl[idx] = acc;
      if (d == 0) {
        cl[kGroup * kD + hh] = M;
        cl[kGroup * kD + kGroup + hh] = L;
      }
    } else {
      a.part_o[part * (kGroup * kD) + idx] = acc;
      if (d == 0) {
        a.part_ml[(part * kGroup + hh) * 2 + 0] = M;
        a.part_ml[(part * kGroup + hh) * 2 + 1] = L;
      }
    }
  }
  if (kCluster) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    {  // rank r merges its share of the outputs across the ranks and gates them
      float *cl = reinterpret_cast<float *>(smem + 16384);
      const int n_rank = (int)cluster.num_blocks();
      const float *rc[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) rc[r] = cluster.map_shared_rank(cl, r < n_rank ? r : 0);
      for (int k = 0; k < kGroup; ++k) {
        if (k * kDecThreads + tid >= merge_n) break;
        const int idx = idx0 + k * kDecThreads, hh = idx / kD;
        float m[4], M = -INFINITY;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          m[r] = r < n_rank ? rc[r][kGroup * kD + hh] : -INFINITY;
          M = fmaxf(M, m[r]);
        }
        const float Mu = M == -INFINITY ? 0.f : M;
        float acc = 0.f, L = 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (r < n_rank) {
            const float sc = ex2_approx(m[r] - Mu);
            acc += sc * rc[r][idx];
            L += sc * rc[r][kGroup * kD + kGroup + hh];
          }
        }
        const float gl = k == 0 ? gate_k[0] : k == 1 ? gate_k[1] : gate_at(idx);
        const size_t o = ((size_t)b * kHq + g * kGroup + hh) * kD + (idx - hh * kD);
        a.out[o] = (uint16_t)(pack_bf16(acc / L / (1.0f + expf(-gl)), 0.f) & 0xFFFFu);
      }
    }
    cluster.sync();  // every CTA's shared memory stays alive until all ranks have read it
  }
}

}  // namespace beam
