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
// row).  Every E4M3 value is exact in fp16, so the codes are widened to fp16 in registers
// and the m16n8k16 MMAs run on fp16 operands with fp32 accumulation; the queries and the
// probabilities are fp16 too.  k_scale joins the score scale, v_scale the partial output.
//
// Operand layout.  A dot product over d may visit d in any order as long as both
// operands use the same one, and so may the sum over keys in P V, so the fragments are
// laid out for wide shared-memory loads instead of the MMA's natural order:
//   S = Q K^T: in k-step ks, MMA k-slot 2c + {0, 1} (+ 8) of lane c = lane % 4 is
//     d = 32 c + 4 ks + {0, 1} ({2, 3}), so a lane reads its 32 bytes of a key row with
//     two 16-byte loads and takes four bytes per k-step;
//   O = P V: MMA n-index n of n-block nb is d = 16 n + nb, so a lane holding n = lane / 4
//     reads 16 contiguous bytes of each of its four key rows and pairs bytes of two keys
//     with a byte permute; the accumulator column n of n-block nb is then d = 16 n + nb.
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
  float k_scale, v_scale;   // value = code * scale
  float inv_k_scale, inv_v_scale;
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

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// kCluster = false (global cache): partials to the workspace, merged by
// decode_combine_kernel.  kCluster = true (local ring): the splits of a (sequence, KV
// head) form one cluster; rank 0 merges through distributed shared memory and gates.
template <bool kCluster>
__global__ void __launch_bounds__(kDecThreads) decode8_attn_kernel(const Decode8Args A) {
  const DecodeArgs &a = A.base;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(16) __half q_prep[kGroup * kD];
  const int s_idx = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
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

  auto load_tile = [&](int tile, int stage) {
    uint8_t *ks = smem + stage * 2 * kDec8TileBytes;
    uint8_t *vs = ks + kDec8TileBytes;
    const int64_t row0 = key_lo + (int64_t)tile * kDec8Tile;
#pragma unroll
    for (int it = 0; it < (kDec8Tile * 8) / kDecThreads; ++it) {
      const int id = tid + it * kDecThreads;
      const int r = id >> 3, c = id & 7;
      const bool valid = row0 + r < key_hi;
      const int64_t row = valid ? row0 + r : key_lo;
      const uint32_t off = swz128(r, c);
      cp_async16(smem_u32(ks + off), kbase + row * kD + c * 16, valid);
      cp_async16(smem_u32(vs + off), vbase + row * kD + c * 16, valid);
    }
  };
#pragma unroll
  for (int st = 0; st < kDec8Stages - 1; ++st) {
    if (st < n_tiles) load_tile(st, st);
    cp_async_commit();
  }

  int patch_tile = -1, patch_row = 0;  // prefetched tile and row of the new slot
  uint2 patch_val = make_uint2(0u, 0u);
  float gate6[kGroup];
  {
    if (kCluster && s_idx == 0) {
#pragma unroll
      for (int i = 0; i < kGroup; ++i) {
        const int h = g * kGroup + i;
        gate6[i] = __uint_as_float((uint32_t)a.gate[((size_t)b * kHq + h) * kD + tid] << 16) +
                   a.gate_bias[h];
      }
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
      uint4 hv;
      hv.x = pack_f16(x[0], x[1]); hv.y = pack_f16(x[2], x[3]);
      hv.z = pack_f16(x[4], x[5]); hv.w = pack_f16(x[6], x[7]);
      *reinterpret_cast<uint4 *>(q_prep + row * kD + l16 * 8) = hv;
    } else if (slot / a.split == s_idx) {
      const uint2 codes = f32x8_to_e4m3(x, row == kGroup ? A.inv_k_scale : A.inv_v_scale);
      uint8_t *cache = row == kGroup ? kbase : vbase;
      *reinterpret_cast<uint2 *>(cache + (size_t)slot * kD + l16 * 8) = codes;
      const int rel = (int)(slot - key_lo);
      if (rel / kDec8Tile < kDec8Stages - 1) {
        patch_tile = rel / kDec8Tile;
        patch_row = rel % kDec8Tile;
        patch_val = codes;
      }
    }
    __threadfence();  // the new row reaches L2 before the later tiles stream it (cp.async.cg)
    __syncthreads();  // the queries are in shared memory
  }

  float factor = a.scale_log2 * A.k_scale;
  if (a.kind == BEAM_GLOBAL) factor *= ssmax_factor(t + 1, a.ssmax_base, a.ssmax_exp);

  // Query fragments (fp16): row h = lane/4 (< 6 valid); k-step ks holds d = 32c + 4ks + 0..3.
  const int c4 = lane & 3, h = lane >> 2;
  uint32_t qa[8][2];
  {
    const __half *qrow = q_prep + (h < kGroup ? h : 0) * kD + c4 * 32;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint2 v = *reinterpret_cast<const uint2 *>(qrow + ks * 4);
      qa[ks][0] = h < kGroup ? v.x : 0u;
      qa[ks][1] = h < kGroup ? v.y : 0u;
    }
  }

  float m_run = -INFINITY;
  float l_run = 0.f;
  float o[16][4];
#pragma unroll
  for (int nb = 0; nb < 16; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;

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
      const uint32_t kw8[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
      for (int kstep = 0; kstep < 8; ++kstep) {
        const uint32_t afr[4] = {qa[kstep][0], 0u, qa[kstep][1], 0u};
        mma_f16_16816(s[nb], afr, e4m3x2_to_f16x2(kw8[kstep]), e4m3x2_to_f16x2(kw8[kstep] >> 16));
      }
    }
    // scale, mask the ragged end, online softmax for head lane/4 (as in the BF16 kernel)
    const int key0 = tile * kDec8Tile + wrow + c4 * 2;
    float mx = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kk = key0 + nb * 8 + e;
        float v = s[nb][e] * factor;
        v = kk < n_keys ? v : -INFINITY;
        s[nb][e] = v;
        mx = fmaxf(mx, v);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float corr = exp2f(m_run - m_use);
    m_run = m_new;
    float p[2][2];
    float psum = 0.f;
#pragma unroll
    for (int nb = 0; nb < 2; ++nb)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        p[nb][e] = exp2f(s[nb][e] - m_use);
        psum += p[nb][e];
      }
    l_run = l_run * corr + psum;
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) { o[nb][0] *= corr; o[nb][1] *= corr; }

    // O[head][d] += P[head][key] V[key][d]: keys wrow + 2c + {0,1} (+ 8), d = 16 (lane/4) + nb
    const uint32_t pa[4] = {pack_f16(p[0][0], p[0][1]), 0u, pack_f16(p[1][0], p[1][1]), 0u};
    const int r0 = wrow + c4 * 2;
    const uint4 va = *reinterpret_cast<const uint4 *>(vs + swz128(r0, h));
    const uint4 vb = *reinterpret_cast<const uint4 *>(vs + swz128(r0 + 1, h));
    const uint4 vc = *reinterpret_cast<const uint4 *>(vs + swz128(r0 + 8, h));
    const uint4 vd = *reinterpret_cast<const uint4 *>(vs + swz128(r0 + 9, h));
    const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
    const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      // byte j of each word is d = 16 (lane/4) + 4q + j: pair the two keys' bytes
      const uint32_t lo01 = prmt(wa[q], wb[q], 0x5140u), lo23 = prmt(wa[q], wb[q], 0x7362u);
      const uint32_t hi01 = prmt(wc[q], wd[q], 0x5140u), hi23 = prmt(wc[q], wd[q], 0x7362u);
      mma_f16_16816(o[4 * q + 0], pa, e4m3x2_to_f16x2(lo01), e4m3x2_to_f16x2(hi01));
      mma_f16_16816(o[4 * q + 1], pa, e4m3x2_to_f16x2(lo01 >> 16), e4m3x2_to_f16x2(hi01 >> 16));
      mma_f16_16816(o[4 * q + 2], pa, e4m3x2_to_f16x2(lo23), e4m3x2_to_f16x2(hi23));
      mma_f16_16816(o[4 * q + 3], pa, e4m3x2_to_f16x2(lo23 >> 16), e4m3x2_to_f16x2(hi23 >> 16));
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // Merge the four warps (accumulator column n of n-block nb is d = 16 n + nb).
  float *sm_o = reinterpret_cast<float *>(smem);                 // [4 warps][6][128]
  float *sm_m = sm_o + 4 * kGroup * kD;                          // [4][6]
  float *sm_l = sm_m + 4 * kGroup;                               // [4][6]
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  if (h < kGroup) {
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      sm_o[(warp * kGroup + h) * kD + (c4 * 2) * 16 + nb] = o[nb][0];
      sm_o[(warp * kGroup + h) * kD + (c4 * 2 + 1) * 16 + nb] = o[nb][1];
    }
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
    if (cluster.block_rank() == 0) {
      float *cl = reinterpret_cast<float *>(smem + 16384);
      const int n_rank = (int)cluster.num_blocks();
      for (int idx = tid; idx < kGroup * kD; idx += kDecThreads) {
        const int hh = idx / kD;
        float M = -INFINITY;
        for (int r = 0; r < n_rank; ++r)
          M = fmaxf(M, cluster.map_shared_rank(cl, r)[kGroup * kD + hh]);
        const float Mu = M == -INFINITY ? 0.f : M;
        float acc = 0.f, L = 0.f;
        for (int r = 0; r < n_rank; ++r) {
          const float *rc = cluster.map_shared_rank(cl, r);
          const float sc = exp2f(rc[kGroup * kD + hh] - Mu);
          acc += sc * rc[idx];
          L += sc * rc[kGroup * kD + kGroup + hh];
        }
        const int hq = g * kGroup + hh;
        const size_t oi = ((size_t)b * kHq + hq) * kD + (idx - hh * kD);
        float gl = gate6[0];  // idx = tid + 128 * hh: this thread's d is tid for every head
#pragma unroll
        for (int i = 1; i < kGroup; ++i) gl = hh == i ? gate6[i] : gl;
        a.out[oi] = (uint16_t)(pack_bf16(acc / L / (1.0f + expf(-gl)), 0.f) & 0xFFFFu);
      }
    }
    cluster.sync();
  }
}

}  // namespace beam
