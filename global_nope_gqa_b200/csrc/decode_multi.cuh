// decode_multi.cuh -- split-K attention for a few new tokens per sequence (T <= 16) over a
// long history: multi-token decode, e.g. the verification of a block of drafted tokens.
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax": new token i of sequence b is the
// query at position t = pos0[b] + i; it sees the earlier keys of its window (local) or all of
// them (global) plus the new keys up to itself (sections "Two attention paths", "KV memory").
// This is the chunked prefill of prefill_tc.cuh for small T, where a 128-row query tile would
// be almost empty and only 24 B units would stream the whole history: here the keys are split
// across CTAs instead, as in the one-token decode.
//
// Key source.  Keys and values are read from rows addressed by a coordinate c:
// base + b * stride_seq + g * stride_head + c * stride_row.  A global layer reads its cache
// (c = slot = position, the new rows already appended); a local layer reads the workspace copy
// [window - 1 ring rows | the T new rows] (c = window - 1 + i for new token i).  Query i's own
// key is at kq + i and it sees c in [max(kq + i - window + 1, kmin), kq + i] (local) or
// [0, kq + i] (global), as in the chunk kernel.
//
// Grid (m-tile + n_mt * split, KV head, sequence), 128 threads: the m-tiles of one run of keys
// are neighbours in launch order, so they stream the same tiles at the same time and all but
// the first read them from L2.  M-tile mt holds new tokens 2 mt and
// 2 mt + 1: MMA rows 6 j + h for token 2 mt + j and head h of the group (rows 12..15 are
// padding).  The CTA prepares those rows (RMSNorm, RoPE at the token's position for a local
// layer; a(t+1) joins the row's score scale), streams its run of key coordinates through a
// 3-stage cp.async ring of 64-row tiles, and writes one partial (m, l, o[128]) per row;
// decode_multi_combine_kernel merges the splits and gates.  Each warp owns 16 keys of every
// tile: S (16 rows x 16 keys) and O (16 rows x 128) on bf16 m16n8k16 MMAs, one online softmax
// per row.
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "prologue.cuh"

namespace beam {

constexpr int kMultiMaxT = 16;          // new tokens per sequence handled here
constexpr int kMultiTokPerTile = 2;     // tokens per 16-row m-tile
constexpr int kMultiRows = kMultiTokPerTile * kGroup;   // 12 valid rows

struct MultiArgs {
  const uint16_t *q_raw;        // [B][T][48*128]
  const uint16_t *key, *val;    // key / value rows by coordinate (see above)
  int64_t stride_seq, stride_head, stride_row;   // elements
  const int64_t *pos0;          // [B]
  const float *qw;
  float eps;
  int kind, window, T, n_mt;
  int prefix;                   // local: window - 1 (kq = prefix), global: 0 (kq = pos0)
  int64_t slots;                // global: cache capacity
  int split, n_split_max;
  float scale_log2, ssmax_base, ssmax_exp;
  float *part_o;                // [B][8][n_mt][n_split_max][16][128]
  float *part_ml;               // [B][8][n_mt][n_split_max][16][2]
  double inv_freq[64];
};

// Key-coordinate range of sequence b and the coordinate of token 0's own key; false when
// the sequence's pos0 is out of range (the prologue has set the status; nothing is done).
__device__ __forceinline__ bool multi_range(const MultiArgs &a, int b, int64_t &kq, int64_t &lo,
                                            int64_t &hi) {
  const int64_t p0 = a.pos0[b];
  if (p0 < 0) return false;
  if (a.kind == BEAM_LOCAL) {
    kq = a.prefix;
    const int64_t kmin = a.prefix - min(p0, (int64_t)a.prefix);
    lo = max(kmin, kq - a.window + 1);
  } else {
    if (p0 + a.T > a.slots) return false;
    kq = p0;
    lo = 0;
  }
  hi = kq + a.T - 1;
  return true;
}

__global__ void __launch_bounds__(kDecThreads) decode_multi_kernel(const MultiArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(16) uint16_t q_prep[16 * kD];
  const int s_idx = blockIdx.x / a.n_mt, mt = blockIdx.x - s_idx * a.n_mt, g = blockIdx.y;
  const int b = blockIdx.z;
  int64_t kq, lo_all, hi_all;
  if (!multi_range(a, b, kq, lo_all, hi_all)) return;
  const int64_t key_lo = lo_all + (int64_t)s_idx * a.split;
  if (key_lo > hi_all) return;
  const int64_t key_hi = min(hi_all + 1, key_lo + a.split);   // exclusive
  const int n_keys = (int)(key_hi - key_lo);
  const int n_tiles = (n_keys + kDecTile - 1) / kDecTile;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint16_t *kbase = a.key + (size_t)b * a.stride_seq + (size_t)g * a.stride_head;
  const uint16_t *vbase = a.val + (size_t)b * a.stride_seq + (size_t)g * a.stride_head;

  auto load_tile = [&](int tile, int stage) {
    uint8_t *ks = smem + stage * 2 * kDecTileBytes;
    uint8_t *vs = ks + kDecTileBytes;
    const int64_t row0 = key_lo + (int64_t)tile * kDecTile;
#pragma unroll
    for (int it = 0; it < (kDecTile * 16) / kDecThreads; ++it) {
      const int id = tid + it * kDecThreads;
      const int r = id >> 4, c = id & 15;
      const bool valid = row0 + r < key_hi;
      const int64_t row = valid ? row0 + r : key_lo;
      const uint32_t off = swz256(r, c);
      cp_async16(smem_u32(ks + off), kbase + row * a.stride_row + c * 8, valid);
      cp_async16(smem_u32(vs + off), vbase + row * a.stride_row + c * 8, valid);
    }
  };
#pragma unroll
  for (int st = 0; st < kDecStages - 1; ++st) {
    if (st < n_tiles) load_tile(st, st);
    cp_async_commit();
  }

  // rows 6 j + h: token 2 mt + j, head g * 6 + h; a half-warp per row, 8 rows per pass
  const int64_t p0 = a.pos0[b];
  {
    const int half = lane >> 4, l16 = lane & 15;
    const unsigned half_mask = 0xFFFFu << (half * 16);
    float w[8];
    load_weights8(a.qw, l16, w);
    for (int row = warp * 2 + half; row < 16; row += 8) {
      const int tok = 2 * mt + row / kGroup;
      uint4 res = make_uint4(0u, 0u, 0u, 0u);
      if (row < kMultiRows && tok < a.T) {   // the shuffles below stay inside the half-warp
        const int h = g * kGroup + row % kGroup;
        const uint4 raw = *reinterpret_cast<const uint4 *>(
            a.q_raw + (((size_t)b * a.T + tok) * kHq + h) * kD + l16 * 8);
        float cs[8], sn[8];
        const bool rope = a.kind == BEAM_LOCAL;
        if (rope) rope_angles(a.inv_freq, p0 + tok, l16 & 7, cs, sn);
        res = norm_rope_row(raw, w, rope, cs, sn, l16, half_mask, a.eps);
      }
      *reinterpret_cast<uint4 *>(q_prep + row * kD + l16 * 8) = res;
    }
  }
  __syncthreads();

  // per row (r = lane/4 and lane/4 + 8): visible coordinates [lo, hi] and score scale
  int row_lo[2], row_hi[2];   // relative to key_lo; hi < lo marks a padding row
  float factor[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int row = (lane >> 2) + 8 * e;
    const int tok = 2 * mt + row / kGroup;
    factor[e] = a.scale_log2;
    if (row < kMultiRows && tok < a.T) {
      const int64_t hi = kq + tok;
      const int64_t lo = a.kind == BEAM_LOCAL ? max(hi - a.window + 1, lo_all) : 0;
      row_hi[e] = (int)max((int64_t)-1, min(hi - key_lo, (int64_t)a.split));
      row_lo[e] = (int)max((int64_t)0, min(lo - key_lo, (int64_t)a.split + 1));
      if (a.kind == BEAM_GLOBAL)
        factor[e] *= ssmax_factor(p0 + tok + 1, a.ssmax_base, a.ssmax_exp);
    } else {
      row_hi[e] = -1;
      row_lo[e] = 0;
    }
  }

  // Query fragments: rows lane/4 (a0, a2) and lane/4 + 8 (a1, a3), 8 k-steps over d.
  uint32_t qa[8][4];
  {
    const uint16_t *r0 = q_prep + (lane >> 2) * kD, *r1 = r0 + 8 * kD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int d0 = ks * 16 + (lane & 3) * 2;
      qa[ks][0] = *reinterpret_cast<const uint32_t *>(r0 + d0);
      qa[ks][1] = *reinterpret_cast<const uint32_t *>(r1 + d0);
      qa[ks][2] = *reinterpret_cast<const uint32_t *>(r0 + d0 + 8);
      qa[ks][3] = *reinterpret_cast<const uint32_t *>(r1 + d0 + 8);
    }
  }

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int nb = 0; nb < 16; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;

  for (int tile = 0; tile < n_tiles; ++tile) {
    cp_async_wait<kDecStages - 2>();
    __syncthreads();
    {
      const int nt = tile + kDecStages - 1;
      if (nt < n_tiles) load_tile(nt, nt % kDecStages);
      cp_async_commit();
    }
    const uint8_t *ks = smem + (tile % kDecStages) * 2 * kDecTileBytes;
    const uint8_t *vs = ks + kDecTileBytes;
    const int wrow = warp * 16;
    float s[2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int kstep = 0; kstep < 8; ++kstep) {
      const int r = wrow + (lane & 7) + ((lane >> 4) << 3);
      const int c = kstep * 2 + ((lane >> 3) & 1);
      uint32_t kb[4];
      ldmatrix_x4(kb, smem_u32(ks + swz256(r, c)));
      mma_bf16_16816(s[0], qa[kstep], kb[0], kb[1]);
      mma_bf16_16816(s[1], qa[kstep], kb[2], kb[3]);
    }
    // s[nb][2e + j]: row lane/4 + 8e, key tile*64 + wrow + 8 nb + 2 (lane%4) + j
    const int key0 = tile * kDecTile + wrow + (lane & 3) * 2;
    float corr[2], p[2][4];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float mx = -INFINITY;
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int kk = key0 + nb * 8 + j;
          float v = s[nb][2 * e + j] * factor[e];
          v = (kk >= row_lo[e] && kk <= row_hi[e]) ? v : -INFINITY;
          s[nb][2 * e + j] = v;
          mx = fmaxf(mx, v);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[e], mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      corr[e] = ex2_approx(m_run[e] - m_use);
      m_run[e] = m_new;
      float psum = 0.f;
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float pv = ex2_approx(s[nb][2 * e + j] - m_use);
          p[e][nb * 2 + j] = pv;
          psum += pv;
        }
      l_run[e] = l_run[e] * corr[e] + psum;
    }
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      o[nb][0] *= corr[0]; o[nb][1] *= corr[0];
      o[nb][2] *= corr[1]; o[nb][3] *= corr[1];
    }
    // P as the A operand: rows lane/4 (+8), keys 2 (lane%4) + {0,1} (+8)
    const uint32_t pa[4] = {pack_bf16(p[0][0], p[0][1]), pack_bf16(p[1][0], p[1][1]),
                            pack_bf16(p[0][2], p[0][3]), pack_bf16(p[1][2], p[1][3])};
#pragma unroll
    for (int nb = 0; nb < 16; nb += 2) {
      const int r = wrow + (lane & 7) + (((lane >> 3) & 1) << 3);
      const int c = nb + (lane >> 4);
      uint32_t vb[4];
      ldmatrix_x4_trans(vb, smem_u32(vs + swz256(r, c)));
      mma_bf16_16816(o[nb], pa, vb[0], vb[1]);
      mma_bf16_16816(o[nb + 1], pa, vb[2], vb[3]);
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // merge the four warps (shared memory is free again), then one partial per row
  float *sm_o = reinterpret_cast<float *>(smem);   // [4 warps][16][128]
  float *sm_m = sm_o + 4 * 16 * kD;                // [4][16]
  float *sm_l = sm_m + 4 * 16;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], 1);
    l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], 2);
    const int row = (lane >> 2) + 8 * e;
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      const int d0 = nb * 8 + (lane & 3) * 2;
      sm_o[(warp * 16 + row) * kD + d0] = o[nb][2 * e];
      sm_o[(warp * 16 + row) * kD + d0 + 1] = o[nb][2 * e + 1];
    }
    if ((lane & 3) == 0) {
      sm_m[warp * 16 + row] = m_run[e];
      sm_l[warp * 16 + row] = l_run[e];
    }
  }
  __syncthreads();
  const size_t part = (((size_t)b * kHkv + g) * a.n_mt + mt) * a.n_split_max + s_idx;
  for (int idx = tid; idx < kMultiRows * kD; idx += kDecThreads) {
    const int row = idx / kD, d = idx - row * kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w * 16 + row]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float sc = ex2_approx(sm_m[w * 16 + row] - Mu);
      acc += sc * sm_o[(w * 16 + row) * kD + d];
      L += sc * sm_l[w * 16 + row];
    }
    a.part_o[(part * 16 + row) * kD + d] = acc;
    if (d == 0) {
      a.part_ml[(part * 16 + row) * 2 + 0] = M;
      a.part_ml[(part * 16 + row) * 2 + 1] = L;
    }
  }
}

struct MultiCombineArgs {
  const float *part_o, *part_ml;
  const int64_t *pos0;
  const uint16_t *gate;       // [B][T][48*128]
  const float *gate_bias;     // [48]
  uint16_t *out;              // [B][T][48*128]
  int kind, window, T, n_mt, prefix, split, n_split_max;
  int64_t slots;
};

// One CTA of 128 threads per (query head, new token, sequence): thread d merges the splits of
// coordinate d (all loads independent), then applies Y = O / l * sigmoid(G + b_h).
__global__ void __launch_bounds__(kD) decode_multi_combine_kernel(const MultiCombineArgs c) {
  const int h = blockIdx.x, tok = blockIdx.y, b = blockIdx.z;
  const int g = h / kGroup, hh = h - g * kGroup;
  const int64_t p0 = c.pos0[b];
  if (p0 < 0 || (c.kind == BEAM_GLOBAL && p0 + c.T > c.slots)) return;  // status set upstream
  int64_t lo, hi = 0;
  if (c.kind == BEAM_LOCAL) {
    const int64_t kmin = c.prefix - min(p0, (int64_t)c.prefix);
    lo = max(kmin, (int64_t)c.prefix - c.window + 1);
    hi = c.prefix + c.T - 1;
  } else {
    lo = 0;
    hi = p0 + c.T - 1;
  }
  const int n_split = (int)((hi - lo) / c.split + 1);
  const int mt = tok / kMultiTokPerTile, row = (tok % kMultiTokPerTile) * kGroup + hh;
  const size_t base = (((size_t)b * kHkv + g) * c.n_mt + mt) * c.n_split_max;
  const int d = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, c.part_ml[((base + s) * 16 + row) * 2]);
  const float Mu = M == -INFINITY ? 0.f : M;
  float acc = 0.f, L = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const size_t pr = (base + s) * 16 + row;
    const float w = ex2_approx(c.part_ml[pr * 2] - Mu);
    acc += w * c.part_o[pr * kD + d];
    L += w * c.part_ml[pr * 2 + 1];
  }
  const size_t oi = (((size_t)b * c.T + tok) * kHq + h) * kD + d;
  const float gl = __uint_as_float((uint32_t)c.gate[oi] << 16) + c.gate_bias[h];
  c.out[oi] = (uint16_t)(pack_bf16(acc / L / (1.0f + expf(-gl)), 0.f) & 0xFFFFu);
}

}  // namespace beam
