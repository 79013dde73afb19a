// prefill_mma.cuh -- flash-attention prefill on warp-level MMAs (m16n8k16).
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax": softmax attention of
// every query row over its visible keys (section "Two attention paths": keys
// t-511 .. t in a local layer, 0 .. t in a global one), query head h reading KV
// head h/6, then Y = O * sigmoid(G + b_h) per coordinate (section "Follow the
// tensors").  The global layer's a(t+1) multiplies each row's fp32 score scale.
//
// CTA = 128 query rows of one head (8 warps x 16 rows), K/V tiles of 64 keys in a
// two-stage cp.async ring; tiles entirely outside the window / causal mask are
// skipped, partial tiles are masked per element.  This is the portable tensor
// path; the tcgen05 kernel replaces it for the full-size workloads.
#pragma once

#include "common.cuh"

namespace beam {

constexpr int kPfBM = 128, kPfBN = 64, kPfThreads = 256;
constexpr int kPfTileBytes = kPfBN * kD * 2;                  // 16 KiB
constexpr int kPfSmem = kPfBM * kD * 2 + 2 * 2 * kPfTileBytes; // 96 KiB

struct PrefillArgs {
  const uint16_t *qn;    // [B][T][48][128] prepared queries
  const uint16_t *kn;    // [B][T][8][128] prepared keys
  const uint16_t *v;     // [B][T][8][128]
  const uint16_t *gate;  // [B][T][48*128]
  const float *gate_bias;
  uint16_t *out;         // [B][T][48*128]
  int T, kind, window, n_qblocks;
  float scale_log2, ssmax_base, ssmax_exp;
};

__global__ void __launch_bounds__(kPfThreads) prefill_mma_kernel(const PrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *qs = smem;
  uint8_t *kv = smem + kPfBM * kD * 2;
  const int qb = a.n_qblocks - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z, g = h / kGroup;
  const int q0 = qb * kPfBM;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool local = a.kind == BEAM_LOCAL;

  const size_t tok0 = (size_t)b * a.T;
  const uint16_t *qbase = a.qn + tok0 * (kHq * kD) + (size_t)h * kD;
  const uint16_t *kbase = a.kn + tok0 * (kHkv * kD) + (size_t)g * kD;
  const uint16_t *vbase = a.v + tok0 * (kHkv * kD) + (size_t)g * kD;

  // key range of the whole CTA, in tiles
  const int q_last = min(a.T, q0 + kPfBM) - 1;
  const int key_lo = local ? max(0, q0 - a.window + 1) : 0;
  const int kt_lo = key_lo / kPfBN, kt_hi = q_last / kPfBN + 1;

  // Q tile
#pragma unroll
  for (int it = 0; it < (kPfBM * 16) / kPfThreads; ++it) {
    const int id = tid + it * kPfThreads;
    const int r = id >> 4, c = id & 15;
    const bool valid = q0 + r < a.T;
    const int row = valid ? q0 + r : 0;
    cp_async16(smem_u32(qs + swz256(r, c)), qbase + (size_t)row * (kHq * kD) + c * 8, valid);
  }
  cp_async_commit();

  auto load_kv = [&](int kt, int stage) {
    uint8_t *ks = kv + stage * 2 * kPfTileBytes;
    uint8_t *vs = ks + kPfTileBytes;
#pragma unroll
    for (int it = 0; it < (kPfBN * 16) / kPfThreads; ++it) {
      const int id = tid + it * kPfThreads;
      const int r = id >> 4, c = id & 15;
      const int j = kt * kPfBN + r;
      const bool valid = j < a.T;
      const int row = valid ? j : 0;
      cp_async16(smem_u32(ks + swz256(r, c)), kbase + (size_t)row * (kHkv * kD) + c * 8, valid);
      cp_async16(smem_u32(vs + swz256(r, c)), vbase + (size_t)row * (kHkv * kD) + c * 8, valid);
    }
  };
  load_kv(kt_lo, 0);
  cp_async_commit();

  // rows of this thread and their score factors
  const int wrow = warp * 16;
  const int r0 = q0 + wrow + (lane >> 2), r1 = r0 + 8;
  float f0 = a.scale_log2, f1 = a.scale_log2;
  if (!local) {
    f0 *= ssmax_factor(r0 + 1, a.ssmax_base, a.ssmax_exp);
    f1 *= ssmax_factor(r1 + 1, a.ssmax_base, a.ssmax_exp);
  }

  cp_async_wait<1>();
  __syncthreads();
  uint32_t qa[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    // matrices: (rows 0-7, d lo), (rows 8-15, d lo), (rows 0-7, d hi), (rows 8-15, d hi)
    const int r = wrow + (lane & 7) + (((lane >> 3) & 1) << 3);
    const int c = ks * 2 + (lane >> 4);
    ldmatrix_x4(qa[ks], smem_u32(qs + swz256(r, c)));
  }

  float o[16][4];
#pragma unroll
  for (int nb = 0; nb < 16; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int kt = kt_lo; kt < kt_hi; ++kt) {
    const int stage = (kt - kt_lo) & 1;
    cp_async_wait<0>();
    __syncthreads();
    if (kt + 1 < kt_hi) load_kv(kt + 1, stage ^ 1);
    cp_async_commit();
    const uint8_t *ks = kv + stage * 2 * kPfTileBytes;
    const uint8_t *vs = ks + kPfTileBytes;

    float s[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int kstep = 0; kstep < 8; ++kstep) {
#pragma unroll
      for (int pr = 0; pr < 4; ++pr) {
        const int r = pr * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int c = kstep * 2 + ((lane >> 3) & 1);
        uint32_t kb[4];
        ldmatrix_x4(kb, smem_u32(ks + swz256(r, c)));
        mma_bf16_16816(s[2 * pr], qa[kstep], kb[0], kb[1]);
        mma_bf16_16816(s[2 * pr + 1], qa[kstep], kb[2], kb[3]);
      }
    }
    // mask + scale
    const int j0 = kt * kPfBN;
    const bool full = (j0 + kPfBN - 1 <= q0) && (!local || (q0 + kPfBM - 1) - j0 <= a.window - 1);
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = j0 + nb * 8 + (lane & 3) * 2 + e;
        float v0 = s[nb][e] * f0, v1 = s[nb][2 + e] * f1;
        if (!full) {
          const bool ok0 = j <= r0 && (!local || r0 - j <= a.window - 1);
          const bool ok1 = j <= r1 && (!local || r1 - j <= a.window - 1);
          v0 = ok0 ? v0 : -INFINITY;
          v1 = ok1 ? v1 : -INFINITY;
        }
        s[nb][e] = v0;
        s[nb][2 + e] = v1;
        mx0 = fmaxf(mx0, v0);
        mx1 = fmaxf(mx1, v1);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = exp2f(m0 - mu0), c1 = exp2f(m1 - mu1);
    m0 = mn0;
    m1 = mn1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      s[nb][0] = exp2f(s[nb][0] - mu0);
      s[nb][1] = exp2f(s[nb][1] - mu0);
      s[nb][2] = exp2f(s[nb][2] - mu1);
      s[nb][3] = exp2f(s[nb][3] - mu1);
      ps0 += s[nb][0] + s[nb][1];
      ps1 += s[nb][2] + s[nb][3];
    }
    l0 = l0 * c0 + ps0;
    l1 = l1 * c1 + ps1;
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      o[nb][0] *= c0; o[nb][1] *= c0;
      o[nb][2] *= c1; o[nb][3] *= c1;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t pa[4] = {pack_bf16(s[2 * kk][0], s[2 * kk][1]),
                              pack_bf16(s[2 * kk][2], s[2 * kk][3]),
                              pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                              pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3])};
#pragma unroll
      for (int nb = 0; nb < 16; nb += 2) {
        const int r = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = nb + (lane >> 4);
        uint32_t vb[4];
        ldmatrix_x4_trans(vb, smem_u32(vs + swz256(r, c)));
        mma_bf16_16816(o[nb], pa, vb[0], vb[1]);
        mma_bf16_16816(o[nb + 1], pa, vb[2], vb[3]);
      }
    }
  }

  // epilogue: O / l * sigmoid(gate + bias)
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = 1.0f / l0, inv1 = 1.0f / l1;
  const float bias = a.gate_bias[h];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = half ? r1 : r0;
    if (r >= a.T) continue;
    const float inv = half ? inv1 : inv0;
    const size_t row_off = (tok0 + r) * (size_t)(kHq * kD) + (size_t)h * kD;
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      const int d = nb * 8 + (lane & 3) * 2;
      const uint32_t graw = *reinterpret_cast<const uint32_t *>(a.gate + row_off + d);
      const float y0 = o[nb][2 * half] * inv / (1.0f + expf(-(bf16_lo(graw) + bias)));
      const float y1 = o[nb][2 * half + 1] * inv / (1.0f + expf(-(bf16_hi(graw) + bias)));
      *reinterpret_cast<uint32_t *>(a.out + row_off + d) = pack_bf16(y0, y1);
    }
  }
}

}  // namespace beam
