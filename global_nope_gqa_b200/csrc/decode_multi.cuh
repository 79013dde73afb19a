// decode_multi.cuh -- the merge of a multi-token decode (a few new tokens per sequence,
// T <= 16, over a long history; the attention itself is decode_tc_kernel in decode_tc.cuh).
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax": new token i of sequence b is the
// query at t = pos0[b] + i (sections "Two attention paths", "KV memory").  The attention
// kernel splits the history into runs of key coordinates, one CTA per run and KV head, and
// writes one partial (m, l, o[128]) per (token, head) row; rows are grouped as m-tiles of
// two new tokens, row 6 j + h for token 2 mt + j and head h of the group, so the partials
// are [B][8][n_mt][n_split_max][16][128] (m, l: [..][16][2]).  Here the runs are merged
// with the log-sum-exp rule and the gate is applied.
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "prologue.cuh"

namespace beam {

constexpr int kMultiMaxT = 16;          // new tokens per sequence handled here
constexpr int kMultiTokPerTile = 2;     // new tokens per 16-row m-tile of the partials

struct MultiCombineArgs {
  const float *part_o, *part_ml;
  const int64_t *pos0;
  const uint16_t *gate;       // [B][T][48*128]
  const float *gate_bias;     // [48]
  uint16_t *out;              // [B][T][48*128]
  int kind, window, T, n_mt, prefix, split, n_split_max;
  int64_t slots;
};

// One CTA of 256 threads per (query head, new token, sequence), organised as the one-token
// combine: split weights in shared memory, then warp w sums the splits w, w + 8, ... with
// float4 loads, the warp sums are added, and Y = O / l * sigmoid(G + b_h).
__global__ void __launch_bounds__(kCombineThreads) decode_multi_combine_kernel(const MultiCombineArgs c) {
  const int h = blockIdx.x, tok = blockIdx.y, b = blockIdx.z;
  const int g = h / kGroup, hh = h - g * kGroup;
  const int64_t p0 = c.pos0[b];
  if (p0 < 0 || (c.kind == BEAM_GLOBAL && p0 + c.T > c.slots)) return;  // status set upstream
  int64_t lo, hi;
  if (c.kind == BEAM_LOCAL) {
    const int64_t kmin = c.prefix - min(p0, (int64_t)c.prefix);
    lo = max(kmin, (int64_t)c.prefix - c.window + 1);
    hi = c.prefix + c.T - 1;
  } else {
    lo = 0;
    hi = p0 + c.T - 1;
  }
  const int n_split = (int)min((hi - lo) / c.split + 1, (int64_t)kCombineMaxSplits);
  const int mt = tok / kMultiTokPerTile, row = (tok % kMultiTokPerTile) * kGroup + hh;
  const size_t base = (((size_t)b * kHkv + g) * c.n_mt + mt) * c.n_split_max;
  __shared__ float sm_w[kCombineMaxSplits];
  __shared__ float sm_red[kCombineThreads / 32];
  __shared__ float4 sm_acc[kCombineThreads / 32][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float mx = -INFINITY;
  for (int s = tid; s < n_split; s += kCombineThreads) {
    const float m = c.part_ml[((base + s) * 16 + row) * 2];
    sm_w[s] = m;
    mx = fmaxf(mx, m);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) sm_red[warp] = mx;
  __syncthreads();
  float M = sm_red[0];
#pragma unroll
  for (int w = 1; w < kCombineThreads / 32; ++w) M = fmaxf(M, sm_red[w]);
  const float Mu = M == -INFINITY ? 0.f : M;
  __syncthreads();
  float lsum = 0.f;
  for (int s = tid; s < n_split; s += kCombineThreads) {
    const float w = ex2_approx(sm_w[s] - Mu);
    sm_w[s] = w;
    lsum += w * c.part_ml[((base + s) * 16 + row) * 2 + 1];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
  __syncthreads();
  if (lane == 0) sm_red[warp] = lsum;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 *po = reinterpret_cast<const float4 *>(c.part_o + (base * 16 + row) * kD) + lane;
#pragma unroll 4
  for (int s = warp; s < n_split; s += kCombineThreads / 32) {
    const float w = sm_w[s];
    const float4 v = po[(size_t)s * 16 * kD / 4];
    acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
  }
  sm_acc[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineThreads / 32; ++w) L += sm_red[w];
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kCombineThreads / 32; ++w) {
      o.x += sm_acc[w][lane].x; o.y += sm_acc[w][lane].y;
      o.z += sm_acc[w][lane].z; o.w += sm_acc[w][lane].w;
    }
    const size_t oi = (((size_t)b * c.T + tok) * kHq + h) * kD + 4 * lane;
    const uint2 graw = *reinterpret_cast<const uint2 *>(c.gate + oi);
    const float bias = c.gate_bias[h], inv = 1.0f / L;
    const float gl[4] = {bf16_lo(graw.x), bf16_hi(graw.x), bf16_lo(graw.y), bf16_hi(graw.y)};
    const float ov[4] = {o.x, o.y, o.z, o.w};
    float y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = ov[e] * inv / (1.0f + expf(-(gl[e] + bias)));
    *reinterpret_cast<uint2 *>(c.out + oi) = make_uint2(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]));
  }
}

}  // namespace beam
