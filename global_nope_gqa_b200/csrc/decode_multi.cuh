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
