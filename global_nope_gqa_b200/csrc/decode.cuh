// decode.cuh -- split-K decode attention over the bf16 KV cache, then the gate.
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax": one new query per
// sequence attends over the cached keys it can see (section "Two attention
// paths": keys t-511 .. t in a local layer, 0 .. t in a global one); the six
// query heads of a GQA group share one KV head (section "Follow the tensors"),
// and the time goes into streaming the global caches, 4 KiB per token per
// layer (section "KV memory").
//
// decode_attn_kernel: grid (split, KV head, sequence), 128 threads.  Every CTA first
// normalises (and, in a local layer, rotates) the six queries of its group itself; the
// CTA whose run holds the new token's slot also prepares and writes the new key and value
// there.  A CTA then
// streams a contiguous run of `split` cache slots of one (sequence, KV head) --
// keys and values are contiguous in the head-major cache -- through a 3-stage
// cp.async ring of 64-slot tiles (16-byte coalesced loads, XOR-swizzled rows).
// The six heads of the group are the M rows of m16n8k16 tensor-core MMAs
// (rows 6..15 are zero): S = Q K^T and O += P V.  The MMAs exist to take the
// 6 x 128 x 2 multiply-adds per cached row off the FP32 pipe, which would
// otherwise bound the kernel below HBM speed.  Each warp keeps its own online
// softmax over a quarter of every tile; the four warps merge in shared memory.  Then
// either the CTAs of a local ring (one thread-block cluster) merge through distributed
// shared memory and gate the output, or each CTA writes one partial (m, l, o[128]) per
// head and
// decode_combine_kernel: one CTA per (sequence, query head) merges the partials
// with the log-sum-exp rule and applies Y = O/l * sigmoid(G + b_h).
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "prologue.cuh"

namespace beam {

constexpr int kDecThreads = 128;
constexpr int kDecTile = 64;    // cache slots per shared-memory tile
constexpr int kDecStages = 3;   // 96 KiB: two CTAs per SM
constexpr int kDecTileBytes = kDecTile * kD * 2;                   // 16 KiB
constexpr int kDecSmem = kDecStages * 2 * kDecTileBytes;

struct DecodeArgs {
  uint16_t *k_cache;
  uint16_t *v_cache;
  int64_t stride_seq, stride_head, slots;
  const int64_t *pos;       // [B] 0-based position of the new token
  int kind, window;
  int split;                // cache slots per CTA (multiple of kDecTile)
  int n_split_max;          // partial slots reserved per (sequence, KV head)
  float scale_log2;         // softmax_scale * log2(e)
  float ssmax_base, ssmax_exp;
  float *part_o;            // global: [B][8][n_split_max][6][128]
  float *part_ml;           // global: [B][8][n_split_max][6][2]  (max in log2 units, sum)
  const uint16_t *q_raw, *k_raw, *v_raw, *gate;  // [B][48*128], [B][8*128] x 2, [B][48*128]
  const float *qw, *kw, *gate_bias;
  uint16_t *out;            // local: [B][48*128] (a global layer's combine writes it)
  int32_t *status;
  float eps;
  double inv_freq[64];
};

// Number of visible slots of sequence b (0 when the position is invalid).
__device__ __forceinline__ int64_t decode_visible(const DecodeArgs &a, int64_t t) {
  if (t < 0) return 0;
  if (a.kind == BEAM_LOCAL) return t + 1 < a.window ? t + 1 : a.window;
  return t < a.slots ? t + 1 : 0;
}

// kCluster = false (global cache): one split of the keys, partials to the workspace,
// merged by decode_combine_kernel.  kCluster = true (local ring): the whole step in one
// launch -- the splits of a (sequence, KV head) form one thread-block cluster (gridDim.x
// CTAs, at most 4 of 128+ ring slots each), and each rank merges its quarter of the outputs
// across the CTAs' partials through distributed shared memory and writes Y = O/l * sigmoid(G + b).
template <bool kCluster>
__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(const DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(16) uint16_t q_prep[kGroup * kD];
  const int s_idx = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  // launched with programmatic serialization: wait for the kernel before (it may have written
  // any of the inputs), then let the merge kernel after this one be scheduled
  pdl_wait();
  pdl_trigger();
  const int64_t t = a.pos[b];
  const int64_t n_vis = decode_visible(a, t);
  if (n_vis == 0) {   // a position outside the cache: nothing is written (a whole cluster
    if (threadIdx.x == 0 && s_idx == 0) set_status(a.status, BEAM_ERR_CAPACITY);  // leaves)
    return;
  }
  const int64_t key_lo = (int64_t)s_idx * a.split;
  if (!kCluster && key_lo >= n_vis) return;   // a cluster CTA stays: its cluster merges below
  const int64_t key_hi = min(n_vis, key_lo + a.split);
  const int n_keys = key_hi > key_lo ? (int)(key_hi - key_lo) : 0;
  const int n_tiles = (n_keys + kDecTile - 1) / kDecTile;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t head_off = (size_t)b * a.stride_seq + (size_t)g * a.stride_head;
  const uint16_t *kbase = a.k_cache + head_off;
  const uint16_t *vbase = a.v_cache + head_off;

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
      cp_async16(smem_u32(ks + off), kbase + row * kD + c * 8, valid);
      cp_async16(smem_u32(vs + off), vbase + row * kD + c * 8, valid);
    }
  };
  // The first tiles are requested before anything else (in the fused kernel, before the
  // new row is written: a prefetched tile holding that slot is patched in shared memory).
#pragma unroll
  for (int st = 0; st < kDecStages - 1; ++st) {
    if (st < n_tiles) load_tile(st, st);
    cp_async_commit();
  }

  int patch_tile = -1, patch_row = 0;  // prefetched tile and row of the new slot
  uint4 patch_val = make_uint4(0u, 0u, 0u, 0u);
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
    const uint4 res = row == kGroup + 1 ? raw
                                        : norm_rope_row(raw, w, rope, cs, sn, l16, half_mask, a.eps);
    const int64_t slot = a.kind == BEAM_LOCAL ? t % a.window : t;
    if (row < kGroup) {
      *reinterpret_cast<uint4 *>(q_prep + row * kD + l16 * 8) = res;
    } else if (slot / a.split == s_idx) {
      uint16_t *cache = row == kGroup ? a.k_cache : a.v_cache;
      *reinterpret_cast<uint4 *>(cache + head_off + (size_t)slot * kD + l16 * 8) = res;
      const int rel = (int)(slot - key_lo);
      if (rel / kDecTile < kDecStages - 1) {
        patch_tile = rel / kDecTile;
        patch_row = rel % kDecTile;
        patch_val = res;
      } else {
        __threadfence();  // a later tile streams this row (cp.async.cg reads L2)
      }
    }
    __syncthreads();  // the queries are in shared memory
  }

  float factor = a.scale_log2;
  if (a.kind == BEAM_GLOBAL) factor *= ssmax_factor(t + 1, a.ssmax_base, a.ssmax_exp);

  // Query fragments: A rows = heads (lane/4 < 6 valid), 8 k-steps over d.
  uint32_t qa[8][2];
  {
    const int h = lane >> 2;
    const uint16_t *qrow = q_prep + (h < kGroup ? h : 0) * kD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int d0 = ks * 16 + (lane & 3) * 2;
      uint32_t lo = *reinterpret_cast<const uint32_t *>(qrow + d0);
      uint32_t hi = *reinterpret_cast<const uint32_t *>(qrow + d0 + 8);
      qa[ks][0] = h < kGroup ? lo : 0u;
      qa[ks][1] = h < kGroup ? hi : 0u;
    }
  }

  float m_run = -INFINITY;   // running max (log2 units) of head lane/4
  float l_run = 0.f;         // this thread's share of the running sum
  float o[16][4];
#pragma unroll
  for (int nb = 0; nb < 16; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;

  const bool any_patch = __syncthreads_or(patch_tile >= 0);
  for (int tile = 0; tile < n_tiles; ++tile) {
    cp_async_wait<kDecStages - 2>();
    __syncthreads();
    if (any_patch && tile < kDecStages - 1) {
      // the new key / value row, written after this tile was requested
      if (patch_tile == tile) {
        uint8_t *ks = smem + (tile % kDecStages) * 2 * kDecTileBytes;
        uint8_t *dst = (warp * 2 + (lane >> 4) == kGroup) ? ks : ks + kDecTileBytes;
        *reinterpret_cast<uint4 *>(dst + swz256(patch_row, lane & 15)) = patch_val;
      }
      __syncthreads();
    }
    {  // refill the stage that the previous iteration finished with
      const int nt = tile + kDecStages - 1;
      if (nt < n_tiles) load_tile(nt, nt % kDecStages);
      cp_async_commit();
    }
    const uint8_t *ks = smem + (tile % kDecStages) * 2 * kDecTileBytes;
    const uint8_t *vs = ks + kDecTileBytes;
    const int wrow = warp * 16;  // this warp's 16 slots of the tile

    // S[head][key] for the warp's 16 keys: two n-blocks of 8 keys.
    float s[2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int kstep = 0; kstep < 8; ++kstep) {
      // matrices: (keys 0-7, d lo), (keys 0-7, d hi), (keys 8-15, d lo), (keys 8-15, d hi)
      const int r = wrow + (lane & 7) + ((lane >> 4) << 3);
      const int c = kstep * 2 + ((lane >> 3) & 1);
      uint32_t kb[4];
      ldmatrix_x4(kb, smem_u32(ks + swz256(r, c)));
      const uint32_t afr[4] = {qa[kstep][0], 0u, qa[kstep][1], 0u};
      mma_bf16_16816(s[0], afr, kb[0], kb[1]);
      mma_bf16_16816(s[1], afr, kb[2], kb[3]);
    }
    // scale, mask the ragged end, online softmax for head lane/4
    const int key0 = tile * kDecTile + wrow + (lane & 3) * 2;  // key of s[0][0] within the run
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

    // O[head][d] += P[head][key16] V[key16][d]
    const uint32_t pa[4] = {pack_bf16(p[0][0], p[0][1]), 0u, pack_bf16(p[1][0], p[1][1]), 0u};
#pragma unroll
    for (int nb = 0; nb < 16; nb += 2) {
      // matrices: (keys 0-7, d block nb), (keys 8-15, nb), (keys 0-7, nb+1), (keys 8-15, nb+1)
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

  // Merge the four warps.  Shared memory is free again: reuse it.
  float *sm_o = reinterpret_cast<float *>(smem);                 // [4 warps][6][128]
  float *sm_m = sm_o + 4 * kGroup * kD;                          // [4][6]
  float *sm_l = sm_m + 4 * kGroup;                               // [4][6]
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  const int h = lane >> 2;
  if (h < kGroup) {
#pragma unroll
    for (int nb = 0; nb < 16; ++nb) {
      const int d0 = nb * 8 + (lane & 3) * 2;
      sm_o[(warp * kGroup + h) * kD + d0] = o[nb][0];
      sm_o[(warp * kGroup + h) * kD + d0 + 1] = o[nb][1];
    }
    if ((lane & 3) == 0) {
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

struct CombineArgs {
  const float *part_o;
  const float *part_ml;
  const int64_t *pos;
  const uint16_t *gate;     // [B][48*128]
  const float *gate_bias;   // [48]
  uint16_t *out;            // [B][48*128]
  int kind, window, split, n_split_max;
  int64_t slots;
};

// One CTA of 256 threads per (query head, sequence).  The split weights 2^(m_s - M) are formed
// once in shared memory (every split's m read in parallel); then warp w sums the splits
// w, w + 8, ... for d = 4 lane .. 4 lane + 3 with independent float4 loads, and the eight
// warp sums are added in shared memory: a few memory latencies in all, not one per split.
// Y = O / l * sigmoid(G + b_h).
constexpr int kCombineMaxSplits = 1024;
constexpr int kCombineThreads = 256;
__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(const CombineArgs a) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int g = h / kGroup, hh = h - g * kGroup;
  pdl_wait();   // the partials of the attention kernel before this one
  const int64_t t = a.pos[b];
  int64_t n_vis;
  if (t < 0) n_vis = 0;
  else if (a.kind == BEAM_LOCAL) n_vis = t + 1 < a.window ? t + 1 : a.window;
  else n_vis = t < a.slots ? t + 1 : 0;
  if (n_vis == 0) return;  // invalid position: output untouched, status set upstream
  const int n_split = (int)min((n_vis + a.split - 1) / a.split, (int64_t)kCombineMaxSplits);
  __shared__ float sm_w[kCombineMaxSplits];
  __shared__ float sm_red[kCombineThreads / 32];
  __shared__ float4 sm_acc[kCombineThreads / 32][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t base = ((size_t)b * kHkv + g) * a.n_split_max;
  // M = max_s m_s
  float mx = -INFINITY;
  for (int s = tid; s < n_split; s += kCombineThreads) {
    const float m = a.part_ml[((base + s) * kGroup + hh) * 2];
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
  // weights and L = sum_s w_s l_s
  float lsum = 0.f;
  for (int s = tid; s < n_split; s += kCombineThreads) {
    const float w = ex2_approx(sm_w[s] - Mu);
    sm_w[s] = w;
    lsum += w * a.part_ml[((base + s) * kGroup + hh) * 2 + 1];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
  __syncthreads();
  if (lane == 0) sm_red[warp] = lsum;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 *po = reinterpret_cast<const float4 *>(a.part_o + (base * kGroup + hh) * kD) + lane;
#pragma unroll 4
  for (int s = warp; s < n_split; s += kCombineThreads / 32) {
    const float w = sm_w[s];
    const float4 v = po[(size_t)s * kGroup * kD / 4];
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
    const size_t oi = ((size_t)b * kHq + h) * kD + 4 * lane;
    const uint2 graw = *reinterpret_cast<const uint2 *>(a.gate + oi);
    const float bias = a.gate_bias[h], inv = 1.0f / L;
    const float gl[4] = {bf16_lo(graw.x), bf16_hi(graw.x), bf16_lo(graw.y), bf16_hi(graw.y)};
    const float ov[4] = {o.x, o.y, o.z, o.w};
    float y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = ov[e] * inv / (1.0f + expf(-(gl[e] + bias)));
    *reinterpret_cast<uint2 *>(a.out + oi) = make_uint2(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]));
  }
}

}  // namespace beam
