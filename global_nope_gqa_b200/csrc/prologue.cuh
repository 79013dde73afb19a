// prologue.cuh -- QK-RMSNorm + RoPE (local) and the KV-cache append.
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax", section "Follow the
// tensors, not the parameter label": Q and K are RMS-normalised along the
// 128-wide head axis (eps 1e-6, learned weight), V is not; local layers then
// rotate Q and K with RoPE; global layers leave K alone and scale only Q by a(p).
// Here a(p) is not applied: the attention kernels fold it into the fp32 score
// scale, so the prepared Q of a global layer is the normalised Q.
//
// One CTA of 128 threads per token.  Each half-warp owns one 128-wide row:
// lane l (0..15) holds coordinates 8l .. 8l+7 as one 16-byte load, so the
// rotate-half partner of lane l is lane l ^ 8.  Each of the 64 RoPE angles of a
// token is formed once, by one thread, in fp64 (t * frequency, then reduced to
// [-pi, pi]), because in fp32 t * frequency is off by up to ~0.06 rad at t ~ 1e6;
// the reduced angle then goes through fp32 sincosf, and the cos / sin values reach
// the other threads through shared memory.  Rows: the 8 key heads, and the 8 value heads
// when a cache is written (copied unchanged); queries are prepared inside the attention
// kernels.
#pragma once

#include "common.cuh"

namespace beam {

// Before the prologue of a chunked prefill (positions pos0[b] .. pos0[b] + T - 1 after
// pos0[b] cached tokens).  Local layer: rows e = 0 .. L-1 (L = window - 1) of each
// sequence's key and value buffers get the ring's rows of positions pos0[b] - L + e, i.e.
// the earlier keys still inside the window of the chunk's first token, zeros before
// position 0.  Ring slots the chunk's own tokens overwrite are saved by those tokens' CTAs
// just before they write them (no other CTA reads or writes such a slot).  Global layer: the
// value slots from pos0[b] + T up to the next multiple of 128 (within the capacity) are
// zeroed: the attention kernel reads whole 128-key blocks, and a masked key's weight is
// exactly 0 but 0 times a non-finite stale value would not be.  Run as extra CTAs of the
// prologue launch, one CTA of 128 threads per row; thread x moves 8 coordinates of head
// x / 16.
constexpr int kChunkPadRows = 128;  // global: CTAs per sequence (at most 127 slots to zero)

struct ChunkPrepArgs {
  const int64_t *pos0;
  const uint16_t *k_cache;   // local: the ring (E4M3 codes when fp8)
  uint16_t *v_cache;         // global: the bf16 values the attention reads (cache or FP8 view)
  const uint16_t *v_ring;    // local: the ring's values (E4M3 codes when fp8)
  int64_t stride_seq, stride_head, slots;
  uint16_t *k_ext, *v_ext;   // local: [B][ext_rows][8*128]
  int ext_rows, prefix, T, window, kind;
  int fp8;                   // the ring holds E4M3 codes: copy their unscaled values as bf16
};

__device__ __forceinline__ void chunk_prep_row(const ChunkPrepArgs &a, int cta) {
  const int per_b = a.kind == BEAM_LOCAL ? a.prefix : kChunkPadRows;
  const int b = cta / per_b, e = cta - b * per_b;
  const int head = threadIdx.x >> 4, c = (threadIdx.x & 15) * 8;
  const int64_t p0 = a.pos0[b];
  const size_t cache_row = (size_t)b * a.stride_seq + (size_t)head * a.stride_head;
  if (a.kind == BEAM_LOCAL) {
    // the token i of this call with i % window == e + 1 that enters the ring takes the slot of
    // position p0 - L + e and saves that row itself before overwriting it; the tokens that
    // enter are T - window .. T - 1 (all of them when T < window), so one exists when T >=
    // window, else when e + 1 <= T - 1
    if (p0 >= 0 && (a.T >= a.window || e + 1 <= a.T - 1)) return;
    const int64_t j = p0 - a.prefix + e;
    uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv;
    if (p0 >= 0 && j >= 0) {
      const size_t off = cache_row + (size_t)(j % a.window) * kD + c;
      if (a.fp8) {
        kv = e4m3x8_to_bf16x8(*reinterpret_cast<const uint2 *>(
            reinterpret_cast<const uint8_t *>(a.k_cache) + off));
        vv = e4m3x8_to_bf16x8(*reinterpret_cast<const uint2 *>(
            reinterpret_cast<const uint8_t *>(a.v_ring) + off));
      } else {
        kv = *reinterpret_cast<const uint4 *>(a.k_cache + off);
        vv = *reinterpret_cast<const uint4 *>(a.v_ring + off);
      }
    }
    const size_t dst = ((size_t)b * a.ext_rows + e) * (kHkv * kD) + head * kD + c;
    *reinterpret_cast<uint4 *>(a.k_ext + dst) = kv;
    *reinterpret_cast<uint4 *>(a.v_ext + dst) = vv;
  } else {
    const int64_t end = p0 + a.T, slot = end + e;
    if (p0 < 0 || end > a.slots || slot >= a.slots || slot >= (end + 127) / 128 * 128) return;
    *reinterpret_cast<uint4 *>(a.v_cache + cache_row + (size_t)slot * kD + c) =
        make_uint4(0u, 0u, 0u, 0u);
  }
}

struct PrologueArgs {
  const uint16_t *k;     // [tokens][8*128]
  const uint16_t *v;     // [tokens][8*128] (read only when a cache is written)
  const float *kw;       // [128]
  uint16_t *k_out;       // prepared keys [B][out_rows][8*128], or null
  uint16_t *v_out;       // raw values copied to [B][out_rows][8*128], or null
  int out_rows;          // rows per sequence in k_out / v_out (0: T)
  int out_row0;          // row of token 0 there (the rows before it hold earlier keys)
  uint16_t *k_cache;     // layer caches, or null
  uint16_t *v_cache;
  int64_t stride_seq, stride_head, slots;
  const int64_t *pos0;   // device [B]: position of token 0 of each sequence, or null (= 0)
  float *rope_tab;       // local layers, or null: (cos, sin) of each token's 64 angles,
                         // angle-major [64][rows] float2 (rows: T, or B * T with rope_per_seq)
  int rope_per_seq;      // rope_tab is [B][T][128] (own positions) rather than [T][128] (0 .. T-1)
  int whole_seq;         // a sequence whose tokens do not all fit is not written at all
  int cache_fp8;         // the caches hold E4M3 codes of value / scale (one byte each)
  float k_scale, v_scale;
  // FP8 chunk: the rows the attention reads (k_out / v_out, and the global view) hold the
  // unscaled values of the written codes as bf16; k_view / v_view: a global layer's bf16 view
  // of the cache (same element strides), or null
  uint16_t *k_view, *v_view;
  int32_t *status;
  int T;                 // tokens per sequence in this call
  // chunked prefill: n_prep extra CTAs after the B * T token CTAs prepare the chunk (the
  // ring rows it still sees, or the value padding); ring_save: a token that takes the ring
  // slot of one of those rows copies the row out first
  ChunkPrepArgs prep;
  int n_prep, ring_save;
  uint32_t *tickets;     // or null: [B][8] merge tickets of the multi-token kernel, zeroed here
  int kind;
  int window;
  float eps;
  double inv_freq[64];   // theta^(-2i/128), formed on the host in double
};

// cos / sin of the angle t * f, formed and reduced to [-pi, pi] in fp64, then evaluated
// in fp32.
__device__ __forceinline__ void rope_angle(double f, int64_t t, float &cs, float &sn) {
  const double two_pi = 6.283185307179586;
  const double inv_two_pi = 0.15915494309189535;
  const double phi = (double)t * f;
  const double n = rint(phi * inv_two_pi);
  const double r = fma(-n, two_pi, phi);  // |r| <= pi (+ rounding)
  sincosf((float)r, &sn, &cs);
}

// The angles t * f_i, i = 8 sub .. 8 sub + 7.
__device__ __forceinline__ void rope_angles(const double *inv_freq, int64_t t, int sub,
                                            float (&cs)[8], float (&sn)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) rope_angle(inv_freq[sub * 8 + e], t, cs[e], sn[e]);
}

// RMSNorm of one 128-wide row held by a half-warp (lane l16 holds coordinates
// 8 l16 .. 8 l16 + 7 as eight bf16 in `raw`), times the weights w, then -- for a local
// layer -- rotate-half RoPE with the angles' cos / sin (the partner of coordinate c < 64 is
// c + 64, held by lane l16 ^ 8).  The eight results in fp32.
__device__ __forceinline__ void norm_rope_f32(uint4 raw, const float (&w)[8], bool rope,
                                              const float (&cs)[8], const float (&sn)[8],
                                              int l16, unsigned half_mask, float eps,
                                              float (&x)[8]) {
  x[0] = bf16_lo(raw.x); x[1] = bf16_hi(raw.x); x[2] = bf16_lo(raw.y); x[3] = bf16_hi(raw.y);
  x[4] = bf16_lo(raw.z); x[5] = bf16_hi(raw.z); x[6] = bf16_lo(raw.w); x[7] = bf16_hi(raw.w);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
  for (int off = 1; off < 16; off <<= 1) ss += __shfl_xor_sync(half_mask, ss, off);
  const float inv_rms = rsqrtf(ss * (1.0f / kD) + eps);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = x[e] * inv_rms * w[e];
  if (rope) {
    float y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float partner = __shfl_xor_sync(half_mask, x[e], 8);
      y[e] = (l16 < 8) ? (x[e] * cs[e] - partner * sn[e]) : (x[e] * cs[e] + partner * sn[e]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = y[e];
  }
}

// The same row rounded to bf16.
__device__ __forceinline__ uint4 norm_rope_row(uint4 raw, const float (&w)[8], bool rope,
                                               const float (&cs)[8], const float (&sn)[8],
                                               int l16, unsigned half_mask, float eps) {
  float x[8];
  norm_rope_f32(raw, w, rope, cs, sn, l16, half_mask, eps, x);
  uint4 res;
  res.x = pack_bf16(x[0], x[1]); res.y = pack_bf16(x[2], x[3]);
  res.z = pack_bf16(x[4], x[5]); res.w = pack_bf16(x[6], x[7]);
  return res;
}

__device__ __forceinline__ void load_weights8(const float *w, int l16, float (&out)[8]) {
  const float4 *w4 = reinterpret_cast<const float4 *>(w) + l16 * 2;
  const float4 x0 = w4[0], x1 = w4[1];
  out[0] = x0.x; out[1] = x0.y; out[2] = x0.z; out[3] = x0.w;
  out[4] = x1.x; out[5] = x1.y; out[6] = x1.z; out[7] = x1.w;
}

__global__ void __launch_bounds__(128, 8) prologue_kernel(const PrologueArgs a) {
  // the workspace and the caches may still be in use by the kernel before this one (the
  // previous call on the stream); the attention kernel after this one waits for all of it
  pdl_wait();
  pdl_trigger();
  const int n_tok = (int)gridDim.x - a.n_prep;
  if ((int)blockIdx.x >= n_tok) {   // a chunk-preparation CTA (the whole CTA returns)
    chunk_prep_row(a.prep, (int)blockIdx.x - n_tok);
    return;
  }
  const int tok = blockIdx.x;
  const int b = tok / a.T;
  const int i = tok - b * a.T;
  if (a.tickets && i == 0 && threadIdx.x < kHkv) a.tickets[(size_t)b * kHkv + threadIdx.x] = 0u;
  const int64_t t = (a.pos0 ? a.pos0[b] : 0) + i;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, l16 = lane & 15;
  const bool local = a.kind == BEAM_LOCAL;

  // Cache target of this token.
  bool write_cache = a.k_cache != nullptr;
  int64_t slot = 0;
  if (write_cache && a.whole_seq) {
    const int64_t p0 = a.pos0 ? a.pos0[b] : 0;
    if (p0 < 0 || (!local && p0 + a.T > a.slots)) {
      if (threadIdx.x == 0 && i == 0) set_status(a.status, BEAM_ERR_CAPACITY);
      write_cache = false;
    }
  }
  if (write_cache) {
    if (t < 0) {
      set_status(a.status, BEAM_ERR_CAPACITY);
      write_cache = false;
    } else if (local) {
      write_cache = i >= a.T - a.window;  // earlier tokens of the call leave the window
      slot = t % a.window;
    } else {
      slot = t;
      if (t >= a.slots) {
        if (threadIdx.x == 0) set_status(a.status, BEAM_ERR_CAPACITY);
        write_cache = false;
      }
    }
  }

  // Rows: half-warp w * 2 + half (0 .. 7) owns key head w * 2 + half and value head
  // w * 2 + half.  Their loads are issued first, so that their latency overlaps the angle
  // computation below.
  const int head = warp * 2 + half;
  const bool k_on = a.k_out != nullptr || write_cache;
  const bool v_on = write_cache || a.v_out != nullptr;
  const size_t src_off = (size_t)tok * (kHkv * kD) + head * kD + l16 * 8;
  const uint4 raw_k = k_on ? *reinterpret_cast<const uint4 *>(a.k + src_off) : make_uint4(0u, 0u, 0u, 0u);
  const uint4 raw_v = v_on ? *reinterpret_cast<const uint4 *>(a.v + src_off) : make_uint4(0u, 0u, 0u, 0u);

  // The token's 64 angles, one per thread of warps 0-1, shared through shared memory: every
  // row of the token uses the same angles (and, for the table at positions 0 .. T-1,
  // every sequence).
  __shared__ float4 s_cs[16], s_sn[16];
  float cs[8], sn[8];
  if (local) {
    if (threadIdx.x < 64) {
      const int f = threadIdx.x;
      float c, s;
      rope_angle(a.inv_freq[f], t < 0 ? 0 : t, c, s);
      reinterpret_cast<float *>(s_cs)[f] = c;
      reinterpret_cast<float *>(s_sn)[f] = s;
      if (a.rope_tab && (a.rope_per_seq || b == 0)) {
        // angle-major: (cos, sin) of angle f at row f * rows + (the token's row)
        const size_t rows = a.rope_per_seq ? (size_t)n_tok : (size_t)a.T;
        reinterpret_cast<float2 *>(a.rope_tab)[(size_t)f * rows + (a.rope_per_seq ? tok : i)] =
            make_float2(c, s);
      }
    }
    __syncthreads();
    const int sub = l16 & 7;   // coordinates 8 l16 .. 8 l16 + 7 use angles 8 sub .. 8 sub + 7
    const float4 c0 = s_cs[2 * sub], c1 = s_cs[2 * sub + 1];
    const float4 s0 = s_sn[2 * sub], s1 = s_sn[2 * sub + 1];
    cs[0] = c0.x; cs[1] = c0.y; cs[2] = c0.z; cs[3] = c0.w;
    cs[4] = c1.x; cs[5] = c1.y; cs[6] = c1.z; cs[7] = c1.w;
    sn[0] = s0.x; sn[1] = s0.y; sn[2] = s0.z; sn[3] = s0.w;
    sn[4] = s1.x; sn[5] = s1.y; sn[6] = s1.z; sn[7] = s1.w;
  }

  float wk[8];
  load_weights8(a.kw, l16, wk);

  const unsigned half_mask = 0xFFFFu << (half * 16);  // shuffles stay inside the half-warp
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    const bool is_k = kv == 0;
    if (!(is_k ? k_on : v_on)) continue;   // the same for the whole CTA
    const uint4 raw = is_k ? raw_k : raw_v;
    float x[8];
    if (!is_k) {
      x[0] = bf16_lo(raw.x); x[1] = bf16_hi(raw.x); x[2] = bf16_lo(raw.y); x[3] = bf16_hi(raw.y);
      x[4] = bf16_lo(raw.z); x[5] = bf16_hi(raw.z); x[6] = bf16_lo(raw.w); x[7] = bf16_hi(raw.w);
    } else {
      norm_rope_f32(raw, wk, local, cs, sn, l16, half_mask, a.eps, x);
    }
    uint4 res = raw;
    if (is_k) {
      res.x = pack_bf16(x[0], x[1]); res.y = pack_bf16(x[2], x[3]);
      res.z = pack_bf16(x[4], x[5]); res.w = pack_bf16(x[6], x[7]);
    }
    uint16_t *dst = is_k ? a.k_out : a.v_out;
    // an FP8 cache stores codes of the fp32 rows, not of their bf16 rounding; the attention
    // of an FP8 chunk reads the codes' unscaled values (its scales apply in the kernel)
    uint2 codes = make_uint2(0u, 0u);
    if (a.cache_fp8 && (write_cache || dst)) codes = f32x8_to_e4m3_div(x, is_k ? a.k_scale : a.v_scale);
    const uint4 att = a.cache_fp8 ? e4m3x8_to_bf16x8(codes) : res;
    if (dst) {
      const size_t orow = (size_t)b * (a.out_rows ? a.out_rows : a.T) + a.out_row0 + i;
      *reinterpret_cast<uint4 *>(dst + orow * (kHkv * kD) + head * kD + l16 * 8) = att;
    }
    if (write_cache) {
      const size_t off = (size_t)b * a.stride_seq + (size_t)head * a.stride_head +
                         (size_t)slot * kD + l16 * 8;
      if (a.cache_fp8) {
        uint8_t *cache = reinterpret_cast<uint8_t *>(is_k ? a.k_cache : a.v_cache);
        const int r = a.ring_save ? i % a.window : 0;
        if (r >= 1) {   // as below, for a ring of codes: its old row's values go to the workspace
          const int64_t q = (t - i) + r - a.window;
          const uint4 old = q >= 0 ? e4m3x8_to_bf16x8(*reinterpret_cast<const uint2 *>(cache + off))
                                   : make_uint4(0u, 0u, 0u, 0u);
          uint16_t *ext = is_k ? a.k_out : a.v_out;
          *reinterpret_cast<uint4 *>(ext + ((size_t)b * a.out_rows + r - 1) * (kHkv * kD) +
                                     head * kD + l16 * 8) = old;
        }
        *reinterpret_cast<uint2 *>(cache + off) = codes;
        uint16_t *view = is_k ? a.k_view : a.v_view;
        if (view) *reinterpret_cast<uint4 *>(view + off) = att;
      } else {
        uint16_t *cache = is_k ? a.k_cache : a.v_cache;
        const int r = a.ring_save ? i % a.window : 0;
        if (r >= 1) {
          // before this call the slot held position q = pos0 + r - window, row r - 1 of the
          // earlier keys the chunk still sees: save it (zeros before position 0) before
          // overwriting it
          const int64_t q = (t - i) + r - a.window;
          const uint4 old = q >= 0 ? *reinterpret_cast<const uint4 *>(cache + off)
                                   : make_uint4(0u, 0u, 0u, 0u);
          uint16_t *ext = is_k ? a.k_out : a.v_out;
          *reinterpret_cast<uint4 *>(ext + ((size_t)b * a.out_rows + r - 1) * (kHkv * kD) +
                                     head * kD + l16 * 8) = old;
        }
        *reinterpret_cast<uint4 *>(cache + off) = res;
      }
    }
  }
}

// The cached rows of an FP8 global cache that a chunk reads (positions 0 .. pos0[b] - 1)
// as bf16 values of their codes, unscaled, into a view with the cache's element strides: the
// tcgen05 attention kernels then read the view as they read a bf16 cache, and the scales
// apply inside them.  Grid (slot blocks of 64, KV head, sequence); 256 threads move 16 codes
// each, twice; a block past the sequence's cached rows returns at once.
constexpr int kViewSlots = 64;

struct Fp8ViewArgs {
  const int64_t *pos0;
  const uint8_t *k_codes, *v_codes;
  uint16_t *k_view, *v_view;
  int64_t stride_seq, stride_head, slots;
};

__global__ void __launch_bounds__(256) fp8_view_kernel(const Fp8ViewArgs a) {
  const int g = blockIdx.y, b = blockIdx.z;
  const int64_t s0 = (int64_t)blockIdx.x * kViewSlots;
  const int64_t n = min(max(a.pos0[b], (int64_t)0), a.slots);   // cached rows of the sequence
  if (s0 >= n) return;
  const size_t row0 = (size_t)b * a.stride_seq + (size_t)g * a.stride_head;
#pragma unroll
  for (int rep = 0; rep < 2; ++rep) {
    const int item = rep * 256 + (int)threadIdx.x;
    const int64_t slot = s0 + item / 8;
    if (slot >= n) continue;
    const size_t off = row0 + (size_t)slot * kD + (item % 8) * 16;
    const uint4 kc = *reinterpret_cast<const uint4 *>(a.k_codes + off);
    const uint4 vc = *reinterpret_cast<const uint4 *>(a.v_codes + off);
    *reinterpret_cast<uint4 *>(a.k_view + off) = e4m3x8_to_bf16x8(make_uint2(kc.x, kc.y));
    *reinterpret_cast<uint4 *>(a.k_view + off + 8) = e4m3x8_to_bf16x8(make_uint2(kc.z, kc.w));
    *reinterpret_cast<uint4 *>(a.v_view + off) = e4m3x8_to_bf16x8(make_uint2(vc.x, vc.y));
    *reinterpret_cast<uint4 *>(a.v_view + off + 8) = e4m3x8_to_bf16x8(make_uint2(vc.z, vc.w));
  }
}

}  // namespace beam
