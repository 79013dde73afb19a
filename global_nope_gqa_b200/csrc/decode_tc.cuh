// decode_tc.cuh -- multi-token decode on tcgen05 tensor cores: a few new tokens per sequence
// (T <= 16, e.g. the verification of a drafted block) against a long history.
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax": new token i of sequence b is the
// query at t = pos0[b] + i and sees the earlier keys of its window (local) or all of them
// (global) plus the new keys up to itself (sections "Two attention paths", "KV memory").
// Keys are addressed by coordinate exactly as in decode_multi.cuh: a global layer reads its
// cache (coordinate = slot, the new rows already appended), a local layer the workspace copy
// [window - 1 ring rows | the T new rows].
//
// One CTA per (run of key coordinates, KV head, sequence).  Its 128-row Q tile holds the
// (token, head) rows r = 6 i + h of the group for all T new tokens (6 T <= 96 rows; the rest
// are zero), so every key tile is multiplied once for all of them, on tcgen05 MMAs:
//   warp 0      TMA producer: 128-key K tiles into a three-slot ring running two blocks
//               ahead of the V tiles (three slots), 128-byte swizzled 128 x 64 boxes;
//   warp 1      MMA issuer (one thread) and the tensor memory (512 columns): S in two
//               buffers [0,128) [128,256), O [256,384) (fp32).  Block j uses S buffer j % 2,
//               its P (bf16 pairs) overwrites the first 64 columns of that buffer, and
//               S(j + 2) is issued right after O += P(j) V(j): the scores of the next block
//               are computed while the rows work on the current one;
//   warps 2-5   one thread per row (tensor-memory lane = row): first RMSNorm (and, for a
//               local layer, RoPE from the per-token cos/sin table) of the row's query into
//               the swizzled Q tile, then the online softmax per block (mask to the row's
//               coordinates, stale max, O rescaled only when the max grows by more than 2^8,
//               after the previous block's P V is done), then one partial (m, l, o[128]).
// decode_multi_combine_kernel merges the runs and gates or, when a sequence's keys span only a
// few runs, the CTA that finishes last merges them (decode_tc_merge).  Every wait is bounded (tc_wait: 1 s
// of device time, then BEAM_ERR_DEVICE_TIMEOUT, an abort flag for the other roles, and the
// in-flight copies and MMAs drained before the tensor memory is freed).
#pragma once

#include "common.cuh"
#include "decode_multi.cuh"
#include "prefill_tc.cuh"
#include "tc_ptx.cuh"

namespace beam {

// Shared-memory plan, thread count and barrier slots.  BF16 caches: K and V rings of three
// 128-key tiles fed by TMA.  FP8 caches (kFp8): TMA brings the E4M3 tiles (16 KiB) into
// two-slot staging rings and two converter warps widen them into two-slot rings of f16 tiles
// for the MMAs (an E4M3 value is exact in f16, and a kind::f16 MMA takes f16 A and B alike:
// the Q tile and P are f16 too).
constexpr uint32_t kDtCodeTile = 128 * 128;   // one 128-key tile of E4M3 codes
template <bool kFp8>
struct DtCfg {
  static constexpr int kThreads = kFp8 ? 256 : 192;
  static constexpr int kKSlots = kFp8 ? 2 : 3, kVSlots = kFp8 ? 2 : 3;
  static constexpr int kStage = kFp8 ? 2 : 0;    // staging slots for K and for V
  static constexpr int kConvThreads = 64;        // warps 6-7 (FP8)
  static constexpr uint32_t kSmemQ = 0;                                 // one 128 x 128 Q tile
  static constexpr uint32_t kSmemK = kTcTileBytes;                      // K ring
  static constexpr uint32_t kSmemV = kSmemK + kKSlots * kTcTileBytes;   // V ring
  static constexpr uint32_t kSmemSK = kSmemV + kVSlots * kTcTileBytes;  // FP8 staging: K
  static constexpr uint32_t kSmemSV = kSmemSK + kStage * kDtCodeTile;   //                V
  static constexpr uint32_t kSmemBar = kSmemSV + kStage * kDtCodeTile;
  static constexpr uint32_t kSmemBytes = kSmemBar + 256 + 1024;         // 230,656 B either way
  // barrier slots (8 bytes each) after kSmemBar
  static constexpr int kKFull = 0, kKEmpty = kKFull + kKSlots, kVFull = kKEmpty + kKSlots,
                       kVEmpty = kVFull + kVSlots, kSFull = kVEmpty + kVSlots, kPFull = kSFull + 2,
                       kPVDone = kPFull + 2, kOFull = kPVDone + 1, kQReady = kOFull + 1,
                       kDrain = kQReady + 1, kStall = kDrain + 1, kSKFull = kStall + 1,
                       kSKEmpty = kSKFull + kStage, kSVFull = kSKEmpty + kStage,
                       kSVEmpty = kSVFull + kStage, kNumBars = kSVEmpty + kStage;
  static constexpr uint32_t kTmemHolder = kNumBars * 8;
  static constexpr uint32_t kAbortFlag = kTmemHolder + 4;
  static_assert(kAbortFlag + 4 <= 256, "the barrier area holds 256 bytes");
  static_assert(kSmemBar <= 7 * kTcTileBytes, "shared memory plan overflows");
};
constexpr uint32_t kDtSmemBytes = DtCfg<false>::kSmemBytes;
static_assert(DtCfg<true>::kSmemBytes == kDtSmemBytes, "one shared-memory opt-in serves both");

// Two floats as an f16 pair (low half first), nearest.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

struct DecodeTcArgs {
  const uint16_t *q_raw;      // [B][T][48*128]
  const float *qw;            // [128]
  float eps;
  const float *rope_tab;      // local: [B][T][128] cos (64) then sin (64) of each new token
  const int64_t *pos0;        // [B]
  int kind, window, T, prefix;  // prefix: local window - 1, global 0
  int64_t slots;              // global: cache capacity
  int split, n_split_max, n_mt;   // split: key coordinates per CTA, a multiple of 128
  float scale_log2, ssmax_base, ssmax_exp;
  float *part_o, *part_ml;    // the layout decode_multi_combine_kernel reads
  // direct != 0: one CTA covers all of a sequence's keys for its KV head (n_split_max == 1),
  // so it writes Y = O / l * sigmoid(G + b_h) itself and no merge runs
  int direct;
  const uint16_t *gate;       // [B][T][48*128]
  const float *gate_bias;     // [48]
  uint16_t *out;              // [B][T][48*128]
  int32_t *status;
  int kv_slot_major;          // K/V maps take (d, slot, head, b) rather than (d, head, t, b)
  int fault_stall;            // tests only: the MMA issuer first waits on a barrier never arrived at
  // fold != 0: no merge kernel follows; the last CTA of each (sequence, KV head) to finish
  // -- found by a ticket, tickets[b * 8 + g], zeroed by the prologue launch of the same call
  // -- merges the partials of all its runs and writes the gated output rows
  int fold;
  uint32_t *tickets;          // [B][8]
  // FP8 caches: the K/V maps read the unscaled values of the codes; keys are k_scale times
  // their values (folded into the score factor), values v_scale times theirs (into o)
  float k_scale, v_scale;
};

// Merge of the runs of one (sequence b, KV head g) by the CTA that finished last, with the
// log-sum-exp rule of decode_multi_combine_kernel, and the gate.  Warp w takes the rows
// r = w, w + 6, ... (row r = 6 i + h: new token i, head h of the group); lane l owns
// coordinates 4 l .. 4 l + 3.  The partials of the other CTAs are read through L2.
__device__ __forceinline__ void decode_tc_merge(const DecodeTcArgs &a, int b, int g, int n_part) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_warps = blockDim.x >> 5;
  for (int r = warp; r < kGroup * a.T; r += n_warps) {
    const int tok = r / kGroup, hh = r - tok * kGroup;
    const int mt = tok / kMultiTokPerTile, row16 = (tok % kMultiTokPerTile) * kGroup + hh;
    const size_t base = (((size_t)b * kHkv + g) * a.n_mt + mt) * a.n_split_max;
    float M = -INFINITY;
    for (int sp = lane; sp < n_part; sp += 32)
      M = fmaxf(M, __ldcg(a.part_ml + ((base + sp) * 16 + row16) * 2));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp = 0; sp < n_part; ++sp) {
      const size_t idx = (base + sp) * 16 + row16;
      const float w = ex2_approx(__ldcg(a.part_ml + idx * 2) - Mu);
      L = fmaf(w, __ldcg(a.part_ml + idx * 2 + 1), L);
      const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.part_o + idx * kD) + lane);
      o.x = fmaf(w, v.x, o.x); o.y = fmaf(w, v.y, o.y);
      o.z = fmaf(w, v.z, o.z); o.w = fmaf(w, v.w, o.w);
    }
    const int h = g * kGroup + hh;
    const size_t oi = (((size_t)b * a.T + tok) * kHq + h) * kD + 4 * lane;
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

template <bool kFp8>
__global__ void __launch_bounds__(DtCfg<kFp8>::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeTcArgs a) {
  using C = DtCfg<kFp8>;
  // operand pairs of the MMAs: bf16 over a bf16 cache, f16 over widened E4M3 codes
  auto pack_op = [](float lo, float hi) { return kFp8 ? pack_f16x2(lo, hi) : pack_bf16(lo, hi); };
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // SW128 tiles need 1024-byte alignment
  uint8_t *sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::kSmemBar;
  volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sgen + C::kSmemBar + C::kAbortFlag);
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  const int s_idx = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool local = a.kind == BEAM_LOCAL;

  // key coordinates of the sequence (see above); an out-of-range pos0 has set the status in
  // the prologue and does nothing here (the whole CTA returns together)
  const int64_t p0 = a.pos0[b];
  if (p0 < 0 || (!local && p0 + a.T > a.slots)) return;
  int64_t kq, lo_all;
  if (local) {
    kq = a.prefix;
    lo_all = max(a.prefix - min(p0, (int64_t)a.prefix), kq - a.window + 1);
  } else {
    kq = p0;
    lo_all = 0;
  }
  const int64_t hi_all = kq + a.T - 1;
  const int64_t key_lo = lo_all + (int64_t)s_idx * a.split;
  if (key_lo > hi_all) return;
  const int n_keys = (int)min(hi_all + 1 - key_lo, (int64_t)a.split);
  const int nb = (n_keys + kTcBN - 1) / kTcBN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) {
      uint32_t count = (i == C::kPFull || i == C::kPFull + 1 || i == C::kQReady) ? 128 : 1;
      // FP8: the converter warps fill the MMA rings and release the staging slots
      if (kFp8 && ((i >= C::kKFull && i < C::kKFull + C::kKSlots) ||
                   (i >= C::kVFull && i < C::kVFull + C::kVSlots) ||
                   (i >= C::kSKEmpty && i < C::kSKEmpty + C::kStage) ||
                   (i >= C::kSVEmpty && i < C::kSVEmpty + C::kStage)))
        count = C::kConvThreads;
      tc::mbar_init(bar(i), count);
    }
    *abort = 0u;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + C::kSmemBar + C::kTmemHolder, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sgen + C::kSmemBar + C::kTmemHolder);

  if (warp == 0) {
    // ------------------------------------------------------------ K/V producer
    // BF16: the MMA rings themselves; FP8: the staging rings of code tiles (one box of 128
    // codes x 128 keys each, K and V slot-major in the cache)
    constexpr int kKS = kFp8 ? C::kStage : C::kKSlots, kVS = kFp8 ? C::kStage : C::kVSlots;
    constexpr int kKF = kFp8 ? C::kSKFull : C::kKFull, kVF = kFp8 ? C::kSVFull : C::kVFull;
    constexpr int kKE = kFp8 ? C::kSKEmpty : C::kKEmpty, kVE = kFp8 ? C::kSVEmpty : C::kVEmpty;
    if (lane == 0) {
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      auto load = [&](bool is_v, int j, uint32_t slot) {
        const int key0 = (int)(key_lo + (int64_t)j * kTcBN);
        const uint32_t full = bar((is_v ? kVF : kKF) + slot);
        const CUtensorMap *map = is_v ? &tm_v : &tm_k;
        if constexpr (kFp8) {
          tc::mbar_expect_tx(full, kDtCodeTile);
          const uint32_t dst = sbase + (is_v ? C::kSmemSV : C::kSmemSK) + slot * kDtCodeTile;
          tc::tma_load_4d(dst, map, full, 0, key0, g, b);
        } else {
          tc::mbar_expect_tx(full, kTcTileBytes);
          const uint32_t dst = sbase + (is_v ? C::kSmemV : C::kSmemK) + slot * kTcTileBytes;
          for (int hf = 0; hf < 2; ++hf) {
            if (a.kv_slot_major)
              tc::tma_load_4d(dst + hf * kTcHalfBytes, map, full, hf * 64, key0, g, b);
            else
              tc::tma_load_4d(dst + hf * kTcHalfBytes, map, full, hf * 64, g, key0, b);
          }
        }
      };
      int ik = 0, iv = 0;
      bool ok = true;
      for (; ik < 2 && ik < nb; ++ik) load(false, ik, ik % kKS);
      while (ok && iv < nb) {
        if (ik < nb) {
          const uint32_t slot = ik % kKS;
          if (ik >= kKS &&
              !(ok = tc_wait(bar(kKE + slot), (ik / kKS - 1) & 1u, abort, a.status)))
            break;
          load(false, ik, slot);
          ++ik;
        }
        const uint32_t slot = iv % kVS;
        if (iv >= kVS && !(ok = tc_wait(bar(kVE + slot), (iv / kVS - 1) & 1u, abort, a.status)))
          break;
        load(true, iv, slot);
        ++iv;
      }
      for (int sl = 0; sl < kKS; ++sl)
        tc_drain(bar(kKF + sl), (uint32_t)(ik + kKS - 1 - sl) / kKS, a.status);
      for (int sl = 0; sl < kVS; ++sl)
        tc_drain(bar(kVF + sl), (uint32_t)(iv + kVS - 1 - sl) / kVS, a.status);
    }
    __syncwarp();
  } else if (kFp8 && warp >= 6) {
    if constexpr (kFp8) {
    // ------------------------------------------------------------ FP8 converters
    // Tiles in the order the MMAs need them (K0, K1, then V j, K j+2): wait for the code tile
    // and for the MMA ring slot, widen 16 codes at a time into the 128-byte swizzled f16
    // layout the TMA would have written (half h = columns 64 h .. 64 h + 63), keys past the
    // last visible one as zeros (0 times a NaN code would poison a masked key), then publish
    // the tile to the MMA issuer (generic -> async proxy) and free the staging slot.
    const int ct = threadIdx.x - 192;   // 0 .. 63
    bool ok = true;
    auto convert = [&](bool is_v, int j) -> bool {
      const uint32_t ss = (uint32_t)j % C::kStage;
      const int ring = is_v ? C::kVSlots : C::kKSlots;
      const uint32_t rs = (uint32_t)j % ring;
      if (!tc_wait(bar((is_v ? C::kSVFull : C::kSKFull) + ss), (j / C::kStage) & 1u, abort, a.status))
        return false;
      if (j >= ring &&
          !tc_wait(bar((is_v ? C::kVEmpty : C::kKEmpty) + rs), (j / ring - 1) & 1u, abort, a.status))
        return false;
      const uint8_t *src = sgen + (is_v ? C::kSmemSV : C::kSmemSK) + ss * kDtCodeTile;
      uint8_t *dst = sgen + (is_v ? C::kSmemV : C::kSmemK) + rs * kTcTileBytes;
      const int64_t key_first = key_lo + (int64_t)j * kTcBN;
      // a quarter-warp covers one 128-byte row: conflict-free loads; the two stores of a
      // thread go to the two halves in alternating order, so eight threads hit eight banks
#pragma unroll 4
      for (int it = 0; it < 16; ++it) {
        const int item = it * C::kConvThreads + ct;   // 0 .. 1023
        const int r = item >> 3, c8 = item & 7;         // key row, 16-code chunk
        uint4 w = *reinterpret_cast<const uint4 *>(src + r * 128 + ((c8 ^ (r & 7)) << 4));
        if (key_first + r > hi_all) w = make_uint4(0u, 0u, 0u, 0u);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
        uint32_t hx[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hx[2 * e] = e4m3x2_to_f16x2(wv[e] & 0xFFFFu);
          hx[2 * e + 1] = e4m3x2_to_f16x2(wv[e] >> 16);
        }
        const int hf = c8 >> 2, cc = (c8 & 3) * 2;   // columns 16 c8 .. 16 c8 + 15
        uint8_t *row = dst + hf * kTcHalfBytes + r * 128;
        const uint4 lo4 = make_uint4(hx[0], hx[1], hx[2], hx[3]);
        const uint4 hi4 = make_uint4(hx[4], hx[5], hx[6], hx[7]);
        const bool swap = hf != 0;   // the second half stores its odd chunk first
        *reinterpret_cast<uint4 *>(row + (((cc + (swap ? 1 : 0)) ^ (r & 7)) << 4)) = swap ? hi4 : lo4;
        *reinterpret_cast<uint4 *>(row + (((cc + (swap ? 0 : 1)) ^ (r & 7)) << 4)) = swap ? lo4 : hi4;
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      tc::mbar_arrive(bar((is_v ? C::kVFull : C::kKFull) + rs));
      tc::mbar_arrive(bar((is_v ? C::kSVEmpty : C::kSKEmpty) + ss));
      return true;
    };
    for (int j = 0; ok && j < 2 && j < nb; ++j) ok = convert(false, j);
    for (int j = 0; ok && j < nb; ++j) {
      ok = convert(true, j);
      if (ok && j + 2 < nb) ok = convert(false, j + 2);
    }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = kFp8 ? tc::idesc_f16(128, 128, false, false)
                                         : tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = kFp8 ? tc::idesc_f16(128, 128, false, true)
                                         : tc::idesc_bf16(128, 128, false, true);
      auto kdesc = [&](uint32_t tile, int ks) {  // K-major, 128 B rows, 8-row groups 1 KiB apart
        return tc::sdesc_sw128(tile + (ks >> 2) * kTcHalfBytes + (ks & 3) * 32, 16, 1024);
      };
      auto vdesc = [&](uint32_t tile, int kk) {  // MN-major: d halves 16 KiB apart
        return tc::sdesc_sw128(tile + kk * 2048, kTcHalfBytes, 1024);
      };
      const uint32_t qt = sbase + C::kSmemQ;
      auto issue_s = [&](int j) {
        const uint32_t kt = sbase + C::kSmemK + (j % C::kKSlots) * kTcTileBytes;
        const uint32_t d = tmem + 128 * (j & 1);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::umma_ss(d, kdesc(qt, ks), kdesc(kt, ks), idesc_qk, ks > 0 ? 1u : 0u);
        tc::umma_commit(bar(C::kSFull + (j & 1)));
        tc::umma_commit(bar(C::kKEmpty + j % C::kKSlots));
      };
      auto issue_pv = [&](int j) {
        const uint32_t vt = sbase + C::kSmemV + (j % C::kVSlots) * kTcTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::umma_ts(tmem + 256, tmem + 128 * (j & 1) + kk * 8, vdesc(vt, kk), idesc_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
        tc::umma_commit(bar(C::kPVDone));
        tc::umma_commit(bar(C::kVEmpty + j % C::kVSlots));
        if (j == nb - 1) tc::umma_commit(bar(C::kOFull));
      };
      bool ok = (!a.fault_stall || tc_wait(bar(C::kStall), 0u, abort, a.status)) &&
                tc_wait(bar(C::kQReady), 0u, abort, a.status);
      for (int jj = 0; ok && jj < 2 && jj < nb; ++jj) {
        if (!(ok = tc_wait(bar(C::kKFull + jj % C::kKSlots), (jj / C::kKSlots) & 1u, abort,
                           a.status)))
          break;
        tc::tc_fence_after();
        issue_s(jj);
      }
      for (int j = 0; ok && j < nb; ++j) {
        if (!(ok = tc_wait(bar(C::kPFull + (j & 1)), (j >> 1) & 1u, abort, a.status))) break;
        if (!(ok = tc_wait(bar(C::kVFull + j % C::kVSlots), (j / C::kVSlots) & 1u, abort,
                           a.status)))
          break;
        tc::tc_fence_after();
        issue_pv(j);
        if (j + 2 < nb) {
          const int j2 = j + 2;
          if (!(ok = tc_wait(bar(C::kKFull + j2 % C::kKSlots), (j2 / C::kKSlots) & 1u, abort,
                             a.status)))
            break;
          tc::tc_fence_after();
          issue_s(j2);
        }
      }
      tc::umma_commit(bar(C::kDrain));
      tc_drain(bar(C::kDrain), 1, a.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ rows
    const int wq = warp & 3;               // tensor-memory lane quarter of this warp
    const int r = wq * 32 + lane;          // row = tensor-memory lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int tok = r / kGroup, hh = r - tok * kGroup;
    const bool row_ok = tok < a.T;
    {  // the row's query: RMSNorm, RoPE for a local layer, into the swizzled Q tile
      uint4 qv[16];
      const uint4 *src = reinterpret_cast<const uint4 *>(
          a.q_raw + (((size_t)b * a.T + (row_ok ? tok : 0)) * kHq + g * kGroup + hh) * kD);
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        qv[c] = row_ok ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w4[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(bf16_lo(w4[e]), bf16_lo(w4[e]), fmaf(bf16_hi(w4[e]), bf16_hi(w4[e]), ss));
      }
      const float inv = rsqrtf(ss * (1.0f / kD) + a.eps);
      const float4 *w4p = reinterpret_cast<const float4 *>(a.qw);
      // the RoPE table is angle-major: (cos, sin) of angle i of this token's row at
      // i * (B * T) + b * T + tok
      const size_t rope_stride = (size_t)gridDim.z * a.T;
      const float2 *tab = local ? reinterpret_cast<const float2 *>(a.rope_tab) +
                                      (size_t)b * a.T + (row_ok ? tok : 0)
                                : nullptr;
#pragma unroll
      for (int c = 0; c < 8; ++c) {   // coordinates 8c .. 8c+7 and their partners + 64
        const uint32_t lw[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
        const uint32_t hw[4] = {qv[c + 8].x, qv[c + 8].y, qv[c + 8].z, qv[c + 8].w};
        const float4 wl0 = __ldg(w4p + 2 * c), wl1 = __ldg(w4p + 2 * c + 1);
        const float4 wh0 = __ldg(w4p + 16 + 2 * c), wh1 = __ldg(w4p + 16 + 2 * c + 1);
        const float wl[8] = {wl0.x, wl0.y, wl0.z, wl0.w, wl1.x, wl1.y, wl1.z, wl1.w};
        const float wh[8] = {wh0.x, wh0.y, wh0.z, wh0.w, wh1.x, wh1.y, wh1.z, wh1.w};
        float xl[8], xh[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          xl[2 * e] = bf16_lo(lw[e]) * inv * wl[2 * e];
          xl[2 * e + 1] = bf16_hi(lw[e]) * inv * wl[2 * e + 1];
          xh[2 * e] = bf16_lo(hw[e]) * inv * wh[2 * e];
          xh[2 * e + 1] = bf16_hi(hw[e]) * inv * wh[2 * e + 1];
        }
        if (local) {  // rotate-half: coordinate i < 64 pairs with i + 64
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 cs = __ldg(tab + (size_t)(8 * c + e) * rope_stride);
            const float a0 = xl[e], b0 = xh[e];
            xl[e] = a0 * cs.x - b0 * cs.y;
            xh[e] = b0 * cs.x + a0 * cs.y;
          }
        }
        const uint32_t sw = (uint32_t)((c ^ (r & 7)) << 4);
        *reinterpret_cast<uint4 *>(sgen + C::kSmemQ + r * 128 + sw) =
            make_uint4(pack_op(xl[0], xl[1]), pack_op(xl[2], xl[3]), pack_op(xl[4], xl[5]),
                       pack_op(xl[6], xl[7]));
        *reinterpret_cast<uint4 *>(sgen + C::kSmemQ + kTcHalfBytes + r * 128 + sw) =
            make_uint4(pack_op(xh[0], xh[1]), pack_op(xh[2], xh[3]), pack_op(xh[4], xh[5]),
                       pack_op(xh[6], xh[7]));
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      tc::mbar_arrive(bar(C::kQReady));
    }
    // this row's visible coordinates, relative to key_lo (empty for a padding row)
    int rlo = 0, rhi = -1;
    float factor = a.scale_log2 * a.k_scale;
    if (row_ok) {
      const int64_t hi = kq + tok;
      const int64_t lo = local ? max(hi - a.window + 1, lo_all) : 0;
      rhi = (int)max((int64_t)-1, min(hi - key_lo, (int64_t)a.split));
      rlo = (int)max((int64_t)0, min(lo - key_lo, (int64_t)a.split + 1));
      if (!local) factor *= ssmax_factor(p0 + tok + 1, a.ssmax_base, a.ssmax_exp);
    }
    const uint32_t t_o = tmem + lane_off + 256;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // A warp whose 32 rows are all padding (6 T <= 32 wq) only keeps the barrier phases: its
    // query rows are zero, so its scores are zero and its P rows stay zero in tensor memory,
    // and P V never mixes rows.  It leaves the special-function units to the real rows.
    const bool warp_rows = wq * 32 < kGroup * a.T;
    for (int j = 0; j < nb && !warp_rows; ++j) {
      if (!(ok = tc_wait(bar(C::kSFull + (j & 1)), (j >> 1) & 1u, abort, a.status))) break;
      tc::mbar_arrive(bar(C::kPFull + (j & 1)));
    }
    for (int j = 0; j < nb && warp_rows; ++j) {
      if (!(ok = tc_wait(bar(C::kSFull + (j & 1)), (j >> 1) & 1u, abort, a.status))) break;
      tc::tc_fence_after();
      const uint32_t t_s = tmem + lane_off + 128 * (j & 1);
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32(t_s + 32 * c, sr[c]);
      tc::tmem_ld_wait();
      const int k0 = j * kTcBN;
      if (k0 + kTcBN - 1 > rhi || k0 < rlo) {
        const int hi = rhi - k0, lo = rlo - k0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kk = c * 32 + i;
            sr[c][i] = (kk >= lo && kk <= hi) ? sr[c][i] : 0xFF800000u;  // -inf
          }
      }
      float mc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mc[q] = __uint_as_float(sr[q >> 1][(q & 1) * 16]);
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int q = (c * 2 + (i >> 4)) & 7;
          mc[q] = tc::max3f(mc[q], __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]));
        }
      const float mx = tc::max3f(tc::max3f(mc[0], mc[1], mc[2]), tc::max3f(mc[3], mc[4], mc[5]),
                                 fmaxf(mc[6], mc[7])) * factor;
      bool rescale;
      float m_new;
      if (j == 0) {
        rescale = false;
        m_new = mx;
      } else {
        rescale = mx > m + 8.0f;
        m_new = rescale ? mx : m;
      }
      const float alpha = rescale ? ex2_approx(m - m_new) : 1.0f;
      m = m_new;
      const float m_use = m == -INFINITY ? 0.f : m;
      const uint64_t f2 = tc::f2_pack(factor, factor), nm2 = tc::f2_pack(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float y0, y1;
          tc::f2_unpack(tc::f2_fma(tc::f2_pack(__uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1])),
                                   f2, nm2),
                        y0, y1);
          const float p0v = ex2_approx(y0), p1v = ex2_approx(y1);
          acc[(i >> 1) & 3] = tc::f2_add(acc[(i >> 1) & 3], tc::f2_pack(p0v, p1v));
          pk[i >> 1] = pack_op(p0v, p1v);
        }
        tc::tmem_st16(t_s + 16 * c, pk);
      }
      {
        float s0, s1, s2, s3, s4, s5, s6, s7;
        tc::f2_unpack(acc[0], s0, s1);
        tc::f2_unpack(acc[1], s2, s3);
        tc::f2_unpack(acc[2], s4, s5);
        tc::f2_unpack(acc[3], s6, s7);
        l = l * alpha + (((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7)));
      }
      // O *= alpha for the rows whose max moved by more than 2^8, once O holds block j - 1
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
        if (!(ok = tc_wait(bar(C::kPVDone), (j - 1) & 1u, abort, a.status))) break;
        tc::tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(t_o + 32 * c, o);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc::tmem_st32(t_o + 32 * c, o);
        }
      }
      tc::tmem_st_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(bar(C::kPFull + (j & 1)));
    }
    if (ok) ok = tc_wait(bar(C::kOFull), 0u, abort, a.status);
    if (a.direct) {
      // the whole key range: Y = O / l * sigmoid(G + b_h) straight to the output row (not
      // written when a wait ran out)
      if (ok) {
        tc::tc_fence_after();
        const int h = g * kGroup + hh;
        const size_t orow = (((size_t)b * a.T + (row_ok ? tok : 0)) * kHq + h) * kD;
        const uint4 *gp = reinterpret_cast<const uint4 *>(a.gate + orow);
        uint4 *op = reinterpret_cast<uint4 *>(a.out + orow);
        const float inv = a.v_scale / l, bias = a.gate_bias[h];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(t_o + 32 * c, o);
          tc::tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 g4 = __ldg(gp + 4 * c + q);
              const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
              uint32_t yw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float y0 = __uint_as_float(o[8 * q + 2 * e]) * inv / (1.0f + expf(-(bf16_lo(gw[e]) + bias)));
                const float y1 = __uint_as_float(o[8 * q + 2 * e + 1]) * inv / (1.0f + expf(-(bf16_hi(gw[e]) + bias)));
                yw[e] = pack_bf16(y0, y1);
              }
              op[4 * c + q] = make_uint4(yw[0], yw[1], yw[2], yw[3]);
            }
          }
        }
      }
      ok = false;   // nothing more to write
    }
    const int mt = tok / kMultiTokPerTile, row16 = (tok % kMultiTokPerTile) * kGroup + hh;
    const size_t part = ((((size_t)b * kHkv + g) * a.n_mt + mt) * a.n_split_max + s_idx) * 16 + row16;
    if (!ok && row_ok && !a.direct) {   // a wait ran out: the merge turns these rows into NaN
      a.part_ml[part * 2] = __int_as_float(0x7fc00000);
      a.part_ml[part * 2 + 1] = __int_as_float(0x7fc00000);
    }
    if (ok) {
      tc::tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tc::tmem_ld32(t_o + 32 * c, o);
        tc::tmem_ld_wait();
        if (row_ok) {
          float4 *dst = reinterpret_cast<float4 *>(a.part_o + part * kD + 32 * c);
          const float vs = a.v_scale;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(o[4 * q]) * vs, __uint_as_float(o[4 * q + 1]) * vs,
                                 __uint_as_float(o[4 * q + 2]) * vs, __uint_as_float(o[4 * q + 3]) * vs);
        }
      }
      if (row_ok) {
        a.part_ml[part * 2] = m;
        a.part_ml[part * 2 + 1] = l;
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
  if (a.fold) {
    // every partial row of this CTA is written (the barrier above); publish them, take a
    // ticket, and let the CTA that takes the last one merge -- no CTA waits for another
    __shared__ uint32_t s_last;
    const int n_part = (int)((hi_all - lo_all) / a.split) + 1;
    if (threadIdx.x == 0) {
      __threadfence();
      const uint32_t tk = atomicAdd(a.tickets + (size_t)b * kHkv + g, 1u);
      s_last = tk == (uint32_t)(n_part - 1);
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      decode_tc_merge(a, b, g, n_part);
    }
  }
}

}  // namespace beam
