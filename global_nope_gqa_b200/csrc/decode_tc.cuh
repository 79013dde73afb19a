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
// (token, head) pairs k = 6 i + h of the group for all T new tokens (6 T <= 96 of them), so
// every key tile is multiplied once for all of them on tcgen05 MMAs.  Pair k sits in row k,
// so a warp whose 32 rows are all padding skips the softmax and leaves its sub-partition's
// special-function unit to the others.  The softmax of one 128-key block is the longest step
// of a block, so two row warpgroups take alternate blocks, each with its own S buffer and its
// own O accumulator, and their two results are merged (log-sum-exp) at the end:
//   warps 0-3   row set A (even blocks: S0, O_A);
//   warps 4-7   row set B (odd blocks: S1, O_B);
//               first both sets prepare the queries, two threads to a row: RMSNorm (and, for
//               a local layer, RoPE from the per-token cos/sin table) into the swizzled Q tile;
//               then a row thread masks its block to its pair's coordinates, keeps a stale max
//               (O rescaled only when the max grows by more than 2^8, once this set's
//               previous P V is done), writes P over the first 64 columns of its S buffer;
//   warp 8      TMA producer: 128-key K and V tiles into three-slot rings;
//   warp 9      MMA issuer (one thread) and the 512 tensor-memory columns: S0 [0,128),
//               S1 [128,256), O_A [256,384), O_B [384,512).  S(j + 2) is issued right after
//               O += P(j) V(j), so a block's scores are ready when its set comes back to it;
//   warps 10-11 FP8 caches only: TMA brings each E4M3 value tile (128 codes x 128 keys,
//               16 KiB) into the second half of its ring slot and these warps widen it in
//               place to the f16 tile the P V MMAs read (an E4M3 value is exact in f16, and P
//               is f16 there: a kind::f16 MMA takes one type for A and B).
// Over an FP8 cache the key codes are not widened: S = Q K^T runs on kind::f8f6f4 MMAs
// straight on the TMA-fed code tiles, each query row split into two E4M3 terms,
// s q = hi + lo with lo = E4M3(s q - hi) and s a power of two that brings the row's largest
// coordinate into [64, 128), which keeps about 8 significant bits (bf16 keeps 8); both
// terms accumulate into one S, and k_scale / s joins the row's score factor.
// After the last block set A merges the two sets' (m, l, O) per row and writes one partial
// (m, l, o[128]) -- or, with one run per (sequence, KV head), the gated output itself.
// decode_multi_combine_kernel merges the runs and gates or, when a sequence's keys span only a
// few runs, the CTA that finishes last merges them (decode_tc_merge).  Every wait is bounded
// (tc_wait: 1 s of device time, then BEAM_ERR_DEVICE_TIMEOUT, an abort flag for the other
// roles, and the in-flight copies and MMAs drained before the tensor memory is freed).
#pragma once

#include "common.cuh"
#include "decode_multi.cuh"
#include "prefill_tc.cuh"
#include "tc_ptx.cuh"

namespace beam {

constexpr uint32_t kDtCodeTile = 128 * 128;   // one 128-key tile of E4M3 codes
constexpr int kFoldMaxSplitsDev = 8;          // most runs the in-kernel merge takes
constexpr int kDtThreads = 384;               // 12 warps (roles above)
constexpr int kDtKSlots = 3, kDtVSlots = 3;
constexpr int kDtConvThreads = 64;            // warps 10-11
// Register split (setmaxnreg): the two row warpgroups kDtRowRegs per thread, warps 8-11
// kDtAuxRegs.  setmaxnreg.inc draws on the registers the CTA was launched with (384 threads
// times the kernel's per-thread count, at most 168 at one CTA per SM), and a request above
// that pool never completes, so the host checks the compiled count before the first launch.
constexpr int kDtRowRegs = 192, kDtAuxRegs = 112;
constexpr int kDtRegPool = 128 * (2 * kDtRowRegs + kDtAuxRegs);
static_assert(kDtRegPool <= kDtThreads * 168, "the split must fit the launch's registers");
constexpr uint32_t kDtSmemQ = 0;                                    // one 128 x 128 Q tile
constexpr uint32_t kDtSmemK = kTcTileBytes;                         // K ring
constexpr uint32_t kDtSmemV = kDtSmemK + kDtKSlots * kTcTileBytes;  // V ring
constexpr uint32_t kDtSmemBar = kDtSmemV + kDtVSlots * kTcTileBytes;
constexpr uint32_t kDtSmemRowScale = kDtSmemBar + 256;              // FP8: 1 / s per row
constexpr uint32_t kDtSmemBytes = kDtSmemRowScale + 512 + 1024;     // 231,168 B

namespace dtd {  // barrier slots (8 bytes each) after kDtSmemBar
constexpr int kKFull = 0, kKEmpty = kKFull + kDtKSlots, kVFull = kKEmpty + kDtKSlots,
              kVEmpty = kVFull + kDtVSlots, kVReady = kVEmpty + kDtVSlots,
              kSFull = kVReady + kDtVSlots, kPFull = kSFull + 2,
              kPVDone = kPFull + 2, kOFull = kPVDone + 2, kQReady = kOFull + 1,
              kDrain = kQReady + 1, kStall = kDrain + 1, kNumBars = kStall + 1;
constexpr uint32_t kTmemHolder = kNumBars * 8;
constexpr uint32_t kAbortFlag = kTmemHolder + 4;
static_assert(kAbortFlag + 4 <= 256, "the barrier area holds 256 bytes");
}  // namespace dtd

// Two floats as an f16 pair (low half first), nearest.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

struct DecodeTcArgs {
  const uint16_t *q_raw;      // [B][T][48*128]
  const float *qw;            // [128]
  float eps;
  const float *rope_tab;      // local: (cos, sin) of each new token's angles, angle-major [64][B * T]
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
// log-sum-exp rule of decode_multi_combine_kernel, and the gate.  A thread takes 8
// coordinates of one row (row r = 6 i + h: new token i, head h of the group) and reads the
// (m, l) and the 8 partial coordinates of every run itself, all loads issued before any is
// used (n_part <= kFoldMaxSplitsDev), so a merge costs about one trip through L2.
__device__ __forceinline__ void decode_tc_merge(const DecodeTcArgs &a, int b, int g, int n_part) {
  const int n_items = kGroup * a.T * (kD / 8);
  for (int it = threadIdx.x; it < n_items; it += blockDim.x) {
    const int r = it >> 4, c8 = (it & 15) * 8;
    const int tok = r / kGroup, hh = r - tok * kGroup;
    const int mt = tok / kMultiTokPerTile, row16 = (tok % kMultiTokPerTile) * kGroup + hh;
    const size_t base = (((size_t)b * kHkv + g) * a.n_mt + mt) * a.n_split_max;
    const int h = g * kGroup + hh;
    const size_t oi = (((size_t)b * a.T + tok) * kHq + h) * kD + c8;
    const uint4 graw = __ldg(reinterpret_cast<const uint4 *>(a.gate + oi));
    const float bias = __ldg(a.gate_bias + h);
    float2 ml[kFoldMaxSplitsDev];
    float4 v0[kFoldMaxSplitsDev], v1[kFoldMaxSplitsDev];
#pragma unroll
    for (int sp = 0; sp < kFoldMaxSplitsDev; ++sp) {
      const size_t idx = (base + sp) * 16 + row16;
      const float4 *src = reinterpret_cast<const float4 *>(a.part_o + idx * kD + c8);
      const bool on = sp < n_part;
      ml[sp] = on ? __ldcg(reinterpret_cast<const float2 *>(a.part_ml) + idx)
                  : make_float2(-INFINITY, 0.f);
      v0[sp] = on ? __ldcg(src) : make_float4(0.f, 0.f, 0.f, 0.f);
      v1[sp] = on ? __ldcg(src + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float M = ml[0].x;
#pragma unroll
    for (int sp = 1; sp < kFoldMaxSplitsDev; ++sp) M = fmaxf(M, ml[sp].x);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f, o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int sp = 0; sp < kFoldMaxSplitsDev; ++sp) {
      const float w = sp < n_part ? ex2_approx(ml[sp].x - Mu) : 0.f;
      L = fmaf(w, ml[sp].y, L);
      o[0] = fmaf(w, v0[sp].x, o[0]); o[1] = fmaf(w, v0[sp].y, o[1]);
      o[2] = fmaf(w, v0[sp].z, o[2]); o[3] = fmaf(w, v0[sp].w, o[3]);
      o[4] = fmaf(w, v1[sp].x, o[4]); o[5] = fmaf(w, v1[sp].y, o[5]);
      o[6] = fmaf(w, v1[sp].z, o[6]); o[7] = fmaf(w, v1[sp].w, o[7]);
    }
    const float inv = 1.0f / L;
    const uint32_t gw[4] = {graw.x, graw.y, graw.z, graw.w};
    uint32_t yw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      yw[e] = pack_bf16(o[2 * e] * inv / (1.0f + expf(-(bf16_lo(gw[e]) + bias))),
                        o[2 * e + 1] * inv / (1.0f + expf(-(bf16_hi(gw[e]) + bias))));
    *reinterpret_cast<uint4 *>(a.out + oi) = make_uint4(yw[0], yw[1], yw[2], yw[3]);
  }
}

template <bool kFp8>
__global__ void __launch_bounds__(kDtThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeTcArgs a) {
  // operand pairs of the MMAs: bf16 over a bf16 cache, f16 over widened E4M3 codes
  auto pack_op = [](float lo, float hi) { return kFp8 ? pack_f16x2(lo, hi) : pack_bf16(lo, hi); };
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // SW128 tiles need 1024-byte alignment
  uint8_t *sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + kDtSmemBar;
  volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sgen + kDtSmemBar + dtd::kAbortFlag);
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  const int s_idx = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool local = a.kind == BEAM_LOCAL;

  // key coordinates of the sequence (see above); an out-of-range pos0 has set the status in
  // the prologue and does nothing here (the whole CTA returns together).  pos0 is read before
  // pdl_wait() (the prologue does not write it; the kernels before the prologue have ended
  // when this one starts) and through L2, past any stale copy in this SM's L1.
  const int64_t p0 = __ldcg(a.pos0 + b);
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
    for (int i = 0; i < dtd::kNumBars; ++i) {
      uint32_t count = 1;
      if (i == dtd::kPFull || i == dtd::kPFull + 1) count = 128;
      if (i == dtd::kQReady) count = 256;
      if (i >= dtd::kVReady && i < dtd::kVReady + kDtVSlots) count = kDtConvThreads;
      tc::mbar_init(bar(i), count);
    }
    *abort = 0u;
    tc::fence_barrier_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(sbase + kDtSmemBar + dtd::kTmemHolder, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sgen + kDtSmemBar + dtd::kTmemHolder);
  // everything above overlaps the prologue (launched just before, with programmatic
  // serialization); from here on its outputs -- new cache rows, workspace rows, RoPE table,
  // merge tickets -- are read
  pdl_wait();
  // the P V MMAs read a value slot once its tile is in the operand format: straight from TMA
  // for a bf16 cache, after the in-place widening for an FP8 one (key tiles: from TMA always)
  constexpr int kVRdy = kFp8 ? dtd::kVReady : dtd::kVFull;

  // the register split (kDtRowRegs / kDtAuxRegs), set at the top of each role
  if (warp == 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kDtAuxRegs) : "memory");
    // ------------------------------------------------------------ K/V producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      auto load = [&](bool is_v, int j, uint32_t slot) {
        const int key0 = (int)(key_lo + (int64_t)j * kTcBN);
        const uint32_t full = bar((is_v ? dtd::kVFull : dtd::kKFull) + slot);
        const uint32_t dst = sbase + (is_v ? kDtSmemV : kDtSmemK) + slot * kTcTileBytes;
        const CUtensorMap *map = is_v ? &tm_v : &tm_k;
        if constexpr (kFp8) {   // key codes at the slot's start, value codes in its second half
          tc::mbar_expect_tx(full, kDtCodeTile);
          tc::tma_load_4d(dst + (is_v ? kTcHalfBytes : 0u), map, full, 0, key0, g, b);
        } else {
          tc::mbar_expect_tx(full, kTcTileBytes);
          for (int hf = 0; hf < 2; ++hf) {
            if (a.kv_slot_major)
              tc::tma_load_4d(dst + hf * kTcHalfBytes, map, full, hf * 64, key0, g, b);
            else
              tc::tma_load_4d(dst + hf * kTcHalfBytes, map, full, hf * 64, g, key0, b);
          }
        }
      };
      // Each ring refills on its own, a tile as soon as its slot is free (a value slot is held
      // until its P V is done, which comes two blocks after the key tile of that block is
      // used), polled without blocking; the wait is bounded like tc_wait's.
      int ik = 0, iv = 0;
      uint64_t t0 = 0;
      for (uint32_t spin = 0; ik < nb || iv < nb;) {
        bool moved = false;
        if (ik < nb && (ik < kDtKSlots || tc::mbar_test_wait(bar(dtd::kKEmpty + ik % kDtKSlots),
                                                             (ik / kDtKSlots - 1) & 1u))) {
          load(false, ik, ik % kDtKSlots);
          ++ik;
          moved = true;
        }
        if (iv < ik && (iv < kDtVSlots || tc::mbar_test_wait(bar(dtd::kVEmpty + iv % kDtVSlots),
                                                             (iv / kDtVSlots - 1) & 1u))) {
          load(true, iv, iv % kDtVSlots);
          ++iv;
          moved = true;
        }
        if (moved) {
          spin = 0;
          t0 = 0;
          continue;
        }
        if (*abort) break;
        if ((++spin & 1023u) == 0) {
          const uint64_t t = globaltimer_ns();
          if (t0 == 0) {
            t0 = t;
          } else if (t - t0 > kTcWaitNs || spin >= kTcSpinLimit) {
            set_status(a.status, BEAM_ERR_DEVICE_TIMEOUT);
            *abort = 1u;
            break;
          }
        }
      }
      for (int sl = 0; sl < kDtKSlots; ++sl)
        tc_drain(bar(dtd::kKFull + sl), (uint32_t)(ik + kDtKSlots - 1 - sl) / kDtKSlots, a.status);
      for (int sl = 0; sl < kDtVSlots; ++sl)
        tc_drain(bar(dtd::kVFull + sl), (uint32_t)(iv + kDtVSlots - 1 - sl) / kDtVSlots, a.status);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kDtAuxRegs) : "memory");
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = kFp8 ? tc::idesc_f16(128, 128, false, true)
                                         : tc::idesc_bf16(128, 128, false, true);
      auto kdesc = [&](uint32_t tile, int ks) {  // K-major, 128 B rows, 8-row groups 1 KiB apart
        return tc::sdesc_sw128(tile + (ks >> 2) * kTcHalfBytes + (ks & 3) * 32, 16, 1024);
      };
      auto vdesc = [&](uint32_t tile, int kk) {  // MN-major: d halves 16 KiB apart
        return tc::sdesc_sw128(tile + kk * 2048, kTcHalfBytes, 1024);
      };
      const uint32_t qt = sbase + kDtSmemQ;
      auto issue_s = [&](int j) {   // S(j) into S buffer j % 2
        const uint32_t kt = sbase + kDtSmemK + (j % kDtKSlots) * kTcTileBytes;
        const uint32_t d = tmem + 128 * (j & 1);
        if constexpr (kFp8) {
          // E4M3 x E4M3, 32 codes of d per MMA: the hi terms, then the lo terms (the second
          // 128 x 128 code tile of the Q area) into the same accumulator
          constexpr uint32_t idesc8 = tc::idesc_e4m3(128, 128);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::umma_ss_f8(d, tc::sdesc_sw128(qt + (ks >> 2) * kTcHalfBytes + (ks & 3) * 32, 16, 1024),
                           tc::sdesc_sw128(kt + (ks & 3) * 32, 16, 1024), idesc8, ks > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::umma_ss(d, kdesc(qt, ks), kdesc(kt, ks), idesc_qk, ks > 0 ? 1u : 0u);
        }
        tc::umma_commit(bar(dtd::kSFull + (j & 1)));
        tc::umma_commit(bar(dtd::kKEmpty + j % kDtKSlots));
      };
      auto issue_pv = [&](int j) {   // O_{j % 2} += P(j) V(j); the set's first block overwrites
        const uint32_t vt = sbase + kDtSmemV + (j % kDtVSlots) * kTcTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::umma_ts(tmem + 256 + 128 * (j & 1), tmem + 128 * (j & 1) + kk * 8, vdesc(vt, kk),
                      idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
        tc::umma_commit(bar(dtd::kPVDone + (j & 1)));
        tc::umma_commit(bar(dtd::kVEmpty + j % kDtVSlots));
      };
      bool ok = (!a.fault_stall || tc_wait(bar(dtd::kStall), 0u, abort, a.status)) &&
                tc_wait(bar(dtd::kQReady), 0u, abort, a.status);
      for (int jj = 0; ok && jj < 2 && jj < nb; ++jj) {
        if (!(ok = tc_wait(bar(dtd::kKFull + jj % kDtKSlots), (jj / kDtKSlots) & 1u, abort,
                           a.status)))
          break;
        tc::tc_fence_after();
        issue_s(jj);
      }
      for (int j = 0; ok && j < nb; ++j) {
        if (!(ok = tc_wait(bar(dtd::kPFull + (j & 1)), (j >> 1) & 1u, abort, a.status))) break;
        if (!(ok = tc_wait(bar(kVRdy + j % kDtVSlots), (j / kDtVSlots) & 1u, abort, a.status)))
          break;
        tc::tc_fence_after();
        issue_pv(j);
        if (j + 2 < nb) {
          const int j2 = j + 2;
          if (!(ok = tc_wait(bar(dtd::kKFull + j2 % kDtKSlots), (j2 / kDtKSlots) & 1u, abort,
                             a.status)))
            break;
          tc::tc_fence_after();
          issue_s(j2);
        }
      }
      if (ok) tc::umma_commit(bar(dtd::kOFull));
      tc::umma_commit(bar(dtd::kDrain));
      tc_drain(bar(dtd::kDrain), 1, a.status);
    }
    __syncwarp();
  } else if (warp >= 10) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kDtAuxRegs) : "memory");
    if constexpr (kFp8) {
      // ------------------------------------------------------------ FP8 values widened in place
      // Value tiles in order.  The code tile sits in the slot's second half, row r at 128 r
      // (128-byte swizzle: 16-code chunk c at (c ^ (r % 8)) * 16); the f16 tile is two halves
      // of 64 columns, row r of half h at h * 16 KiB + 128 r -- the code row's own bytes for
      // h = 1 -- so each thread widens whole rows (ct and ct + 64), all eight chunks read
      // before any is written.  Keys past the last visible one become zeros (0 times a NaN
      // code would poison a masked key).
      const int ct = threadIdx.x - 320;   // 0 .. 63
      for (int j = 0; j < nb; ++j) {
        const uint32_t slot = (uint32_t)j % kDtVSlots;
        if (!tc_wait(bar(dtd::kVFull + slot), (j / kDtVSlots) & 1u, abort, a.status)) break;
        uint8_t *tile = sgen + kDtSmemV + slot * kTcTileBytes;
        const int64_t key_first = key_lo + (int64_t)j * kTcBN;
#pragma unroll 1
        for (int rr = 0; rr < 2; ++rr) {
          const int r = ct + 64 * rr, sw = r & 7;
          uint8_t *row = tile + r * 128;
          uint4 w[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            w[c] = *reinterpret_cast<const uint4 *>(row + kTcHalfBytes + ((c ^ sw) << 4));
          const bool dead = key_first + r > hi_all;
#pragma unroll
          for (int c = 0; c < 8; ++c) {   // codes 16 c .. 16 c + 15 -> f16 chunks 2 c, 2 c + 1
            const uint32_t wv[4] = {dead ? 0u : w[c].x, dead ? 0u : w[c].y, dead ? 0u : w[c].z,
                                    dead ? 0u : w[c].w};
            uint32_t hx[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              hx[2 * e] = e4m3x2_to_f16x2(wv[e] & 0xFFFFu);
              hx[2 * e + 1] = e4m3x2_to_f16x2(wv[e] >> 16);
            }
            uint8_t *dst = row + (c >> 2) * kTcHalfBytes;
            const int q = (c & 3) * 2;
            *reinterpret_cast<uint4 *>(dst + ((q ^ sw) << 4)) = make_uint4(hx[0], hx[1], hx[2], hx[3]);
            *reinterpret_cast<uint4 *>(dst + (((q + 1) ^ sw) << 4)) =
                make_uint4(hx[4], hx[5], hx[6], hx[7]);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        tc::mbar_arrive(bar(dtd::kVReady + slot));
      }
    }
  } else {
    // ------------------------------------------------------------ rows (sets A and B)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kDtRowRegs) : "memory");
    const int set = warp >> 2;             // 0: warps 0-3 (even blocks), 1: warps 4-7 (odd)
    const int wq = warp & 3;               // tensor-memory lane quarter of this warp
    const int r = wq * 32 + lane;          // row = tensor-memory lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int k = r;                       // the (token, head) pair of this row: k = 6 i + h
    const int tok = k / kGroup, hh = k - tok * kGroup;
    const bool row_ok = tok < a.T;
    {
      // ---- the queries: RMSNorm, RoPE for a local layer, into the Q tile.  All 256 row
      // threads take part, two to a row: thread (qr, half) takes coordinates
      // 32 half .. 32 half + 31 and their partners 64 + 32 half .. (the row's sums of squares
      // and, over an FP8 cache, its largest pair norm are combined across the pair)
      const int qr = (warp * 32 + lane) >> 1, half = lane & 1;
      const int qtok = qr / kGroup, qhh = qr - qtok * kGroup;
      const bool q_ok = qtok < a.T;
      const uint4 *src = reinterpret_cast<const uint4 *>(
          a.q_raw + (((size_t)b * a.T + (q_ok ? qtok : 0)) * kHq + g * kGroup + qhh) * kD);
      uint4 qv[8];   // chunks 4 half .. 4 half + 3 (qv[0..3]) and 8 + 4 half .. (qv[4..7])
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        qv[c] = q_ok ? __ldg(src + (c < 4 ? 4 * half + c : 8 + 4 * half + (c - 4)))
                     : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w4[4] = {qv[c].x, qv[c].y, qv[c].z, qv[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(bf16_lo(w4[e]), bf16_lo(w4[e]), fmaf(bf16_hi(w4[e]), bf16_hi(w4[e]), ss));
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      const float inv = rsqrtf(ss * (1.0f / kD) + a.eps);
      const float4 *w4p = reinterpret_cast<const float4 *>(a.qw);
      // the RoPE table is angle-major: (cos, sin) of angle i of this token's row at
      // i * (B * T) + b * T + tok
      const size_t rope_stride = (size_t)gridDim.z * a.T;
      const float2 *tab = local ? reinterpret_cast<const float2 *>(a.rope_tab) +
                                      (size_t)b * a.T + (q_ok ? qtok : 0)
                                : nullptr;
      // coordinates 8c .. 8c+7 (xl) and their partners 64 + 8c .. (xh), c = 4 half + cc:
      // normalised, weighted and, when rot, rotated
      auto coords = [&](int cc, float (&xl)[8], float (&xh)[8], bool rot) {
        const int c = 4 * half + cc;
        const uint32_t lw[4] = {qv[cc].x, qv[cc].y, qv[cc].z, qv[cc].w};
        const uint32_t hw[4] = {qv[cc + 4].x, qv[cc + 4].y, qv[cc + 4].z, qv[cc + 4].w};
        const float4 wl0 = __ldg(w4p + 2 * c), wl1 = __ldg(w4p + 2 * c + 1);
        const float4 wh0 = __ldg(w4p + 16 + 2 * c), wh1 = __ldg(w4p + 16 + 2 * c + 1);
        const float wl[8] = {wl0.x, wl0.y, wl0.z, wl0.w, wl1.x, wl1.y, wl1.z, wl1.w};
        const float wh[8] = {wh0.x, wh0.y, wh0.z, wh0.w, wh1.x, wh1.y, wh1.z, wh1.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          xl[2 * e] = bf16_lo(lw[e]) * inv * wl[2 * e];
          xl[2 * e + 1] = bf16_hi(lw[e]) * inv * wl[2 * e + 1];
          xh[2 * e] = bf16_lo(hw[e]) * inv * wh[2 * e];
          xh[2 * e + 1] = bf16_hi(hw[e]) * inv * wh[2 * e + 1];
        }
        if (rot) {  // rotate-half: coordinate i < 64 pairs with i + 64
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 cs = __ldg(tab + (size_t)(8 * c + e) * rope_stride);
            const float a0 = xl[e], b0 = xh[e];
            xl[e] = a0 * cs.x - b0 * cs.y;
            xh[e] = b0 * cs.x + a0 * cs.y;
          }
        }
      };
      if constexpr (kFp8) {
        // the row's scale s: a rotation keeps each pair's norm, so the largest pair norm
        // bounds every coordinate before and after RoPE
        float m2 = 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float xl[8], xh[8];
          coords(cc, xl, xh, false);
#pragma unroll
          for (int e = 0; e < 8; ++e) m2 = fmaxf(m2, fmaf(xl[e], xl[e], xh[e] * xh[e]));
        }
        m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, 1));
        int ex;
        frexpf(sqrtf(m2), &ex);                       // largest |coordinate| < 2^ex
        const int sk = max(-100, min(100, 7 - ex));   // s = 2^sk: into [64, 128)
        const float qs = ldexpf(1.0f, sk);
        if (half == 0) reinterpret_cast<float *>(sgen + kDtSmemRowScale)[qr] = ldexpf(1.0f, -sk);
        // s q = hi + lo, 16 coordinates (one 16-byte chunk of codes) at a time
        auto split16 = [&](const float (&x0)[8], const float (&x1)[8], int chunk) {
          const uint2 h0 = f32x8_to_e4m3(x0, qs), h1 = f32x8_to_e4m3(x1, qs);
          const uint32_t hw[8] = {h0.x & 0xFFFFu, h0.x >> 16, h0.y & 0xFFFFu, h0.y >> 16,
                                  h1.x & 0xFFFFu, h1.x >> 16, h1.y & 0xFFFFu, h1.y >> 16};
          float r0[8], r1[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {   // residuals s q - hi, exact in fp32
            const uint32_t a2 = e4m3x2_to_f16x2(hw[e]), b2 = e4m3x2_to_f16x2(hw[e + 4]);
            r0[2 * e] = fmaf(x0[2 * e], qs, -__half2float(__ushort_as_half(a2 & 0xFFFFu)));
            r0[2 * e + 1] = fmaf(x0[2 * e + 1], qs, -__half2float(__ushort_as_half(a2 >> 16)));
            r1[2 * e] = fmaf(x1[2 * e], qs, -__half2float(__ushort_as_half(b2 & 0xFFFFu)));
            r1[2 * e + 1] = fmaf(x1[2 * e + 1], qs, -__half2float(__ushort_as_half(b2 >> 16)));
          }
          const uint2 l0 = f32x8_to_e4m3(r0, 1.0f), l1 = f32x8_to_e4m3(r1, 1.0f);
          const uint32_t off = qr * 128 + ((chunk ^ (qr & 7)) << 4);
          *reinterpret_cast<uint4 *>(sgen + kDtSmemQ + off) = make_uint4(h0.x, h0.y, h1.x, h1.y);
          *reinterpret_cast<uint4 *>(sgen + kDtSmemQ + kTcHalfBytes + off) =
              make_uint4(l0.x, l0.y, l1.x, l1.y);
        };
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {   // coordinates 16 m .. 16 m + 15 and 64 + 16 m .., m = 2 half + mm
          float al[8], ah[8], bl[8], bh[8];
          coords(2 * mm, al, ah, local);
          coords(2 * mm + 1, bl, bh, local);
          split16(al, bl, 2 * half + mm);
          split16(ah, bh, 4 + 2 * half + mm);
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float xl[8], xh[8];
          coords(cc, xl, xh, local);
          const uint32_t sw = (uint32_t)(((4 * half + cc) ^ (qr & 7)) << 4);
          *reinterpret_cast<uint4 *>(sgen + kDtSmemQ + qr * 128 + sw) =
              make_uint4(pack_bf16(xl[0], xl[1]), pack_bf16(xl[2], xl[3]),
                         pack_bf16(xl[4], xl[5]), pack_bf16(xl[6], xl[7]));
          *reinterpret_cast<uint4 *>(sgen + kDtSmemQ + kTcHalfBytes + qr * 128 + sw) =
              make_uint4(pack_bf16(xh[0], xh[1]), pack_bf16(xh[2], xh[3]),
                         pack_bf16(xh[4], xh[5]), pack_bf16(xh[6], xh[7]));
        }
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      tc::mbar_arrive(bar(dtd::kQReady));
    }
    bool ok = true;
    // this row's visible coordinates, relative to key_lo (empty for a padding row)
    int rlo = 0, rhi = -1;
    float factor = a.scale_log2 * a.k_scale;
    if constexpr (kFp8) {   // 1 / s of the row, written before the Q-ready arrivals
      ok = tc_wait(bar(dtd::kQReady), 0u, abort, a.status);
      factor *= reinterpret_cast<const float *>(sgen + kDtSmemRowScale)[r];
    }
    if (row_ok) {
      const int64_t hi = kq + tok;
      const int64_t lo = local ? max(hi - a.window + 1, lo_all) : 0;
      rhi = (int)max((int64_t)-1, min(hi - key_lo, (int64_t)a.split));
      rlo = (int)max((int64_t)0, min(lo - key_lo, (int64_t)a.split + 1));
      if (!local) factor *= ssmax_factor(p0 + tok + 1, a.ssmax_base, a.ssmax_exp);
    }
    const uint32_t t_s = tmem + lane_off + 128 * set;
    const uint32_t t_o = tmem + lane_off + 256 + 128 * set;
    float m = -INFINITY, l = 0.f;
    // A warp whose 32 rows are all padding (6 T <= 32 wq) only keeps the barrier phases: its
    // P rows are whatever its S rows hold, and P V never mixes rows, so only these rows' O
    // (never read) sees them.  It leaves the special-function units to the real rows.
    const bool warp_rows = __any_sync(0xffffffffu, row_ok);
    for (int j = set; ok && j < nb; j += 2) {
      if (!(ok = __all_sync(0xffffffffu,
                            tc_wait(bar(dtd::kSFull + set), (j >> 1) & 1u, abort, a.status))))
        break;
      if (!warp_rows) {
        tc::mbar_arrive(bar(dtd::kPFull + set));
        continue;
      }
      tc::tc_fence_after();
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
      if (j < 2) {
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
      // O_set *= alpha for the rows whose max moved by more than 2^8, once O_set holds this
      // set's previous block (block j - 2)
      if (j >= 2 && __any_sync(0xffffffffu, rescale)) {
        if (!(ok = __all_sync(0xffffffffu, tc_wait(bar(dtd::kPVDone + set), ((j >> 1) - 1) & 1u,
                                                   abort, a.status))))
          break;
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
      tc::mbar_arrive(bar(dtd::kPFull + set));
    }
    if (ok) ok = tc_wait(bar(dtd::kOFull), 0u, abort, a.status);
    // ---- merge of the two sets: set B hands its (m, l) over through shared memory (the Q
    // tile is free once every MMA is done); set A combines O_A and O_B
    float *ml_b = reinterpret_cast<float *>(sgen + kDtSmemQ);   // [128][2]
    if (set == 1) {
      ml_b[2 * r] = m;
      ml_b[2 * r + 1] = l;
    }
    asm volatile("bar.sync 1, 256;\n" ::: "memory");
    if (set == 1) {
      // nothing more: set A writes the row
    } else {
      const bool has_b = nb > 1;   // with one block set B never wrote O_B
      const float mb = has_b ? ml_b[2 * r] : -INFINITY, lb = has_b ? ml_b[2 * r + 1] : 0.f;
      const float M = fmaxf(m, mb);
      const float Mu = M == -INFINITY ? 0.f : M;
      const float wa = ex2_approx(m - Mu), wb = has_b ? ex2_approx(mb - Mu) : 0.f;
      const float L = wa * l + wb * lb;
      const uint32_t t_oa = tmem + lane_off + 256, t_ob = tmem + lane_off + 384;
      auto o_chunk = [&](int c, uint32_t (&o)[32]) {   // wa O_A + wb O_B, columns 32 c ..
        tc::tmem_ld32(t_oa + 32 * c, o);
        tc::tmem_ld_wait();
        if (has_b) {
          uint32_t ob[32];
          tc::tmem_ld32(t_ob + 32 * c, ob);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            o[i] = __float_as_uint(fmaf(wa, __uint_as_float(o[i]), wb * __uint_as_float(ob[i])));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(wa * __uint_as_float(o[i]));
        }
      };
      if (a.direct) {
        // the whole key range: Y = O / L * sigmoid(G + b_h) straight to the output row (not
        // written when a wait ran out)
        if (ok) {
          tc::tc_fence_after();
          const int h = g * kGroup + hh;
          const size_t orow = (((size_t)b * a.T + (row_ok ? tok : 0)) * kHq + h) * kD;
          const uint4 *gp = reinterpret_cast<const uint4 *>(a.gate + orow);
          uint4 *op = reinterpret_cast<uint4 *>(a.out + orow);
          const float inv = a.v_scale / L, bias = a.gate_bias[h];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            o_chunk(c, o);
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
      } else {
        const int mt = tok / kMultiTokPerTile, row16 = (tok % kMultiTokPerTile) * kGroup + hh;
        const size_t part =
            ((((size_t)b * kHkv + g) * a.n_mt + mt) * a.n_split_max + s_idx) * 16 + row16;
        if (!ok && row_ok) {   // a wait ran out: the merge turns these rows into NaN
          a.part_ml[part * 2] = __int_as_float(0x7fc00000);
          a.part_ml[part * 2 + 1] = __int_as_float(0x7fc00000);
        }
        if (ok) {
          tc::tc_fence_after();
          const float vs = a.v_scale;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            o_chunk(c, o);
            if (row_ok) {
              float4 *dst = reinterpret_cast<float4 *>(a.part_o + part * kD + 32 * c);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(__uint_as_float(o[4 * q]) * vs, __uint_as_float(o[4 * q + 1]) * vs,
                                     __uint_as_float(o[4 * q + 2]) * vs, __uint_as_float(o[4 * q + 3]) * vs);
            }
          }
          if (row_ok) {
            a.part_ml[part * 2] = M;
            a.part_ml[part * 2 + 1] = L;
          }
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
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
