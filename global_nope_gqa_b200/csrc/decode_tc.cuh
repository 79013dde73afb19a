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
// decode_multi_combine_kernel merges the runs and gates.  Every wait is bounded (tc_wait: 1 s
// of device time, then BEAM_ERR_DEVICE_TIMEOUT, an abort flag for the other roles, and the
// in-flight copies and MMAs drained before the tensor memory is freed).
#pragma once

#include "common.cuh"
#include "decode_multi.cuh"
#include "prefill_tc.cuh"
#include "tc_ptx.cuh"

namespace beam {

constexpr int kDtThreads = 192;
constexpr int kDtKSlots = 3, kDtVSlots = 3;
constexpr uint32_t kDtSmemQ = 0;                                    // one 128 x 128 Q tile
constexpr uint32_t kDtSmemK = kTcTileBytes;                         // K ring
constexpr uint32_t kDtSmemV = kDtSmemK + kDtKSlots * kTcTileBytes;  // V ring
constexpr uint32_t kDtSmemBar = kDtSmemV + kDtVSlots * kTcTileBytes;
constexpr uint32_t kDtSmemBytes = kDtSmemBar + 256 + 1024;          // 230,656 B

namespace dtd {  // barrier slots (8 bytes each) after kDtSmemBar, laid out from the ring sizes
constexpr int kKFull = 0, kKEmpty = kKFull + kDtKSlots, kVFull = kKEmpty + kDtKSlots,
              kVEmpty = kVFull + kDtVSlots, kSFull = kVEmpty + kDtVSlots, kPFull = kSFull + 2,
              kPVDone = kPFull + 2, kOFull = kPVDone + 1, kQReady = kOFull + 1,
              kDrain = kQReady + 1, kStall = kDrain + 1, kNumBars = kStall + 1;
static_assert(kNumBars * 8 + 8 <= 256, "the barrier area holds 256 bytes");
constexpr uint32_t kTmemHolder = kNumBars * 8;
constexpr uint32_t kAbortFlag = kTmemHolder + 4;
}  // namespace dtd

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
};

__global__ void __launch_bounds__(kDtThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeTcArgs a) {
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
    for (int i = 0; i < dtd::kNumBars; ++i)
      tc::mbar_init(bar(i), (i == dtd::kPFull || i == dtd::kPFull + 1 || i == dtd::kQReady) ? 128 : 1);
    *abort = 0u;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + kDtSmemBar + dtd::kTmemHolder, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sgen + kDtSmemBar + dtd::kTmemHolder);

  if (warp == 0) {
    // ------------------------------------------------------------ K/V producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      auto load = [&](bool is_v, int j, uint32_t slot) {
        const int key0 = (int)(key_lo + (int64_t)j * kTcBN);
        const uint32_t full = bar((is_v ? dtd::kVFull : dtd::kKFull) + slot);
        tc::mbar_expect_tx(full, kTcTileBytes);
        const uint32_t dst = sbase + (is_v ? kDtSmemV : kDtSmemK) + slot * kTcTileBytes;
        const CUtensorMap *map = is_v ? &tm_v : &tm_k;
        for (int hf = 0; hf < 2; ++hf) {
          if (a.kv_slot_major)
            tc::tma_load_4d(dst + hf * kTcHalfBytes, map, full, hf * 64, key0, g, b);
          else
            tc::tma_load_4d(dst + hf * kTcHalfBytes, map, full, hf * 64, g, key0, b);
        }
      };
      int ik = 0, iv = 0;
      bool ok = true;
      for (; ik < 2 && ik < nb; ++ik) load(false, ik, ik % kDtKSlots);
      while (ok && iv < nb) {
        if (ik < nb) {
          const uint32_t slot = ik % kDtKSlots;
          if (ik >= kDtKSlots && !(ok = tc_wait(bar(dtd::kKEmpty + slot),
                                                (ik / kDtKSlots - 1) & 1u, abort, a.status)))
            break;
          load(false, ik, slot);
          ++ik;
        }
        const uint32_t slot = iv % kDtVSlots;
        if (iv >= kDtVSlots &&
            !(ok = tc_wait(bar(dtd::kVEmpty + slot), (iv / kDtVSlots - 1) & 1u, abort, a.status)))
          break;
        load(true, iv, slot);
        ++iv;
      }
      for (int sl = 0; sl < kDtKSlots; ++sl)
        tc_drain(bar(dtd::kKFull + sl), (uint32_t)(ik + kDtKSlots - 1 - sl) / kDtKSlots, a.status);
      for (int sl = 0; sl < kDtVSlots; ++sl)
        tc_drain(bar(dtd::kVFull + sl), (uint32_t)(iv + kDtVSlots - 1 - sl) / kDtVSlots, a.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(128, 128, false, true);
      auto kdesc = [&](uint32_t tile, int ks) {  // K-major, 128 B rows, 8-row groups 1 KiB apart
        return tc::sdesc_sw128(tile + (ks >> 2) * kTcHalfBytes + (ks & 3) * 32, 16, 1024);
      };
      auto vdesc = [&](uint32_t tile, int kk) {  // MN-major: d halves 16 KiB apart
        return tc::sdesc_sw128(tile + kk * 2048, kTcHalfBytes, 1024);
      };
      const uint32_t qt = sbase + kDtSmemQ;
      auto issue_s = [&](int j) {
        const uint32_t kt = sbase + kDtSmemK + (j % kDtKSlots) * kTcTileBytes;
        const uint32_t d = tmem + 128 * (j & 1);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::umma_ss(d, kdesc(qt, ks), kdesc(kt, ks), idesc_qk, ks > 0 ? 1u : 0u);
        tc::umma_commit(bar(dtd::kSFull + (j & 1)));
        tc::umma_commit(bar(dtd::kKEmpty + j % kDtKSlots));
      };
      auto issue_pv = [&](int j) {
        const uint32_t vt = sbase + kDtSmemV + (j % kDtVSlots) * kTcTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::umma_ts(tmem + 256, tmem + 128 * (j & 1) + kk * 8, vdesc(vt, kk), idesc_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
        tc::umma_commit(bar(dtd::kPVDone));
        tc::umma_commit(bar(dtd::kVEmpty + j % kDtVSlots));
        if (j == nb - 1) tc::umma_commit(bar(dtd::kOFull));
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
        if (!(ok = tc_wait(bar(dtd::kVFull + j % kDtVSlots), (j / kDtVSlots) & 1u, abort,
                           a.status)))
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
      tc::umma_commit(bar(dtd::kDrain));
      tc_drain(bar(dtd::kDrain), 1, a.status);
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
      const float4 *tab = local ? reinterpret_cast<const float4 *>(
                                      a.rope_tab + ((size_t)b * a.T + (row_ok ? tok : 0)) * 128)
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
          const float4 c0 = __ldg(tab + 2 * c), c1 = __ldg(tab + 2 * c + 1);
          const float4 s0 = __ldg(tab + 16 + 2 * c), s1 = __ldg(tab + 16 + 2 * c + 1);
          const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a0 = xl[e], b0 = xh[e];
            xl[e] = a0 * cv[e] - b0 * sv[e];
            xh[e] = b0 * cv[e] + a0 * sv[e];
          }
        }
        const uint32_t sw = (uint32_t)((c ^ (r & 7)) << 4);
        *reinterpret_cast<uint4 *>(sgen + kDtSmemQ + r * 128 + sw) =
            make_uint4(pack_bf16(xl[0], xl[1]), pack_bf16(xl[2], xl[3]), pack_bf16(xl[4], xl[5]),
                       pack_bf16(xl[6], xl[7]));
        *reinterpret_cast<uint4 *>(sgen + kDtSmemQ + kTcHalfBytes + r * 128 + sw) =
            make_uint4(pack_bf16(xh[0], xh[1]), pack_bf16(xh[2], xh[3]), pack_bf16(xh[4], xh[5]),
                       pack_bf16(xh[6], xh[7]));
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      tc::mbar_arrive(bar(dtd::kQReady));
    }
    // this row's visible coordinates, relative to key_lo (empty for a padding row)
    int rlo = 0, rhi = -1;
    float factor = a.scale_log2;
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
      if (!(ok = tc_wait(bar(dtd::kSFull + (j & 1)), (j >> 1) & 1u, abort, a.status))) break;
      tc::mbar_arrive(bar(dtd::kPFull + (j & 1)));
    }
    for (int j = 0; j < nb && warp_rows; ++j) {
      if (!(ok = tc_wait(bar(dtd::kSFull + (j & 1)), (j >> 1) & 1u, abort, a.status))) break;
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
          pk[i >> 1] = pack_bf16(p0v, p1v);
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
        if (!(ok = tc_wait(bar(dtd::kPVDone), (j - 1) & 1u, abort, a.status))) break;
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
      tc::mbar_arrive(bar(dtd::kPFull + (j & 1)));
    }
    if (ok) ok = tc_wait(bar(dtd::kOFull), 0u, abort, a.status);
    if (a.direct) {
      // the whole key range: Y = O / l * sigmoid(G + b_h) straight to the output row (not
      // written when a wait ran out)
      if (ok) {
        tc::tc_fence_after();
        const int h = g * kGroup + hh;
        const size_t orow = (((size_t)b * a.T + (row_ok ? tok : 0)) * kHq + h) * kD;
        const uint4 *gp = reinterpret_cast<const uint4 *>(a.gate + orow);
        uint4 *op = reinterpret_cast<uint4 *>(a.out + orow);
        const float inv = 1.0f / l, bias = a.gate_bias[h];
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
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                 __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
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
}

}  // namespace beam
