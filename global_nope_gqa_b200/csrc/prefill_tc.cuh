// prefill_tc.cuh -- flash-attention prefill on tcgen05 tensor cores (TMEM accumulators,
// TMA-staged operands), sm_100a.
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax": every query row attends over
// its visible keys (section "Two attention paths in one decoder": keys t-511 .. t in a
// local layer, 0 .. t in a global layer); query head h reads KV head h/6; the output is
// Y = O * sigmoid(G + b_h) per coordinate (section "Follow the tensors").  The global
// layer's scalable-softmax factor a(t+1) multiplies each row's fp32 score scale.
//
// One CTA = 128 query rows x two query heads of one GQA group (two 128 x 128 Q tiles that
// share every K/V tile), 384 threads in warp roles:
//   warp 0      TMA producer: Q tiles once, then K and V tiles of 128 keys into a
//               two-stage ring (128-byte swizzled boxes of 128 rows x 64 columns);
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T (both operands in shared memory)
//               and O_t += P_t V (P from tensor memory, V in shared memory), t = 0, 1;
//               the whole warp also allocates and frees the 512 tensor-memory columns:
//               S_0 [0,128) S_1 [128,256) O_0 [256,384) O_1 [384,512) (fp32), with P_t
//               written as bf16 pairs over the first 64 columns of S_t;
//   warps 2-3   idle;
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one thread per query row
//               (tensor-memory lane = row; warp % 4 picks the lane quarter a warp may use).  Each reads its S row, masks the window /
//               causal edge, keeps the online max m and sum l in exp2 units, writes P and,
//               only when the row max grew by more than 2^8, rescales its O row in tensor
//               memory first (the stale max keeps every P <= 256, safe in fp32 and bf16).
//               The last block's wait also serves as the epilogue: O/l * sigmoid(G + b).
// MMAs issued by one thread run in issue order, so S_t(j+1), which overwrites P_t(j),
// is issued after O_t += P_t(j) V_j; the commit that publishes S_t(j) also covers the
// O_t update of block j-1, which lets the softmax rescale O_t without a further wait.
// Key blocks entirely outside the window or the causal triangle are never loaded.
// Every mbarrier wait is bounded; a wait that runs out sets BEAM_ERR_DEVICE_TIMEOUT in
// the status word, raises an abort flag that the other roles also watch, and the CTA
// still frees its tensor memory before it returns.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace beam {

constexpr int kTcThreads = 384;
constexpr int kTcBM = 128;      // query rows per tile
constexpr int kTcBN = 128;      // keys per block
constexpr uint32_t kTcTileBytes = 128 * 128 * 2;   // 32 KiB: one 128 x 128 bf16 tile
constexpr uint32_t kTcHalfBytes = kTcTileBytes / 2;  // one 128 x 64 TMA box
constexpr uint32_t kTcSmemQ = 0;                      // Q_0, Q_1
constexpr uint32_t kTcSmemK = 2 * kTcTileBytes;       // K stage 0, 1
constexpr uint32_t kTcSmemV = 4 * kTcTileBytes;       // V stage 0, 1
constexpr uint32_t kTcSmemBar = 6 * kTcTileBytes;     // mbarriers
constexpr uint32_t kTcSmemBytes = kTcSmemBar + 256 + 1024;  // + barriers + alignment slack
constexpr uint32_t kTcSpinLimit = 1u << 22;

struct PrefillTcArgs {
  const uint16_t *gate;   // [B][T][48*128]
  const float *gate_bias; // [48]
  uint16_t *out;          // [B][T][48*128]
  int32_t *status;
  int T, kind, window, n_qblocks;
  float scale_log2, ssmax_base, ssmax_exp;
};

namespace tcd {
// barrier slots (8 bytes each) after kTcSmemBar
constexpr int kQFull = 0, kKFull = 1, kVFull = 3, kKVEmpty = 5, kSFull = 7, kPFull = 9,
              kOFull = 11, kNumBars = 13;
constexpr uint32_t kTmemHolder = kNumBars * 8;      // u32: tensor-memory base address
constexpr uint32_t kAbortFlag = kTmemHolder + 4;    // u32: set when a wait ran out
}  // namespace tcd

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait on an mbarrier phase; false when it ran out or another role aborted.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile uint32_t *abort,
                                        int32_t *status) {
  for (uint32_t i = 0; i < kTcSpinLimit; ++i) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
  }
  set_status(status, BEAM_ERR_DEVICE_TIMEOUT);
  *abort = 1u;
  return false;
}

__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrefillTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // SW128 tiles need 1024-byte alignment
  uint8_t *sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + kTcSmemBar;
  volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sgen + kTcSmemBar + tcd::kAbortFlag);
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x % (kHq / 2), b = blockIdx.x / (kHq / 2);
  const int qb = a.n_qblocks - 1 - (int)blockIdx.y;  // longest rows first
  const int h0 = 2 * pair, g = h0 / kGroup;
  const int q0 = qb * kTcBM;
  const bool local = a.kind == BEAM_LOCAL;
  const int kb_lo = local ? max(0, q0 - a.window + 1) / kTcBN : 0;
  const int kb_hi = qb;  // q_last = min(T, q0 + 128) - 1 < (qb + 1) * 128
  const int n_blk = kb_hi - kb_lo + 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < tcd::kNumBars; ++i) {
      uint32_t count = 1;
      if (i == tcd::kPFull || i == tcd::kPFull + 1) count = 128;
      tc::mbar_init(bar(i), count);
    }
    *abort = 0u;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sbase + kTcSmemBar + tcd::kTmemHolder, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sgen + kTcSmemBar + tcd::kTmemHolder);

  // Register split (per warpgroup): warps 0-3 (producer, MMA issuer, two idle) keep 56
  // registers, the softmax warpgroups get 224: 4*56 + 8*224 = 12*168, what the CTA is
  // launched with, and on every SM sub-partition 56 + 2*224 <= 512 registers per lane.
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      tc::mbar_expect_tx(bar(tcd::kQFull), 2 * kTcTileBytes);
      for (int t = 0; t < 2; ++t)
        for (int hf = 0; hf < 2; ++hf)
          tc::tma_load_4d(sbase + kTcSmemQ + t * kTcTileBytes + hf * kTcHalfBytes, &tm_q,
                          bar(tcd::kQFull), hf * 64, h0 + t, q0, b);
      for (int j = 0; j < n_blk; ++j) {
        const int s = j & 1;
        if (j >= 2 && !tc_wait(bar(tcd::kKVEmpty + s), ((j >> 1) - 1) & 1, abort, a.status)) break;
        const int key0 = (kb_lo + j) * kTcBN;
        tc::mbar_expect_tx(bar(tcd::kKFull + s), kTcTileBytes);
        for (int hf = 0; hf < 2; ++hf)
          tc::tma_load_4d(sbase + kTcSmemK + s * kTcTileBytes + hf * kTcHalfBytes, &tm_k,
                          bar(tcd::kKFull + s), hf * 64, g, key0, b);
        tc::mbar_expect_tx(bar(tcd::kVFull + s), kTcTileBytes);
        for (int hf = 0; hf < 2; ++hf)
          tc::tma_load_4d(sbase + kTcSmemV + s * kTcTileBytes + hf * kTcHalfBytes, &tm_v,
                          bar(tcd::kVFull + s), hf * 64, g, key0, b);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(128, 128, false, true);
      auto qk_desc = [&](uint32_t tile, int ks) {  // K-major, 128 B rows, 8-row groups 1 KiB apart
        return tc::sdesc_sw128(tile + (ks >> 2) * kTcHalfBytes + (ks & 3) * 32, 16, 1024);
      };
      auto v_desc = [&](uint32_t tile, int kk) {  // MN-major: d halves 16 KiB apart
        return tc::sdesc_sw128(tile + kk * 2048, kTcHalfBytes, 1024);
      };
      auto issue_pv = [&](int t, int jb) {
        const uint32_t vt = sbase + kTcSmemV + (jb & 1) * kTcTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::umma_ts(tmem + 256 + 128 * t, tmem + 128 * t + kk * 8, v_desc(vt, kk), idesc_pv,
                      (jb > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = tc_wait(bar(tcd::kQFull), 0, abort, a.status);
      for (int j = 0; ok && j < n_blk; ++j) {
        const int s = j & 1;
        if (!(ok = tc_wait(bar(tcd::kKFull + s), (j >> 1) & 1, abort, a.status))) break;
        tc::tc_fence_after();
        const uint32_t kt = sbase + kTcSmemK + s * kTcTileBytes;
        for (int t = 0; t < 2 && ok; ++t) {
          if (j > 0) {
            if (!(ok = tc_wait(bar(tcd::kPFull + t), (j - 1) & 1, abort, a.status))) break;
            if (t == 0 &&
                !(ok = tc_wait(bar(tcd::kVFull + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort, a.status)))
              break;
            tc::tc_fence_after();
            issue_pv(t, j - 1);
            if (t == 1) tc::umma_commit(bar(tcd::kKVEmpty + ((j - 1) & 1)));
          }
          const uint32_t qt = sbase + kTcSmemQ + t * kTcTileBytes;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::umma_ss(tmem + 128 * t, qk_desc(qt, ks), qk_desc(kt, ks), idesc_qk, ks > 0 ? 1u : 0u);
          tc::umma_commit(bar(tcd::kSFull + t));
        }
      }
      const int jl = n_blk - 1;
      for (int t = 0; t < 2 && ok; ++t) {
        if (!(ok = tc_wait(bar(tcd::kPFull + t), jl & 1, abort, a.status))) break;
        if (t == 0 && !(ok = tc_wait(bar(tcd::kVFull + (jl & 1)), (jl >> 1) & 1, abort, a.status)))
          break;
        tc::tc_fence_after();
        issue_pv(t, jl);
        tc::umma_commit(bar(tcd::kOFull + t));
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;\n" ::: "memory");
    const int t = (warp - 4) >> 2;      // tile: 0 for warps 4-7, 1 for warps 8-11
    const int wq = warp & 3;            // tensor-memory lane quarter this warp may access
    const int r = wq * 32 + lane;       // query row within the tile
    const int tok = q0 + r;
    const int h = h0 + t;
    float factor = a.scale_log2;
    if (!local) factor *= ssmax_factor((int64_t)tok + 1, a.ssmax_base, a.ssmax_exp);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t t_s = tmem + lane_off + 128 * t;
    const uint32_t t_o = tmem + lane_off + 256 + 128 * t;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_blk; ++j) {
      if (!(ok = tc_wait(bar(tcd::kSFull + t), j & 1, abort, a.status))) break;
      tc::tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32(t_s + 32 * c, sr[c]);
      tc::tmem_ld_wait();
      const int kb = kb_lo + j;
      const bool need_mask =
          kb == qb || (local && (q0 + kTcBM - 1) - kb * kTcBN > a.window - 1);
      if (need_mask) {
        // key kb*128 + i is visible to row tok iff lo <= i <= hi
        const int hi = tok - kb * kTcBN;
        const int lo = local ? tok - a.window + 1 - kb * kTcBN : INT_MIN;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kk = c * 32 + i;
            sr[c][i] = (kk >= lo && kk <= hi) ? sr[c][i] : 0xFF800000u;  // -inf
          }
      }
      // row max of the raw scores: eight independent chains of 3-input max
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
                             fmaxf(mc[6], mc[7])) * factor;   // factor > 0
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
      // P = exp2(s * factor - m) in fp32 pairs; bf16 pairs over the first 64 columns of S
      const uint64_t f2 = tc::f2_pack(factor, factor), nm2 = tc::f2_pack(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float y0, y1;
          tc::f2_unpack(tc::f2_fma(tc::f2_pack(__uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1])),
                                   f2, nm2), y0, y1);
          const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
          acc[(i >> 1) & 3] = tc::f2_add(acc[(i >> 1) & 3], tc::f2_pack(p0, p1));
          pk[i >> 1] = pack_bf16(p0, p1);
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
      // O *= alpha for the rows whose max moved by more than 2^8 (O is final through
      // the previous block: the commit that published S covers that MMA)
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
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
      tc::mbar_arrive(bar(tcd::kPFull + t));
    }
    if (ok) ok = tc_wait(bar(tcd::kOFull + t), 0, abort, a.status);
    if (ok) {
      tc::tc_fence_after();
      const float inv = 1.0f / l;
      const float bias = a.gate_bias[h];
      const bool valid = tok < a.T;
      const size_t row = ((size_t)b * a.T + (valid ? tok : 0)) * (kHq * kD) + (size_t)h * kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tc::tmem_ld32(t_o + 32 * c, o);
        tc::tmem_ld_wait();
        if (valid) {
          const uint4 *gp = reinterpret_cast<const uint4 *>(a.gate + row + c * 32);
          uint4 *op = reinterpret_cast<uint4 *>(a.out + row + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 gr = gp[q];
            const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w};
            uint32_t yw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float g0 = bf16_lo(gw[e]) + bias, g1 = bf16_hi(gw[e]) + bias;
              const float y0 = __uint_as_float(o[q * 8 + 2 * e]) * inv / (1.0f + __expf(-g0));
              const float y1 = __uint_as_float(o[q * 8 + 2 * e + 1]) * inv / (1.0f + __expf(-g1));
              yw[e] = pack_bf16(y0, y1);
            }
            op[q] = make_uint4(yw[0], yw[1], yw[2], yw[3]);
          }
        }
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
