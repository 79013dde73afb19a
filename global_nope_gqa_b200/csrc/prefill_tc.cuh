// prefill_tc.cuh -- flash-attention prefill on tcgen05 tensor cores (TMEM accumulators,
// TMA-staged operands), sm_100a.
//
// "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax": every query row attends over
// its visible keys (section "Two attention paths in one decoder": keys t-511 .. t in a
// local layer, 0 .. t in a global layer); query head h reads KV head h/6; the output is
// Y = O * sigmoid(G + b_h) per coordinate (section "Follow the tensors").  The global
// layer's scalable-softmax factor a(t+1) multiplies each row's fp32 score scale.
//
// Work unit: 128 query rows x two query heads of one GQA group -- two 128 x 128 Q tiles
// that share every K/V tile.  The kernel is persistent: one CTA per SM walks the units
// u = blockIdx.x, blockIdx.x + gridDim.x, ... in order of decreasing work (the causal
// triangle's longest rows first), so the next unit's loads and first Q K^T overlap the
// current unit's epilogue, and set-up (barriers, tensor memory) happens once.
// 512 threads in warp roles:
//   warp 0      K/V producer (TMA): K tiles of 128 keys into a two-slot ring running a
//               block ahead, V tiles into one slot (128-byte swizzled 128 x 64 boxes);
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T (both operands in shared memory)
//               and O_t += P_t V (P from tensor memory, V in shared memory), t = 0, 1;
//               the whole warp also allocates and frees the 512 tensor-memory columns:
//               S_0 [0,128) S_1 [128,256) O_0 [256,384) O_1 [384,512) (fp32), with P_t
//               written as bf16 pairs over the first 64 columns of S_t;
//   warp 2      Q producer (TMA): the raw Q tiles of unit n into Q set n % 2, so the next
//               unit's Q is loaded and prepared while the current unit runs;
//   warp 3      output store (TMA), global layer: the softmax threads stage a unit's Y
//               tiles in the unit's own Q set, whose Q is no longer read once O is final;
//               one thread stores both tiles (rows past T are clipped by the copy) and
//               hands the set back to the Q producer once the copies have read it.  A
//               local layer's units are short (at most five key blocks), too short to hide
//               that later release (the set's next Q must be loaded and prepared while the
//               following unit runs), so there the softmax threads store their rows
//               directly and the MMA issuer releases the set after the unit's last Q K^T;
//   warps 12-15 Q preparation: once a unit's raw Q tiles have landed, RMSNorm (and RoPE
//               with a per-position cos/sin table for a local layer) each row in place in
//               shared memory, then release the tiles to the MMA issuer;
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one thread per query row
//               (tensor-memory lane = row; warp % 4 picks the lane quarter a warp may use).
//               Each reads its S row, masks the window / causal edge, keeps the online max
//               m and sum l in exp2 units, writes P and, only when the row max grew by more
//               than 2^8, rescales its O row in tensor memory (the stale max keeps every
//               P <= 256, safe in fp32 and bf16).  After a unit's last block the same
//               threads run the epilogue O/l * sigmoid(G + b), release O and write Y
//               as bf16 rows, into the unit's Q tile t for the store warp or to HBM.
// MMAs issued by one thread run in issue order, so S_t(j+1), which overwrites P_t(j), is
// issued after O_t += P_t(j) V_j; the commit that publishes S_t(j) also covers the O_t
// update of block j-1, which lets the softmax rescale O_t without a further wait.  Key
// blocks entirely outside the window or the causal triangle are never loaded.
// Every mbarrier wait is bounded (about a second of device time); a wait that runs out sets
// BEAM_ERR_DEVICE_TIMEOUT in the status word and raises an abort flag that the other roles
// also watch.  Before the CTA returns, each producer waits (bounded again) for the tiles it
// issued to land and the MMA issuer for its MMAs to finish, so nothing writes shared or
// tensor memory after the CTA has freed it.  For tests of that path a launch may ask the
// MMA issuer to start with a wait on a barrier that nothing arrives at.
#pragma once

#include <climits>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace beam {

constexpr int kTcThreads = 512;
// Register split (setmaxnreg) per 128 threads: warps 0-3 56 each, the two softmax warpgroups
// 176, the Q-preparation warpgroup 104 -- exactly the 512 x 128 registers of the launch.
constexpr int kTcRegPool = 128 * (56 + 176 + 176 + 104);
static_assert(kTcRegPool <= kTcThreads * 128, "the split must fit the launch's registers");
constexpr int kTcBM = 128;      // query rows per tile
constexpr int kTcBN = 128;      // keys per block
constexpr uint32_t kTcTileBytes = 128 * 128 * 2;   // 32 KiB: one 128 x 128 bf16 tile
constexpr uint32_t kTcHalfBytes = kTcTileBytes / 2;  // one 128 x 64 TMA box
constexpr uint32_t kTcSmemQ = 0;                      // Q: 2 sets (units n even / odd) x 2 tiles
constexpr uint32_t kTcSmemKV = 4 * kTcTileBytes;      // K ring (slots 0, 1) and V slot (2)
constexpr uint32_t kTcKVSlots = 3;
constexpr uint32_t kTcSmemBar = kTcSmemKV + kTcKVSlots * kTcTileBytes;  // mbarriers
constexpr uint32_t kTcSmemBytes = kTcSmemBar + 256 + 1024;  // 230,656 B: barriers + alignment slack
constexpr uint64_t kTcWaitNs = 1000000000ull;  // give up a wait after 1 s of device time
constexpr uint32_t kTcSpinLimit = 1u << 25;     // backstop on the polls of one wait
constexpr uint32_t kTcDrainLimit = 1u << 22;    // polls for in-flight work after an abort

struct PrefillTcArgs {
  const float *q_norm_w;  // [128]
  const float *rope_tab;  // local: angle-major float2 (cos, sin) [64][rows]; null for global
  float eps;
  const uint16_t *gate;   // [B][T][48*128]
  const float *gate_bias; // [48]
  uint16_t *out;          // [B][T][48*128], written directly or through the map tm_o
  int32_t *status;
  int B, T, kind, window, n_qblocks, n_units;
  float scale_log2, ssmax_base, ssmax_exp;
  int fault_stall;        // tests only: the MMA issuer first waits on a barrier never arrived at
  // Chunked prefill (new tokens after pos0[b] cached ones); pos0 == null for a plain prefill.
  const int64_t *pos0;    // [B] position of each sequence's first new token
  int64_t slots;          // global: cache slots per sequence (the K/V maps cover the cache)
  int ext_prefix;         // local: rows of earlier keys in front of the new ones (window - 1)
  int kv_slot_major;      // K/V maps take coordinates (d, slot, head, b), not (d, head, t, b)
  int rope_rows;          // rows per sequence in rope_tab (0: one table of T rows for all)
  // Output factor: v_scale over an FP8 cache, whose K/V maps read the unscaled values of the
  // codes (k_scale is folded into scale_log2 by the host); 1 for a bf16 cache
  float v_scale;
};

namespace tcd {
// barrier slots (8 bytes each) after kTcSmemBar
constexpr int kQFull = 0, kQEmpty = 2, kQReady = 4, kKVFull = 6, kKVEmpty = 9, kSFull = 12,
              kPFull = 14, kOFull = 16, kOEmpty = 18, kDrain = 20, kStall = 21, kYReady = 22,
              kNumBars = 24;
constexpr uint32_t kTmemHolder = kNumBars * 8;      // u32: tensor-memory base address
constexpr uint32_t kAbortFlag = kTmemHolder + 4;    // u32: set when a wait ran out
}  // namespace tcd
static_assert(tcd::kAbortFlag + 4 <= 256, "barrier area of the prefill kernel overflows");

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase; false when it ran out or another role aborted.  The
// clock is read every 1024 polls only, so a wait that succeeds soon never reads it.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile uint32_t *abort,
                                        int32_t *status) {
  uint64_t t0 = 0;
  for (uint32_t i = 0; i < kTcSpinLimit; ++i) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if ((i & 1023u) == 1023u) {
      const uint64_t t = globaltimer_ns();
      if (t0 == 0) t0 = t;
      else if (t - t0 > kTcWaitNs) break;
    }
  }
  set_status(status, BEAM_ERR_DEVICE_TIMEOUT);
  *abort = 1u;
  return false;
}

// Wait for the `count`-th completion (count >= 1) of a barrier that only its own producer
// arms: in-flight copies must land before the CTA returns, whether or not it aborted.
__device__ __forceinline__ void tc_drain(uint32_t bar, uint32_t count, int32_t *status) {
  if (count == 0) return;
  for (uint32_t i = 0; i < kTcDrainLimit; ++i)
    if (tc::mbar_try_wait(bar, (count - 1) & 1u)) return;
  set_status(status, BEAM_ERR_DEVICE_TIMEOUT);
}

// Work unit u -> (sequence, q block, head pair): sequence-major, so the CTAs share one
// sequence's K/V (8 heads x T x 512 B, 32 MiB at T = 8192) while it stays in L2, and within
// a sequence the units with more key blocks come first.
// Keys are addressed by their coordinate in the K/V maps: query row r of the unit has its
// own key at kq + r and sees the coordinates max(kq + r - window + 1, kmin) .. kq + r
// (local) or 0 .. kq + r (global).  A plain prefill has kq = q0, kmin = 0.  A chunk of a
// global layer reads the cache itself (coordinate = slot = position, kq = pos0 + q0); a
// chunk of a local layer reads keys laid out as window - 1 earlier rows, then the new ones
// (kq = window - 1 + q0; rows below kmin precede the sequence's first token).  t0 is the
// position of row 0 (for a(p)); `bad` marks a sequence whose pos0 is out of range: its
// rows are computed on clamped coordinates and not written.
struct TcUnit {
  int qb, pair, b, q0, kb_lo, n_blk, kq, kmin, t0;
  bool bad;
};
__device__ __forceinline__ TcUnit tc_unit(const PrefillTcArgs &a, int u) {
  TcUnit w;
  const int per_b = (kHq / 2) * a.n_qblocks;
  w.b = u / per_b;
  const int rem = u - w.b * per_b;
  w.qb = a.n_qblocks - 1 - rem / (kHq / 2);
  w.pair = rem % (kHq / 2);
  w.q0 = w.qb * kTcBM;
  w.kq = w.q0;
  w.kmin = 0;
  w.t0 = w.q0;
  w.bad = false;
  const bool local = a.kind == BEAM_LOCAL;
  if (a.pos0) {
    int64_t p0 = a.pos0[w.b];
    if (p0 < 0) {
      w.bad = true;
      p0 = 0;
    }
    if (local) {
      w.kq = a.ext_prefix + w.q0;
      w.kmin = a.ext_prefix - (int)min(p0, (int64_t)a.ext_prefix);
    } else {
      if (p0 > a.slots - a.T) {
        w.bad = true;
        p0 = a.slots - a.T;   // >= 0: the host checks T <= slots
      }
      w.kq = (int)p0 + w.q0;
      w.t0 = w.kq;
    }
  }
  w.kb_lo = local ? max(w.kmin, w.kq - a.window + 1) / kTcBN : 0;
  // the last visible key of the unit is the own key of its last row below T
  w.n_blk = (w.kq + min(kTcBM - 1, a.T - 1 - w.q0)) / kTcBN - w.kb_lo + 1;
  return w;
}

// Y = O * inv * (1 + tanh((G + b) / 2)) (inv = 1 / (2 l), hb = b / 2) for the 8 coordinates
// of one 16-byte word: o holds the 32 fp32 O values of a chunk, q picks 8 of them.
__device__ __forceinline__ uint4 gated_y8(const uint4 g4, const uint32_t (&o)[32], int q, float inv,
                                          float hb) {
  const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
  uint32_t yw[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float s0 = 1.0f + tanh_approx(fmaf(0.5f, bf16_lo(gw[e]), hb));
    const float s1 = 1.0f + tanh_approx(fmaf(0.5f, bf16_hi(gw[e]), hb));
    yw[e] = pack_bf16(__uint_as_float(o[q * 8 + 2 * e]) * inv * s0,
                      __uint_as_float(o[q * 8 + 2 * e + 1]) * inv * s1);
  }
  return make_uint4(yw[0], yw[1], yw[2], yw[3]);
}

// kStage: the output goes through shared memory and the store warp (global layer).
// kWide: the gate, output and RoPE-table rows are 32-byte aligned, so each thread moves
// its row with 32-byte accesses (half the requests of 16-byte ones).  The forms are separate
// instantiations so that each keeps its own register allocation.
template <bool kStage, bool kWide>

__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const PrefillTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // SW128 tiles need 1024-byte alignment
  uint8_t *sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + kTcSmemBar;
  volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sgen + kTcSmemBar + tcd::kAbortFlag);
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool local = a.kind == BEAM_LOCAL;

  if (threadIdx.x == 0) {
    for (int i = 0; i < tcd::kNumBars; ++i) {
      uint32_t count = 1;
      if (i == tcd::kPFull || i == tcd::kPFull + 1 || i == tcd::kOEmpty || i == tcd::kOEmpty + 1 ||
          i == tcd::kQReady || i == tcd::kQReady + 1 || i == tcd::kYReady || i == tcd::kYReady + 1)
        count = 128;
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

  // Register split (per warpgroup) of the 512 x 128 registers the CTA is launched with:
  // warps 0-3 (two producers, MMA issuer, idle) keep 56, the Q-preparation warpgroup
  // (warps 12-15) 104, the two softmax warpgroups 176: 128*(56 + 104) + 256*176 = 65536,
  // and on every SM sub-partition 56 + 104 + 2*176 = 512 registers per lane.
  // K tiles of the CTA's block sequence go to a two-slot ring (block i in slot i % 2), V
  // tiles to one slot; K runs a block ahead of V, so K(i+1) loads as soon as both Q K(i-1)^T
  // are done, and V(i) once both P V(i-1) are.  Barrier slots kKVFull/kKVEmpty + 0, 1 are
  // the K ring, + 2 the V slot.
  if (warp == 0) {
    // ------------------------------------------------------------ K/V producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
    if (lane == 0) {
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      struct Cursor {  // walks (unit, block) in the order the MMA issuer consumes them
        int u, j, b, g, kb_lo, n_blk;
        bool valid;
      };
      auto set_unit = [&](Cursor &c) {
        c.valid = c.u < a.n_units;
        if (c.valid) {
          const TcUnit w = tc_unit(a, c.u);
          c.b = w.b;
          c.g = (2 * w.pair) / kGroup;
          c.kb_lo = w.kb_lo;
          c.n_blk = w.n_blk;
        }
      };
      auto start = [&](Cursor &c) {
        c.u = blockIdx.x;
        c.j = 0;
        set_unit(c);
      };
      auto advance = [&](Cursor &c) {
        if (++c.j == c.n_blk) {
          c.j = 0;
          c.u += gridDim.x;
          set_unit(c);
        }
      };
      auto load = [&](const Cursor &c, bool is_v, uint32_t slot) {
        const int g = c.g, key0 = (c.kb_lo + c.j) * kTcBN;
        tc::mbar_expect_tx(bar(tcd::kKVFull + slot), kTcTileBytes);
        const uint32_t dst = sbase + kTcSmemKV + slot * kTcTileBytes;
        const CUtensorMap *map = is_v ? &tm_v : &tm_k;
        for (int hf = 0; hf < 2; ++hf) {
          if (a.kv_slot_major)
            tc::tma_load_4d(dst + hf * kTcHalfBytes, map, bar(tcd::kKVFull + slot), hf * 64, key0, g,
                            c.b);
          else
            tc::tma_load_4d(dst + hf * kTcHalfBytes, map, bar(tcd::kKVFull + slot), hf * 64, g, key0,
                            c.b);
        }
      };
      Cursor kc, vc;
      start(kc);
      start(vc);
      uint32_t ik = 0, iv = 0;  // K and V tiles issued so far
      bool ok = true;
      if (kc.valid) {
        load(kc, false, 0);
        ++ik;
        advance(kc);
      }
      while (ok && vc.valid) {
        if (kc.valid) {
          const uint32_t slot = ik & 1u;
          if (ik >= 2 &&
              !(ok = tc_wait(bar(tcd::kKVEmpty + slot), ((ik >> 1) - 1) & 1u, abort, a.status)))
            break;
          load(kc, false, slot);
          ++ik;
          advance(kc);
        }
        if (iv >= 1 && !(ok = tc_wait(bar(tcd::kKVEmpty + 2), (iv - 1) & 1u, abort, a.status)))
          break;
        load(vc, true, 2);
        ++iv;
        advance(vc);
      }
      // K slot 0 took loads 0, 2, 4, ..., slot 1 loads 1, 3, ...; V slot 2 all iv
      tc_drain(bar(tcd::kKVFull + 0), (ik + 1) >> 1, a.status);
      tc_drain(bar(tcd::kKVFull + 1), ik >> 1, a.status);
      tc_drain(bar(tcd::kKVFull + 2), iv, a.status);
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
      // O_t += P_t V with V in ring slot `slot`; `first` overwrites O_t.
      auto issue_pv = [&](int t, uint32_t slot, bool first) {
        const uint32_t vt = sbase + kTcSmemKV + slot * kTcTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::umma_ts(tmem + 256 + 128 * t, tmem + 128 * t + kk * 8, v_desc(vt, kk), idesc_pv,
                      (!first || kk > 0) ? 1u : 0u);
      };
      uint32_t it = 0;  // blocks of the CTA started so far
      bool ok = !a.fault_stall || tc_wait(bar(tcd::kStall), 0u, abort, a.status);
      for (int u = blockIdx.x, n = 0; ok && u < a.n_units; u += gridDim.x, ++n) {
        const TcUnit w = tc_unit(a, u);
        const int qset = n & 1;
        if (!(ok = tc_wait(bar(tcd::kQReady + qset), (n >> 1) & 1, abort, a.status))) break;
        // step j: O_t += P_t(j-1) V(j-1) (j > 0), then S_t(j) = Q_t K(j)^T (j < n_blk)
        for (int j = 0; ok && j <= w.n_blk; ++j) {
          const bool has_s = j < w.n_blk;
          const uint32_t ks_slot = it & 1u;
          if (has_s &&
              !(ok = tc_wait(bar(tcd::kKVFull + ks_slot), (it >> 1) & 1u, abort, a.status)))
            break;
          tc::tc_fence_after();
          const uint32_t kt = sbase + kTcSmemKV + ks_slot * kTcTileBytes;
          for (int t = 0; t < 2 && ok; ++t) {
            if (j > 0) {
              if (!(ok = tc_wait(bar(tcd::kPFull + t), (it - 1) & 1u, abort, a.status))) break;
              if (t == 0 &&
                  !(ok = tc_wait(bar(tcd::kKVFull + 2), (it - 1) & 1u, abort, a.status)))
                break;
              // the first P V of a unit overwrites O_t: the previous epilogue must be done
              if (j == 1 && n > 0 &&
                  !(ok = tc_wait(bar(tcd::kOEmpty + t), (n - 1) & 1, abort, a.status)))
                break;
              tc::tc_fence_after();
              issue_pv(t, 2, j == 1);
              if (t == 1) tc::umma_commit(bar(tcd::kKVEmpty + 2));
              if (!has_s) tc::umma_commit(bar(tcd::kOFull + t));
            }
            if (has_s) {
              const uint32_t qt = sbase + kTcSmemQ + (qset * 2 + t) * kTcTileBytes;
#pragma unroll
              for (int ks = 0; ks < 8; ++ks)
                tc::umma_ss(tmem + 128 * t, qk_desc(qt, ks), qk_desc(kt, ks), idesc_qk,
                            ks > 0 ? 1u : 0u);
              tc::umma_commit(bar(tcd::kSFull + t));
              if (t == 1) {
                tc::umma_commit(bar(tcd::kKVEmpty + ks_slot));
                if (j == w.n_blk - 1 && !kStage) tc::umma_commit(bar(tcd::kQEmpty + qset));
              }
            }
          }
          if (has_s) ++it;
        }
      }
      // every MMA issued so far must be done before the tensor memory is freed
      tc::umma_commit(bar(tcd::kDrain));
      tc_drain(bar(tcd::kDrain), 1, a.status);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ Q producer
    // Raw Q tiles of unit n into set n & 1, as soon as unit n - 2 has released the set (its
    // last Q K^T is done or, when its Y tiles were staged there, their copies have read them).
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      bool ok = true;
      int nq = 0;   // units whose Q tiles were issued (set n & 1 took units n, n + 2, ...)
      for (int u = blockIdx.x, n = 0; ok && u < a.n_units; u += gridDim.x, ++n) {
        const TcUnit w = tc_unit(a, u);
        const int qset = n & 1;
        if (n >= 2 &&
            !(ok = tc_wait(bar(tcd::kQEmpty + qset), ((n >> 1) - 1) & 1, abort, a.status)))
          break;
        tc::mbar_expect_tx(bar(tcd::kQFull + qset), 2 * kTcTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int hf = 0; hf < 2; ++hf)
            tc::tma_load_4d(sbase + kTcSmemQ + (qset * 2 + t) * kTcTileBytes + hf * kTcHalfBytes,
                            &tm_q, bar(tcd::kQFull + qset), hf * 64, 2 * w.pair + t, w.q0, w.b);
        nq = n + 1;
      }
      tc_drain(bar(tcd::kQFull + 0), (nq + 1) >> 1, a.status);
      tc_drain(bar(tcd::kQFull + 1), nq >> 1, a.status);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------ output store
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
    if (lane == 0) {
      tc::prefetch_tmap(&tm_o);
      bool ok = true;
      uint32_t ns = 0;   // staged units so far (phases of the kYReady barriers)
      for (int u = blockIdx.x, n = 0; ok && u < a.n_units; u += gridDim.x, ++n) {
        if (!kStage) break;
        const TcUnit w = tc_unit(a, u);
        const int qset = n & 1;
        for (int t = 0; t < 2; ++t) {
          if (!(ok = tc_wait(bar(tcd::kYReady + t), ns & 1u, abort, a.status))) break;
          if (!w.bad)   // a sequence whose pos0 is out of range is not written
            for (int hf = 0; hf < 2; ++hf)
              tc::tma_store_4d(&tm_o, sbase + kTcSmemQ + (qset * 2 + t) * kTcTileBytes + hf * kTcHalfBytes,
                               hf * 64, 2 * w.pair + t, w.q0, w.b);
        }
        tc::bulk_commit_group();
        tc::bulk_wait_read_all();   // the set may be overwritten once the copies have read it
        if (ok) tc::mbar_arrive(bar(tcd::kQEmpty + qset));
        ++ns;
      }
      tc::bulk_wait_all();   // the output rows are written before the CTA ends
    }
    __syncwarp();
  } else if (warp >= 12) {
    // ------------------------------------------------------------ Q preparation
    // RMSNorm of each raw Q row in shared memory (in place), then RoPE for a local layer;
    // thread r owns row r of both tiles (same position, so the same angles).  The RoPE table
    // is angle-major (entry (i, row) = (cos, sin) at i * stride + row), so the 32 rows of a
    // warp read one contiguous run per angle; chunk 0 is fetched before the Q tiles land,
    // chunk c + 1 while chunk c is worked.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 104;\n" ::: "memory");
    const int r = threadIdx.x - 384;
    const float4 *w4 = reinterpret_cast<const float4 *>(a.q_norm_w);
    const float2 *tab2 = reinterpret_cast<const float2 *>(a.rope_tab);
    const size_t rope_stride = a.rope_rows ? (size_t)a.B * a.rope_rows : (size_t)a.T;
    bool ok = true;
    for (int u = blockIdx.x, n = 0; ok && u < a.n_units; u += gridDim.x, ++n) {
      const TcUnit w = tc_unit(a, u);
      const int tok = w.q0 + r;
      // a global layer (kStage) has no RoPE: its instantiation carries none of this code
      const bool rope = !kStage && local;
      const float2 *tab =
          rope ? tab2 + (size_t)(a.rope_rows ? w.b * a.rope_rows : 0) + min(tok, a.T - 1) : nullptr;
      float2 tb[8];   // (cos, sin) of the 8 angles of the chunk in hand
      const float2 *tab_next = tab;   // angle 8 c of the next chunk to fetch
      auto tab_load = [&]() {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          tb[e] = __ldg(tab_next);
          tab_next += rope_stride;
        }
      };
      if (rope) tab_load();
      const int qset = n & 1;
      if (!(ok = tc_wait(bar(tcd::kQFull + qset), (n >> 1) & 1, abort, a.status))) break;
      auto chunk = [&](int t, int hf, int c) -> uint4 * {   // 8 bf16 at d = 64 hf + 8 c
        return reinterpret_cast<uint4 *>(sgen + kTcSmemQ + (qset * 2 + t) * kTcTileBytes +
                                         r * 128 + hf * kTcHalfBytes + ((c ^ (r & 7)) << 4));
      };
      float inv[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        float ss = 0.f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = *chunk(t, hf, c);
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = bf16_lo(vw[e]), x1 = bf16_hi(vw[e]);
              ss = fmaf(x0, x0, fmaf(x1, x1, ss));
            }
          }
        inv[t] = rsqrtf(ss * (1.0f / kD) + a.eps);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 wl0 = __ldg(w4 + 2 * c), wl1 = __ldg(w4 + 2 * c + 1);
        const float4 wh0 = __ldg(w4 + 16 + 2 * c), wh1 = __ldg(w4 + 16 + 2 * c + 1);
        const float wl[8] = {wl0.x, wl0.y, wl0.z, wl0.w, wl1.x, wl1.y, wl1.z, wl1.w};
        const float wh[8] = {wh0.x, wh0.y, wh0.z, wh0.w, wh1.x, wh1.y, wh1.z, wh1.w};
        float cv[8], sv[8];
        if (rope) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            cv[e] = tb[e].x;
            sv[e] = tb[e].y;
          }
          if (c < 7) tab_load();   // the next chunk's angles, while this chunk is worked
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint4 lo = *chunk(t, 0, c), hi = *chunk(t, 1, c);
          const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w}, hw[4] = {hi.x, hi.y, hi.z, hi.w};
          float xl[8], xh[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            xl[2 * e] = bf16_lo(lw[e]) * inv[t] * wl[2 * e];
            xl[2 * e + 1] = bf16_hi(lw[e]) * inv[t] * wl[2 * e + 1];
            xh[2 * e] = bf16_lo(hw[e]) * inv[t] * wh[2 * e];
            xh[2 * e + 1] = bf16_hi(hw[e]) * inv[t] * wh[2 * e + 1];
          }
          if (rope) {  // rotate-half: coordinate i < 64 pairs with i + 64
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float a0 = xl[e], b0 = xh[e];
              xl[e] = a0 * cv[e] - b0 * sv[e];
              xh[e] = b0 * cv[e] + a0 * sv[e];
            }
          }
          *chunk(t, 0, c) = make_uint4(pack_bf16(xl[0], xl[1]), pack_bf16(xl[2], xl[3]),
                                       pack_bf16(xl[4], xl[5]), pack_bf16(xl[6], xl[7]));
          *chunk(t, 1, c) = make_uint4(pack_bf16(xh[0], xh[1]), pack_bf16(xh[2], xh[3]),
                                       pack_bf16(xh[4], xh[5]), pack_bf16(xh[6], xh[7]));
        }
      }
      // generic-proxy writes -> visible to the tensor cores' async proxy, then publish
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      tc::mbar_arrive(bar(tcd::kQReady + qset));
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 176;\n" ::: "memory");
    const int t = (warp - 4) >> 2;      // tile: 0 for warps 4-7, 1 for warps 8-11
    const int wq = warp & 3;            // tensor-memory lane quarter this warp may access
    const int r = wq * 32 + lane;       // query row within the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t t_s = tmem + lane_off + 128 * t;
    const uint32_t t_o = tmem + lane_off + 256 + 128 * t;
    uint32_t it = 0;  // blocks processed so far (barrier phases)
    bool ok = true;
    for (int u = blockIdx.x, n = 0; ok && u < a.n_units; u += gridDim.x, ++n) {
      const TcUnit w = tc_unit(a, u);
      // the row's visible key coordinates are lo_base .. hi_base; rows of a sequence whose
      // pos0 is out of range count as past T (computed, not written)
      const int hi_base = w.kq + r;
      const int lo_base = local ? max(hi_base - a.window + 1, w.kmin) : -(1 << 30);
      const int tok = w.bad ? a.T : w.q0 + r;
      const int h = 2 * w.pair + t;
      float factor = a.scale_log2;
      if (!local) factor *= ssmax_factor((int64_t)w.t0 + r + 1, a.ssmax_base, a.ssmax_exp);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < w.n_blk; ++j, ++it) {
        if (!(ok = tc_wait(bar(tcd::kSFull + t), it & 1u, abort, a.status))) break;
        tc::tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_ld32(t_s + 32 * c, sr[c]);
        tc::tmem_ld_wait();
        const int k0 = (w.kb_lo + j) * kTcBN;
        // masked only where the block holds a key outside this row's range.  Key k0 + i is
        // visible to row r iff lo <= i <= hi; the window start and the causal edge move by
        // one key per row, so in most 32-key chunks a warp's 32 rows agree: a chunk whose
        // keys are all visible to every row of the warp is passed over.
        if (__any_sync(0xffffffffu, k0 + kTcBN - 1 > hi_base || k0 < lo_base)) {
          const int hi = hi_base - k0;
          const int lo = lo_base - k0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const bool all_in = __all_sync(0xffffffffu, lo <= 32 * c && hi >= 32 * c + 31);
            const bool all_out = __all_sync(0xffffffffu, hi < 32 * c || lo > 32 * c + 31);
            if (!all_in) {   // (an all-invisible chunk takes an empty range)
              const int lo_c = all_out ? 32 : lo - 32 * c, hi_c = hi - 32 * c;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                sr[c][i] = (i >= lo_c && i <= hi_c) ? sr[c][i] : 0xFF800000u;  // -inf
            }
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
            tc::f2_unpack(tc::f2_fma(tc::f2_pack(__uint_as_float(sr[c][i]),
                                                 __uint_as_float(sr[c][i + 1])),
                                     f2, nm2),
                          y0, y1);
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
      if (!ok) break;
      // ---- epilogue: Y = O / l * sigmoid(G + b_h), sigmoid(x) = (1 + tanh(x/2)) / 2, as
      // bf16 into row r of the unit's Q tile t (128-byte swizzled, as the copies read it)
      // or, for a unit that is not staged, straight to its output row.
      // The gate row is fetched before the wait for the last P V, to hide its latency.
      const bool valid = tok < a.T;
      const size_t row = ((size_t)w.b * a.T + (valid ? tok : 0)) * (kHq * kD) + (size_t)h * kD;
      uint4 gr[16];
      {
        const uint4 *gp = reinterpret_cast<const uint4 *>(a.gate + row);
        if constexpr (kWide) {
#pragma unroll
          for (int q = 0; q < 16; q += 2) {
            if (valid) tc::ld_nc_v8(gp + q, gr[q], gr[q + 1]);
            else gr[q] = gr[q + 1] = make_uint4(0u, 0u, 0u, 0u);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) gr[q] = valid ? __ldg(gp + q) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (!(ok = tc_wait(bar(tcd::kOFull + t), n & 1, abort, a.status))) break;
      tc::tc_fence_after();
      const float inv = (0.5f / l) * a.v_scale;
      const float hb = 0.5f * a.gate_bias[h];
      if constexpr (kStage) {
        // row r of the tile, with the row's swizzle (r % 8) in the chunk bits: the row starts
        // on a 128-byte boundary, so chunk k sits at yrow ^ (k << 4)
        const uint32_t yrow =
            (sbase + kTcSmemQ + ((n & 1) * 2 + t) * kTcTileBytes + r * 128) | ((r & 7) << 4);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(t_o + 32 * c, o);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 4; ++q) {   // d = 32 c + 8 q: half c / 2, chunk 4 (c % 2) + q
            const uint4 y = gated_y8(gr[4 * c + q], o, q, inv, hb);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(
                             (yrow ^ (((c & 1) * 4 + q) << 4)) + (c >> 1) * kTcHalfBytes),
                         "r"(y.x), "r"(y.y), "r"(y.z), "r"(y.w) : "memory");
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(t_o + 32 * c, o);
          tc::tmem_ld_wait();
          if (valid) {
            uint4 *op = reinterpret_cast<uint4 *>(a.out + row + c * 32);
#pragma unroll
            for (int q = 0; q < 4; q += 2) {
              const uint4 y0 = gated_y8(gr[4 * c + q], o, q, inv, hb);
              const uint4 y1 = gated_y8(gr[4 * c + q + 1], o, q + 1, inv, hb);
              if constexpr (kWide) {
                tc::st_v8(op + q, y0, y1);
              } else {
                op[q] = y0;
                op[q + 1] = y1;
              }
            }
          }
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(bar(tcd::kOEmpty + t));
      if constexpr (kStage) {
        // generic-proxy writes -> visible to the copies' async proxy, then publish the tile
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        tc::mbar_arrive(bar(tcd::kYReady + t));
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
