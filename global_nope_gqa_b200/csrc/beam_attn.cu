// beam_attn.cu -- the C ABI of the attention core (declared in beam_attn.h):
// host-side validation, workspace carving and kernel launches.
//
// Every call validates its arguments on the host and returns before any launch
// when they are wrong; kernels are launched on the caller's stream and the call
// returns without synchronising.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "beam_attn.h"
#include "common.cuh"
#include "decode.cuh"
#include "decode8.cuh"
#include "decode_multi.cuh"
#include "decode_tc.cuh"
#include "prefill_tc.cuh"
#include "prologue.cuh"

using namespace beam;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
};
DeviceInfo g_dev[kMaxDevices];

// With BEAM_VERBOSE set in the environment, CUDA failures are also printed to stderr.
bool verbose() {
  static const bool v = std::getenv("BEAM_VERBOSE") != nullptr;
  return v;
}

int cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return BEAM_OK;
  if (verbose()) std::fprintf(stderr, "beam_attn: %s: %s\n", what, cudaGetErrorString(e));
  return BEAM_ERR_CUDA;
}


// A warp-specialised kernel redistributes its registers between roles (setmaxnreg); the
// roles' shares must fit in what the CTA is launched with, or the increase never completes.
// Checked against the compiled per-thread count once per device, before any launch.
int check_register_pool(const void *kernel, int threads, int pool) {
  cudaFuncAttributes fa;
  int st = cuda_status(cudaFuncGetAttributes(&fa, kernel), "kernel attributes");
  if (st) return st;
  if ((int64_t)fa.numRegs * threads < pool) {
    if (verbose())
      std::fprintf(stderr, "beam_attn: %d registers x %d threads < register split %d\n", fa.numRegs,
                   threads, pool);
    return BEAM_ERR_UNSUPPORTED;
  }
  return BEAM_OK;
}

// Per-device attributes: SM count, the dynamic shared-memory opt-ins and the register
// pools of the warp-specialised kernels.
int device_info(DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BEAM_ERR_CUDA;
  DeviceInfo &d = g_dev[dev];
  if (!d.ready) {
    int st;
    if ((st = cuda_status(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev),
                          "SM count")))
      return st;
    if ((st = cuda_status(cudaFuncSetAttribute(decode_attn_kernel<false>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem),
                          "decode shared-memory opt-in")))
      return st;
    if ((st = cuda_status(cudaFuncSetAttribute(decode_attn_kernel<true>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem),
                          "decode shared-memory opt-in")))
      return st;
    for (auto kernel : {decode_tc_kernel<false>, decode_tc_kernel<true>})
      if ((st = cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kDtSmemBytes),
                            "multi-token decode shared-memory opt-in")))
        return st;
    if ((st = cuda_status(cudaFuncSetAttribute(decode8_attn_kernel<false>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kDec8Smem),
                          "FP8 decode shared-memory opt-in")))
      return st;
    if ((st = cuda_status(cudaFuncSetAttribute(decode8_attn_kernel<true>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kDec8Smem),
                          "FP8 decode shared-memory opt-in")))
      return st;
    for (auto kernel : {prefill_tc_kernel<true, true>, prefill_tc_kernel<true, false>,
                        prefill_tc_kernel<false, true>, prefill_tc_kernel<false, false>})
      if ((st = cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kTcSmemBytes),
                            "prefill shared-memory opt-in")) ||
          (st = check_register_pool(reinterpret_cast<const void *>(kernel), kTcThreads, kTcRegPool)))
        return st;
    for (auto kernel : {decode_tc_kernel<false>, decode_tc_kernel<true>})
      if ((st = check_register_pool(reinterpret_cast<const void *>(kernel), kDtThreads, kDtRegPool)))
        return st;
    d.ready = true;
  }
  *out = &d;
  return BEAM_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_params(int kind, const beam_attn_params *p) {
  if (!p) return BEAM_ERR_INVALID_ARG;
  if (kind != BEAM_LOCAL && kind != BEAM_GLOBAL) return BEAM_ERR_INVALID_ARG;
  if (p->n_q_heads != kHq || p->n_kv_heads != kHkv || p->head_dim != kD)
    return BEAM_ERR_UNSUPPORTED;
  if (p->window < 1) return BEAM_ERR_INVALID_ARG;
  if (!(p->rms_eps >= 0.f) || !(p->ssmax_base > 0.f) || !(p->rope_theta > 0.f) ||
      !std::isfinite(p->softmax_scale) || !std::isfinite(p->ssmax_exp))
    return BEAM_ERR_INVALID_ARG;
  return BEAM_OK;
}

int check_layout(int kind, const beam_attn_params *p, const beam_kv_layout_t *L) {
  if (!L) return BEAM_ERR_INVALID_ARG;
  if (L->slots_per_seq < 1 || L->stride_slot != kD) return BEAM_ERR_INVALID_ARG;
  if (L->stride_head < L->slots_per_seq * kD || L->stride_seq < kHkv * L->stride_head)
    return BEAM_ERR_INVALID_ARG;
  if ((L->stride_head % 8) || (L->stride_seq % 8)) return BEAM_ERR_ALIGNMENT;
  if (kind == BEAM_LOCAL && L->slots_per_seq != p->window) return BEAM_ERR_INVALID_ARG;
  return BEAM_OK;
}

// An FP8 cache holds one-byte codes: its rows must start on 16 bytes as well.
int check_layout_fp8(int kind, const beam_attn_params *p, const beam_kv_layout_t *L) {
  int st = check_layout(kind, p, L);
  if (st) return st;
  if ((L->stride_head % 16) || (L->stride_seq % 16)) return BEAM_ERR_ALIGNMENT;
  return BEAM_OK;
}

bool valid_scale(float s) { return std::isfinite(s) && s > 0.f && std::isfinite(1.0f / s); }

void fill_inv_freq(double (&f)[64], double theta) {
  for (int i = 0; i < 64; ++i) f[i] = std::pow(theta, -2.0 * i / (double)kD);
}

int launch_status() { return cuda_status(cudaGetLastError(), "kernel launch"); }

// A launch with programmatic stream serialization: the kernel may start while the one before
// it in the stream finishes; it calls pdl_wait() before it touches that kernel's results.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
               Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kernel, args...), "kernel launch");
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

int encode_fn() {
  if (g_encode_tiled) return BEAM_OK;
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return BEAM_ERR_CUDA;
  g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return BEAM_OK;
}

// 4-D bf16 map over a token-major activation [B][T][heads][128]: coordinates
// (d, head, t, b), 128-byte swizzled boxes of 64 d x 1 head x 128 tokens.  Tokens past
// T read as zeros.
int make_head_map(CUtensorMap *map, const void *base, int heads, int T, int B) {
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)heads, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)heads * kD * 2,
                                 (cuuint64_t)T * heads * kD * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)kTcBM, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BEAM_OK : BEAM_ERR_CUDA;
}

// 4-D bf16 map over a head-major cache [B][8][slots][128] with the layout's strides:
// coordinates (d, slot, head, b), the same boxes; slots past the capacity read as zeros.
int make_cache_map(CUtensorMap *map, const void *base, const beam_kv_layout_t *L, int B) {
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)L->slots_per_seq, (cuuint64_t)kHkv,
                              (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)L->stride_slot * 2, (cuuint64_t)L->stride_head * 2,
                                 (cuuint64_t)L->stride_seq * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)kTcBN, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BEAM_OK : BEAM_ERR_CUDA;
}

// 4-D map over an FP8 cache [B][8][slots][128] of one-byte codes: coordinates (d, slot,
// head, b), 128-byte swizzled boxes of 128 codes x 128 slots; slots past the capacity read
// as zero codes.
int make_cache_map_u8(CUtensorMap *map, const void *base, const beam_kv_layout_t *L, int B) {
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)L->slots_per_seq, (cuuint64_t)kHkv,
                              (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)L->stride_slot, (cuuint64_t)L->stride_head,
                                 (cuuint64_t)L->stride_seq};
  const cuuint32_t box[4] = {(cuuint32_t)kD, (cuuint32_t)kTcBN, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BEAM_OK : BEAM_ERR_CUDA;
}

// The persistent tcgen05 attention kernel over B sequences of T query rows.  The caller
// fills the pointers and the chunk fields of `fa`; the shape and scale fields are set here.
// k_scale: the keys' factor over an FP8 cache (1 for bf16), folded into the score scale.
int launch_prefill_attention(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                             const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                             const CUtensorMap &tm_v, PrefillTcArgs fa, const DeviceInfo *dev,
                             cudaStream_t s, float k_scale = 1.0f) {
  fa.eps = p->rms_eps;
  fa.B = B;
  fa.T = T;
  fa.kind = kind;
  fa.window = p->window;
  fa.n_qblocks = (T + kTcBM - 1) / kTcBM;
  fa.scale_log2 = p->softmax_scale * kLog2e * k_scale;
  fa.ssmax_base = p->ssmax_base;
  fa.ssmax_exp = p->ssmax_exp;
  // Fault injection for tests of the device-timeout path: with BEAM_FAULT_INJECT set to
  // prefill_wait_stall, the attention kernel's MMA issuer waits on a barrier that nothing
  // arrives at, so the wait runs out and the call reports BEAM_ERR_DEVICE_TIMEOUT.
  {
    const char *f = std::getenv("BEAM_FAULT_INJECT");
    fa.fault_stall = f != nullptr && std::strcmp(f, "prefill_wait_stall") == 0;
  }
  const int64_t n_units = (int64_t)fa.n_qblocks * (kHq / 2) * B;
  if (n_units > INT32_MAX) return BEAM_ERR_UNSUPPORTED;
  fa.n_units = (int)n_units;
  CUtensorMap tm_o;   // the output rows, stored tile by tile (rows past T are clipped)
  if (int st = make_head_map(&tm_o, fa.out, kHq, T, B)) return st;
  // persistent: one CTA per SM (the kernel's shared memory admits one per SM)
  const int grid = (int)std::min<int64_t>(n_units, dev->sm_count);
  // 32-byte row accesses need the gate and output rows 32-byte aligned (the RoPE table is
  // read in 8-byte pieces)
  const bool wide = ((reinterpret_cast<uintptr_t>(fa.gate) | reinterpret_cast<uintptr_t>(fa.out)) &
                     31u) == 0;
  auto kernel = kind == BEAM_GLOBAL ? (wide ? prefill_tc_kernel<true, true> : prefill_tc_kernel<true, false>)
                                    : (wide ? prefill_tc_kernel<false, true> : prefill_tc_kernel<false, false>);
  kernel<<<grid, kTcThreads, kTcSmemBytes, s>>>(tm_q, tm_k, tm_v, tm_o, fa);
  return launch_status();
}

// Decode split size: cache slots per CTA.  A local ring is cut into at most four
// splits (one thread-block cluster); a global cache is cut so that the grid holds about
// three waves of resident CTAs at its largest context (2 per SM for a BF16 cache, 3 for
// FP8), in runs of at least 512 slots.  Longer runs measured faster than more waves of
// shorter ones: each CTA pays a fixed start (queries, first tiles) and end (merge).
int decode_split(int kind, const beam_attn_params *p, int32_t B, int64_t slots, int sm_count,
                 bool fp8) {
  if (kind == BEAM_LOCAL) {  // the ring: one split, or up to 4 (a cluster) for small batches
    const size_t ring = round_up((size_t)p->window, kDecTile);
    if ((int64_t)B * kHkv >= 2 * sm_count) return (int)ring;
    return (int)std::max<size_t>(kDecTile, round_up(((size_t)p->window + 3) / 4, kDecTile));
  }
  const int64_t target_ctas = (int64_t)sm_count * (fp8 ? 3 : 2) * 3;
  int64_t split = 512;
  while (split < 16384 && (int64_t)B * kHkv * ((slots + split - 1) / split) > target_ctas)
    split *= 2;
  while ((slots + split - 1) / split > kCombineMaxSplits) split *= 2;  // the combine's limit
  return (int)split;
}

// What beam_decode_workspace_bytes reports for a local layer, which needs no workspace:
// a small nonzero size, because 0 reports invalid arguments.
constexpr size_t kDecodeNoWorkspace = 16;

struct DecodeWorkspace {
  float *part_o;
  float *part_ml;
  size_t bytes;
};

DecodeWorkspace decode_workspace(void *base, int32_t B, int n_split_max) {
  DecodeWorkspace w;
  uint8_t *p = static_cast<uint8_t *>(base);
  size_t off = 0;
  w.part_o = reinterpret_cast<float *>(p + off);
  off += round_up((size_t)B * kHkv * n_split_max * kGroup * kD * 4, 256);
  w.part_ml = reinterpret_cast<float *>(p + off);
  off += round_up((size_t)B * kHkv * n_split_max * kGroup * 2 * 4, 256);
  w.bytes = off;
  return w;
}

}  // namespace

extern "C" {

void beam_default_params(beam_attn_params *p) {
  if (!p) return;
  p->n_q_heads = kHq;
  p->n_kv_heads = kHkv;
  p->head_dim = kD;
  p->window = 512;
  p->rope_theta = 10000.f;
  p->rms_eps = 1e-6f;
  p->ssmax_base = 2048.f;
  p->ssmax_exp = 0.1f;
  p->softmax_scale = (float)(1.0 / std::sqrt(128.0));
}

int beam_kv_layout(int kind, const beam_attn_params *p, int32_t batch, int64_t capacity_tokens,
                   beam_kv_layout_t *out) {
  int st = check_params(kind, p);
  if (st) return st;
  if (!out || batch < 0) return BEAM_ERR_INVALID_ARG;
  const int64_t slots = kind == BEAM_LOCAL ? (int64_t)p->window : capacity_tokens;
  if (slots < 1) return BEAM_ERR_INVALID_ARG;
  out->slots_per_seq = slots;
  out->stride_slot = kD;
  out->stride_head = slots * kD;
  out->stride_seq = (int64_t)kHkv * slots * kD;
  out->bytes_k = (int64_t)batch * out->stride_seq * 2;
  out->bytes_v = out->bytes_k;
  return BEAM_OK;
}

size_t beam_prefill_workspace_bytes(const beam_attn_params *p, int32_t B, int32_t T) {
  (void)p;
  if (B <= 0 || T <= 0) return 0;
  const size_t tok = (size_t)B * T;
  // prepared keys [B][T][8][128] bf16, then the RoPE cos/sin table [T][128] fp32
  return round_up(tok * kHkv * kD * 2, 256) + round_up((size_t)T * 128 * 4, 256);
}

int beam_attn_prefill(int kind, const beam_attn_params *p, int32_t B, int32_t T, const void *q,
                      const void *k, const void *v, const void *gate, const float *q_norm_w,
                      const float *k_norm_w, const float *gate_bias, void *out, void *k_cache,
                      void *v_cache, const beam_kv_layout_t *layout, void *workspace,
                      size_t workspace_bytes, int32_t *dev_status, beam_stream_t stream) {
  int st = check_params(kind, p);
  if (st) return st;
  if (B < 0 || T < 0) return BEAM_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return BEAM_OK;
  if (!q || !k || !v || !gate || !q_norm_w || !k_norm_w || !gate_bias || !out)
    return BEAM_ERR_INVALID_ARG;
  if ((k_cache == nullptr) != (v_cache == nullptr)) return BEAM_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(out) ||
      !aligned16(q_norm_w) || !aligned16(k_norm_w) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(workspace))
    return BEAM_ERR_ALIGNMENT;
  if (k_cache) {
    st = check_layout(kind, p, layout);
    if (st) return st;
    if (kind == BEAM_GLOBAL && layout->slots_per_seq < T) return BEAM_ERR_CAPACITY;
  }
  const size_t need = beam_prefill_workspace_bytes(p, B, T);
  if (!workspace || workspace_bytes < need) return BEAM_ERR_WORKSPACE;
  if ((int64_t)B * T > INT32_MAX) return BEAM_ERR_UNSUPPORTED;
  DeviceInfo *dev = nullptr;
  if ((st = device_info(&dev))) return st;

  const size_t tok = (size_t)B * T;
  uint16_t *kn = static_cast<uint16_t *>(workspace);
  float *rope_tab = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                              round_up(tok * kHkv * kD * 2, 256));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  PrologueArgs pa;
  memset(&pa, 0, sizeof pa);
  pa.k = static_cast<const uint16_t *>(k);
  pa.v = static_cast<const uint16_t *>(v);
  pa.kw = k_norm_w;   // queries are normalised inside the attention kernel
  pa.k_out = kn;
  pa.rope_tab = kind == BEAM_LOCAL ? rope_tab : nullptr;
  pa.k_cache = static_cast<uint16_t *>(k_cache);
  pa.v_cache = static_cast<uint16_t *>(v_cache);
  if (k_cache) {
    pa.stride_seq = layout->stride_seq;
    pa.stride_head = layout->stride_head;
    pa.slots = layout->slots_per_seq;
  }
  pa.pos0 = nullptr;
  pa.status = dev_status;
  pa.T = T;
  pa.kind = kind;
  pa.window = p->window;
  pa.eps = p->rms_eps;
  fill_inv_freq(pa.inv_freq, p->rope_theta);
  prologue_kernel<<<(unsigned)tok, 128, 0, s>>>(pa);
  if ((st = launch_status())) return st;

  if ((st = encode_fn())) return st;
  CUtensorMap tm_q, tm_k, tm_v;
  if ((st = make_head_map(&tm_q, q, kHq, T, B))) return st;
  if ((st = make_head_map(&tm_k, kn, kHkv, T, B))) return st;
  if ((st = make_head_map(&tm_v, v, kHkv, T, B))) return st;
  PrefillTcArgs fa;
  memset(&fa, 0, sizeof fa);
  fa.q_norm_w = q_norm_w;
  fa.rope_tab = kind == BEAM_LOCAL ? rope_tab : nullptr;
  fa.gate = static_cast<const uint16_t *>(gate);
  fa.gate_bias = gate_bias;
  fa.out = static_cast<uint16_t *>(out);
  fa.status = dev_status;
  fa.v_scale = 1.0f;
  return launch_prefill_attention(kind, p, B, T, tm_q, tm_k, tm_v, fa, dev, s);
}

}  // extern "C"

namespace {

// Split-K plan of a chunk of T <= 16 new tokens (decode_tc_kernel): key coordinates
// covered per sequence (at most), run length per CTA and runs per sequence.
struct MultiPlan {
  int n_mt;            // m-tiles of two new tokens
  int64_t range;       // largest number of key coordinates one sequence spans
  int split;           // coordinates per CTA (multiple of the 64-row tile)
  int n_split_max;
};

MultiPlan multi_plan(int kind, const beam_attn_params *p, int32_t B, int32_t T, int64_t slots,
                     int sm_count) {
  MultiPlan m;
  m.n_mt = (T + kMultiTokPerTile - 1) / kMultiTokPerTile;
  m.range = kind == BEAM_LOCAL ? (int64_t)p->window - 1 + T : slots;
  // one CTA per SM fits (225 KB of shared memory): about two waves, runs of whole
  // 128-key tiles
  const int64_t target = (int64_t)sm_count * 2;
  const int64_t per_run = (int64_t)B * kHkv;
  const int64_t runs = std::max<int64_t>(1, target / per_run);
  const int64_t split = std::max<int64_t>(kTcBN, round_up((size_t)((m.range + runs - 1) / runs),
                                                          kTcBN));
  m.split = (int)std::min<int64_t>(split, INT32_MAX / 2);
  m.n_split_max = (int)((m.range + m.split - 1) / m.split);
  return m;
}

// One bf16 view of an FP8 cache (the cache's element strides, two bytes an element).
size_t fp8_view_bytes(int32_t B, const beam_kv_layout_t *layout) {
  return round_up((size_t)B * (size_t)layout->stride_seq * 2, 256);
}

// Runs per sequence up to which the multi-token kernel merges them itself (the last CTA of
// each (sequence, KV head)); beyond it a merge kernel spreads the work over many CTAs.
constexpr int kFoldMaxSplits = kFoldMaxSplitsDev;

// partials o [B][8][n_mt][n_split_max][16][128] and (m, l), then the merge tickets [B][8]
size_t multi_partial_bytes(int32_t B, const MultiPlan &m) {
  const size_t parts = (size_t)B * kHkv * m.n_mt * m.n_split_max * 16;
  return round_up(parts * kD * 4, 256) + round_up(parts * 2 * 4, 256) +
         round_up((size_t)B * kHkv * 4, 256);
}

size_t chunk_workspace_bytes(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                             const beam_kv_layout_t *layout, bool fp8);
int chunk_call(int kind, const beam_attn_params *p, int32_t B, int32_t T, const void *q,
               const void *k, const void *v, const void *gate, const float *q_norm_w,
               const float *k_norm_w, const float *gate_bias, const int64_t *pos0, void *out,
               void *k_cache, void *v_cache, const beam_kv_layout_t *layout, void *workspace,
               size_t workspace_bytes, int32_t *dev_status, beam_stream_t stream, bool fp8,
               float k_scale, float v_scale);

}  // namespace


extern "C" {

size_t beam_prefill_chunk_workspace_bytes(int kind, const beam_attn_params *p, int32_t B,
                                          int32_t T, const beam_kv_layout_t *layout) {
  return chunk_workspace_bytes(kind, p, B, T, layout, false);
}

size_t beam_prefill_chunk_fp8_workspace_bytes(int kind, const beam_attn_params *p, int32_t B,
                                              int32_t T, const beam_kv_layout_t *layout) {
  if (kind == BEAM_GLOBAL && !layout) return 0;
  return chunk_workspace_bytes(kind, p, B, T, layout, true);
}

int beam_attn_prefill_chunk(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                            const void *q, const void *k, const void *v, const void *gate,
                            const float *q_norm_w, const float *k_norm_w, const float *gate_bias,
                            const int64_t *pos0, void *out, void *k_cache, void *v_cache,
                            const beam_kv_layout_t *layout, void *workspace,
                            size_t workspace_bytes, int32_t *dev_status, beam_stream_t stream) {
  return chunk_call(kind, p, B, T, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0, out,
                    k_cache, v_cache, layout, workspace, workspace_bytes, dev_status, stream,
                    false, 1.0f, 1.0f);
}

int beam_attn_prefill_chunk_fp8(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                                const void *q, const void *k, const void *v, const void *gate,
                                const float *q_norm_w, const float *k_norm_w,
                                const float *gate_bias, const int64_t *pos0, void *out,
                                void *k_cache, void *v_cache, const beam_kv_layout_t *layout,
                                float k_scale, float v_scale, void *workspace,
                                size_t workspace_bytes, int32_t *dev_status, beam_stream_t stream) {
  return chunk_call(kind, p, B, T, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0, out,
                    k_cache, v_cache, layout, workspace, workspace_bytes, dev_status, stream,
                    true, k_scale, v_scale);
}

}  // extern "C"

namespace {

// Workspace of a chunk call: for a local layer the ring rows it still sees and the new rows
// ([B][window - 1 + T][8][128] bf16, keys and values) and the RoPE table [B][T][128] fp32;
// for T <= 16 the split-K partials and merge tickets; for a global layer over an FP8 cache
// the bf16 view of the cache (keys and values, the cache's element strides) at the end.
size_t chunk_workspace_bytes(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                             const beam_kv_layout_t *layout, bool fp8) {
  if (!p || B <= 0 || T <= 0 || p->window < 1) return 0;
  size_t bytes = 0;
  if (kind == BEAM_LOCAL) {
    // keys and values [B][window - 1 + T][8][128] bf16 (the ring rows the chunk still sees,
    // then the new rows), then the RoPE table [B][T][128] fp32
    const size_t rows = (size_t)B * ((size_t)p->window - 1 + T);
    bytes = 2 * round_up(rows * kHkv * kD * 2, 256) + round_up((size_t)B * T * 128 * 4, 256);
  }
  if (T <= kMultiMaxT) {  // split-K partials of the few-token path
    DeviceInfo *dev = nullptr;
    int sm = 148;
    if (device_info(&dev) == BEAM_OK) sm = dev->sm_count;
    const int64_t slots = layout ? layout->slots_per_seq : (int64_t)p->window;
    bytes += multi_partial_bytes(B, multi_plan(kind, p, B, T, slots, sm));
  }
  // a long global chunk over an FP8 cache reads a bf16 view; a few-token one widens the
  // code tiles in the kernel
  if (fp8 && kind == BEAM_GLOBAL && T > kMultiMaxT) bytes += 2 * fp8_view_bytes(B, layout);
  return bytes;
}

int chunk_call(int kind, const beam_attn_params *p, int32_t B, int32_t T, const void *q,
               const void *k, const void *v, const void *gate, const float *q_norm_w,
               const float *k_norm_w, const float *gate_bias, const int64_t *pos0, void *out,
               void *k_cache, void *v_cache, const beam_kv_layout_t *layout, void *workspace,
               size_t workspace_bytes, int32_t *dev_status, beam_stream_t stream, bool fp8,
               float k_scale, float v_scale) {
  int st = check_params(kind, p);
  if (st) return st;
  if (B < 0 || T < 0) return BEAM_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return BEAM_OK;
  if (!q || !k || !v || !gate || !q_norm_w || !k_norm_w || !gate_bias || !pos0 || !out ||
      !k_cache || !v_cache)
    return BEAM_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(out) ||
      !aligned16(q_norm_w) || !aligned16(k_norm_w) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(pos0) & 7u))
    return BEAM_ERR_ALIGNMENT;
  if ((st = fp8 ? check_layout_fp8(kind, p, layout) : check_layout(kind, p, layout))) return st;
  if (fp8 && (!valid_scale(k_scale) || !valid_scale(v_scale))) return BEAM_ERR_INVALID_ARG;
  const bool local = kind == BEAM_LOCAL;
  if (!local && layout->slots_per_seq < T) return BEAM_ERR_CAPACITY;
  if (!local && layout->slots_per_seq > INT32_MAX - kTcBN) return BEAM_ERR_UNSUPPORTED;
  const size_t need = chunk_workspace_bytes(kind, p, B, T, layout, fp8);
  if (need && (!workspace || workspace_bytes < need)) return BEAM_ERR_WORKSPACE;
  const int64_t ext_rows = local ? (int64_t)p->window - 1 + T : T;
  if ((int64_t)B * ext_rows > INT32_MAX) return BEAM_ERR_UNSUPPORTED;
  DeviceInfo *dev = nullptr;
  if ((st = device_info(&dev))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  const size_t ext_bytes = round_up((size_t)B * ext_rows * kHkv * kD * 2, 256);
  uint16_t *k_ext = local ? static_cast<uint16_t *>(workspace) : nullptr;
  uint16_t *v_ext = local ? reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(workspace) +
                                                         ext_bytes)
                          : nullptr;
  float *rope_tab = local ? reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                                      2 * ext_bytes)
                          : nullptr;
  const int prefix = local ? p->window - 1 : 0;

  // the ring rows the chunk still sees (local), or the value padding (global): extra CTAs of
  // the prologue launch
  ChunkPrepArgs ca;
  ca.pos0 = pos0;
  ca.k_cache = static_cast<const uint16_t *>(k_cache);
  ca.v_cache = static_cast<uint16_t *>(v_cache);   // the view instead for an FP8 cache (below)
  ca.v_ring = static_cast<const uint16_t *>(v_cache);
  ca.fp8 = fp8;
  ca.stride_seq = layout->stride_seq;
  ca.stride_head = layout->stride_head;
  ca.slots = layout->slots_per_seq;
  ca.k_ext = k_ext;
  ca.v_ext = v_ext;
  ca.ext_rows = (int)ext_rows;
  ca.prefix = prefix;
  ca.T = T;
  ca.window = p->window;
  ca.kind = kind;
  const int64_t prep_ctas = (int64_t)B * (local ? prefix : kChunkPadRows);

  // the few-token path's plan and workspace (split-K partials, merge tickets)
  const bool few = T <= kMultiMaxT;
  MultiPlan mp{};
  uint8_t *pw = nullptr;
  size_t parts = 0;
  bool fold = false;
  if (few) {
    mp = multi_plan(kind, p, B, T, layout->slots_per_seq, dev->sm_count);
    pw = static_cast<uint8_t *>(workspace) +
         (local ? 2 * ext_bytes + round_up((size_t)B * T * 128 * 4, 256) : 0);
    parts = (size_t)B * kHkv * mp.n_mt * mp.n_split_max * 16;
    fold = mp.n_split_max > 1 && mp.n_split_max <= kFoldMaxSplits;
  }
  uint32_t *tickets = few ? reinterpret_cast<uint32_t *>(pw + round_up(parts * kD * 4, 256) +
                                                         round_up(parts * 2 * 4, 256))
                          : nullptr;
  // a global layer over an FP8 cache: the attention reads a bf16 view of the cache (the
  // codes' unscaled values) at the end of the workspace; the cached rows are converted
  // first, the prologue writes the new rows into both
  uint16_t *k_view = nullptr, *v_view = nullptr;
  const bool widen_in_kernel = fp8 && !local && few;   // decode_tc_kernel<true>
  if (fp8 && !local && !few) {
    const size_t vb = fp8_view_bytes(B, layout);
    uint8_t *end = static_cast<uint8_t *>(workspace) + need;
    k_view = reinterpret_cast<uint16_t *>(end - 2 * vb);
    v_view = reinterpret_cast<uint16_t *>(end - vb);
    Fp8ViewArgs fv;
    fv.pos0 = pos0;
    fv.k_codes = static_cast<const uint8_t *>(k_cache);
    fv.v_codes = static_cast<const uint8_t *>(v_cache);
    fv.k_view = k_view;
    fv.v_view = v_view;
    fv.stride_seq = layout->stride_seq;
    fv.stride_head = layout->stride_head;
    fv.slots = layout->slots_per_seq;
    const int64_t blocks = (layout->slots_per_seq + kViewSlots - 1) / kViewSlots;
    if (blocks > INT32_MAX || B > 65535) return BEAM_ERR_UNSUPPORTED;
    fp8_view_kernel<<<dim3((unsigned)blocks, kHkv, B), 256, 0, s>>>(fv);
    if ((st = launch_status())) return st;
  }
  // the caches the attention kernels read as bf16
  void *k_att = k_view ? static_cast<void *>(k_view) : k_cache;
  void *v_att = v_view ? static_cast<void *>(v_view) : v_cache;
  ca.v_cache = static_cast<uint16_t *>(v_att);   // global: the value padding the attention reads

  // 1. prepared keys (and raw values) of the new tokens: into the cache and, for a local
  //    layer, behind the earlier rows; the RoPE table at each sequence's own positions (and
  //    the merge tickets of the few-token path zeroed)
  PrologueArgs pa;
  memset(&pa, 0, sizeof pa);
  pa.k = static_cast<const uint16_t *>(k);
  pa.v = static_cast<const uint16_t *>(v);
  pa.kw = k_norm_w;
  pa.k_out = k_ext;
  pa.v_out = v_ext;
  pa.out_rows = (int)ext_rows;
  pa.out_row0 = prefix;
  pa.k_cache = static_cast<uint16_t *>(k_cache);
  pa.v_cache = static_cast<uint16_t *>(v_cache);
  pa.stride_seq = layout->stride_seq;
  pa.stride_head = layout->stride_head;
  pa.slots = layout->slots_per_seq;
  pa.pos0 = pos0;
  pa.rope_tab = rope_tab;
  pa.rope_per_seq = 1;
  pa.whole_seq = 1;
  pa.status = dev_status;
  pa.T = T;
  pa.kind = kind;
  pa.window = p->window;
  pa.eps = p->rms_eps;
  fill_inv_freq(pa.inv_freq, p->rope_theta);
  pa.prep = ca;
  // the in-kernel widening zeroes keys past the last visible one itself: no value padding
  // (which would treat the code array as bf16)
  pa.n_prep = widen_in_kernel ? 0 : (int)prep_ctas;
  pa.ring_save = local;
  pa.tickets = fold ? tickets : nullptr;
  pa.cache_fp8 = fp8;
  pa.k_scale = k_scale;
  pa.v_scale = v_scale;
  pa.k_view = k_view;
  pa.v_view = v_view;
  if ((int64_t)B * T + pa.n_prep > INT32_MAX) return BEAM_ERR_UNSUPPORTED;
  if ((st = launch_pdl(prologue_kernel, dim3((unsigned)((int64_t)B * T + pa.n_prep)), dim3(128), 0,
                       s, pa)))
    return st;

  // 2. attention of the new rows over the earlier and the new keys
  if (few) {
    // a few new tokens (multi-token decode): split the keys across CTAs, then merge (in the
    // same kernel when a sequence's keys span at most kFoldMaxSplits runs)
    if ((st = encode_fn())) return st;
    CUtensorMap tk, tv;
    if (local) {
      if ((st = make_head_map(&tk, k_ext, kHkv, (int)ext_rows, B))) return st;
      if ((st = make_head_map(&tv, v_ext, kHkv, (int)ext_rows, B))) return st;
    } else if (widen_in_kernel) {
      if ((st = make_cache_map_u8(&tk, k_cache, layout, B))) return st;
      if ((st = make_cache_map_u8(&tv, v_cache, layout, B))) return st;
    } else {
      if ((st = make_cache_map(&tk, k_att, layout, B))) return st;
      if ((st = make_cache_map(&tv, v_att, layout, B))) return st;
    }
    DecodeTcArgs da;
    memset(&da, 0, sizeof da);
    da.q_raw = static_cast<const uint16_t *>(q);
    da.qw = q_norm_w;
    da.eps = p->rms_eps;
    da.rope_tab = rope_tab;
    da.pos0 = pos0;
    da.kind = kind;
    da.window = p->window;
    da.T = T;
    da.prefix = prefix;
    da.slots = layout->slots_per_seq;
    da.split = mp.split;
    da.n_split_max = mp.n_split_max;
    da.n_mt = mp.n_mt;
    da.scale_log2 = p->softmax_scale * kLog2e;
    da.ssmax_base = p->ssmax_base;
    da.ssmax_exp = p->ssmax_exp;
    da.part_o = reinterpret_cast<float *>(pw);
    da.part_ml = reinterpret_cast<float *>(pw + round_up(parts * kD * 4, 256));
    da.status = dev_status;
    da.kv_slot_major = local ? 0 : 1;
    // a plan with one split (many sequences, or a short history) needs no merge: the CTA
    // that sees every key of its (sequence, KV head) writes the gated output itself
    da.direct = mp.n_split_max == 1;
    da.fold = fold;
    da.tickets = tickets;
    da.k_scale = k_scale;
    da.v_scale = v_scale;
    da.gate = static_cast<const uint16_t *>(gate);
    da.gate_bias = gate_bias;
    da.out = static_cast<uint16_t *>(out);
    {  // the same test-only fault injection as the prefill kernel's
      const char *f = std::getenv("BEAM_FAULT_INJECT");
      da.fault_stall = f != nullptr && std::strcmp(f, "prefill_wait_stall") == 0;
    }
    if (mp.n_split_max > 65535 || B > 65535) return BEAM_ERR_UNSUPPORTED;
    if ((st = launch_pdl(widen_in_kernel ? decode_tc_kernel<true> : decode_tc_kernel<false>,
                         dim3(mp.n_split_max, kHkv, B), dim3(kDtThreads), kDtSmemBytes, s, tk, tv,
                         da)))
      return st;
    if (da.direct || da.fold) return BEAM_OK;
    MultiCombineArgs mc;
    mc.part_o = da.part_o;
    mc.part_ml = da.part_ml;
    mc.pos0 = pos0;
    mc.gate = static_cast<const uint16_t *>(gate);
    mc.gate_bias = gate_bias;
    mc.out = static_cast<uint16_t *>(out);
    mc.kind = kind;
    mc.window = p->window;
    mc.T = T;
    mc.n_mt = mp.n_mt;
    mc.prefix = prefix;
    mc.split = mp.split;
    mc.n_split_max = mp.n_split_max;
    mc.slots = layout->slots_per_seq;
    decode_multi_combine_kernel<<<dim3(kHq, T, B), kCombineThreads, 0, s>>>(mc);
    return launch_status();
  }
  if ((st = encode_fn())) return st;
  CUtensorMap tm_q, tm_k, tm_v;
  if ((st = make_head_map(&tm_q, q, kHq, T, B))) return st;
  if (local) {
    if ((st = make_head_map(&tm_k, k_ext, kHkv, (int)ext_rows, B))) return st;
    if ((st = make_head_map(&tm_v, v_ext, kHkv, (int)ext_rows, B))) return st;
  } else {
    if ((st = make_cache_map(&tm_k, k_att, layout, B))) return st;
    if ((st = make_cache_map(&tm_v, v_att, layout, B))) return st;
  }
  PrefillTcArgs fa;
  memset(&fa, 0, sizeof fa);
  fa.q_norm_w = q_norm_w;
  fa.rope_tab = rope_tab;
  fa.rope_rows = T;
  fa.gate = static_cast<const uint16_t *>(gate);
  fa.gate_bias = gate_bias;
  fa.out = static_cast<uint16_t *>(out);
  fa.status = dev_status;
  fa.pos0 = pos0;
  fa.slots = layout->slots_per_seq;
  fa.ext_prefix = prefix;
  fa.kv_slot_major = local ? 0 : 1;
  fa.v_scale = v_scale;
  return launch_prefill_attention(kind, p, B, T, tm_q, tm_k, tm_v, fa, dev, s, k_scale);
}

}  // namespace

extern "C" {

int beam_kv_append(int kind, const beam_attn_params *p, int32_t B, int32_t T, const void *k,
                   const void *v, const float *k_norm_w, const int64_t *pos0, void *k_cache,
                   void *v_cache, const beam_kv_layout_t *layout, int32_t *dev_status,
                   beam_stream_t stream) {
  int st = check_params(kind, p);
  if (st) return st;
  if (B < 0 || T < 0) return BEAM_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return BEAM_OK;
  if (!k || !v || !k_norm_w || !pos0 || !k_cache || !v_cache) return BEAM_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_norm_w) || !aligned16(k_cache) ||
      !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(pos0) & 7u))
    return BEAM_ERR_ALIGNMENT;
  if ((st = check_layout(kind, p, layout))) return st;
  if ((int64_t)B * T > INT32_MAX) return BEAM_ERR_UNSUPPORTED;
  DeviceInfo *dev = nullptr;
  if ((st = device_info(&dev))) return st;
  PrologueArgs pa;
  memset(&pa, 0, sizeof pa);
  pa.k = static_cast<const uint16_t *>(k);
  pa.v = static_cast<const uint16_t *>(v);
  pa.kw = k_norm_w;
  pa.k_cache = static_cast<uint16_t *>(k_cache);
  pa.v_cache = static_cast<uint16_t *>(v_cache);
  pa.stride_seq = layout->stride_seq;
  pa.stride_head = layout->stride_head;
  pa.slots = layout->slots_per_seq;
  pa.pos0 = pos0;
  pa.status = dev_status;
  pa.T = T;
  pa.kind = kind;
  pa.window = p->window;
  pa.eps = p->rms_eps;
  fill_inv_freq(pa.inv_freq, p->rope_theta);
  prologue_kernel<<<(unsigned)((size_t)B * T), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(pa);
  return launch_status();
}

size_t beam_decode_workspace_bytes(int kind, const beam_attn_params *p, int32_t B,
                                   const beam_kv_layout_t *layout) {
  if (check_params(kind, p) || !layout || B <= 0 || layout->slots_per_seq < 1) return 0;
  // a ring decode merges its splits in distributed shared memory: no workspace
  if (kind == BEAM_LOCAL) return kDecodeNoWorkspace;
  DeviceInfo *dev = nullptr;
  int sm = 148;
  if (device_info(&dev) == BEAM_OK) sm = dev->sm_count;
  // one workspace size serves a BF16 and an FP8 cache: the smaller of their splits
  const int split = std::min(decode_split(kind, p, B, layout->slots_per_seq, sm, false),
                             decode_split(kind, p, B, layout->slots_per_seq, sm, true));
  const int64_t vis_max = kind == BEAM_LOCAL ? p->window : layout->slots_per_seq;
  const int n_split_max = (int)((vis_max + split - 1) / split);
  return decode_workspace(nullptr, B, n_split_max).bytes;
}

}  // extern "C"

namespace {

// One decode step over a BF16 cache (fp8 == false) or an FP8 E4M3 cache with the given
// scales: validation, then one cluster launch (local ring) or split-K + combine (global).
int decode_call(int kind, const beam_attn_params *p, int32_t B, const void *q, const void *k,
                const void *v, const void *gate, const float *q_norm_w, const float *k_norm_w,
                const float *gate_bias, const int64_t *pos, void *k_cache, void *v_cache,
                const beam_kv_layout_t *layout, void *out, void *workspace,
                size_t workspace_bytes, int32_t *dev_status, beam_stream_t stream, bool fp8,
                float k_scale, float v_scale) {
  int st = check_params(kind, p);
  if (st) return st;
  if (B < 0) return BEAM_ERR_INVALID_ARG;
  if (B == 0) return BEAM_OK;
  if (!q || !k || !v || !gate || !q_norm_w || !k_norm_w || !gate_bias || !pos || !k_cache ||
      !v_cache || !out)
    return BEAM_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(out) ||
      !aligned16(q_norm_w) || !aligned16(k_norm_w) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(pos) & 7u))
    return BEAM_ERR_ALIGNMENT;
  if ((st = fp8 ? check_layout_fp8(kind, p, layout) : check_layout(kind, p, layout))) return st;
  if (fp8 && (!valid_scale(k_scale) || !valid_scale(v_scale))) return BEAM_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  if ((st = device_info(&dev))) return st;
  const int split = decode_split(kind, p, B, layout->slots_per_seq, dev->sm_count, fp8);
  const int64_t vis_max = kind == BEAM_LOCAL ? p->window : layout->slots_per_seq;
  const int n_split_max = (int)((vis_max + split - 1) / split);
  // only the split-K path of a global layer keeps partial results in the workspace
  DecodeWorkspace w = decode_workspace(workspace, B, n_split_max);
  if (kind == BEAM_GLOBAL && (!workspace || workspace_bytes < w.bytes)) return BEAM_ERR_WORKSPACE;
  if (n_split_max > 65535) return BEAM_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  DecodeArgs da;
  memset(&da, 0, sizeof da);
  da.k_cache = static_cast<uint16_t *>(k_cache);
  da.v_cache = static_cast<uint16_t *>(v_cache);
  da.stride_seq = layout->stride_seq;
  da.stride_head = layout->stride_head;
  da.slots = layout->slots_per_seq;
  da.pos = pos;
  da.kind = kind;
  da.window = p->window;
  da.split = split;
  da.n_split_max = n_split_max;
  da.scale_log2 = p->softmax_scale * kLog2e;
  da.ssmax_base = p->ssmax_base;
  da.ssmax_exp = p->ssmax_exp;
  da.part_o = w.part_o;
  da.part_ml = w.part_ml;
  dim3 grid(n_split_max, kHkv, B);
  // every CTA normalises (local: rotates) its group's queries; the owner of the new
  // token's slot also appends its key and value
  da.q_raw = static_cast<const uint16_t *>(q);
  da.k_raw = static_cast<const uint16_t *>(k);
  da.v_raw = static_cast<const uint16_t *>(v);
  da.gate = static_cast<const uint16_t *>(gate);
  da.qw = q_norm_w;
  da.kw = k_norm_w;
  da.gate_bias = gate_bias;
  da.out = static_cast<uint16_t *>(out);
  da.status = dev_status;
  da.eps = p->rms_eps;
  fill_inv_freq(da.inv_freq, p->rope_theta);
  Decode8Args d8;
  d8.base = da;
  d8.k_scale = k_scale;
  d8.v_scale = v_scale;

  if (kind == BEAM_LOCAL) {
    // one launch: the ring's splits form a cluster that also merges through distributed
    // shared memory and gates
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = fp8 ? kDec8Smem : kDecSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)n_split_max;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cuda_status(fp8 ? cudaLaunchKernelEx(&cfg, decode8_attn_kernel<true>, d8)
                           : cudaLaunchKernelEx(&cfg, decode_attn_kernel<true>, da),
                       "ring decode launch");
  }

  if ((st = fp8 ? launch_pdl(decode8_attn_kernel<false>, grid, dim3(kDecThreads), kDec8Smem, s, d8)
                : launch_pdl(decode_attn_kernel<false>, grid, dim3(kDecThreads), kDecSmem, s, da)))
    return st;

  CombineArgs ca;
  ca.part_o = w.part_o;
  ca.part_ml = w.part_ml;
  ca.pos = pos;
  ca.gate = static_cast<const uint16_t *>(gate);
  ca.gate_bias = gate_bias;
  ca.out = static_cast<uint16_t *>(out);
  ca.kind = kind;
  ca.window = p->window;
  ca.split = split;
  ca.n_split_max = n_split_max;
  ca.slots = layout->slots_per_seq;
  return launch_pdl(decode_combine_kernel, dim3(kHq, B), dim3(kCombineThreads), 0, s, ca);
}

}  // namespace

extern "C" {

int beam_attn_decode(int kind, const beam_attn_params *p, int32_t B, const void *q, const void *k,
                     const void *v, const void *gate, const float *q_norm_w,
                     const float *k_norm_w, const float *gate_bias, const int64_t *pos,
                     void *k_cache, void *v_cache, const beam_kv_layout_t *layout, void *out,
                     void *workspace, size_t workspace_bytes, int32_t *dev_status,
                     beam_stream_t stream) {
  return decode_call(kind, p, B, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos, k_cache,
                     v_cache, layout, out, workspace, workspace_bytes, dev_status, stream, false,
                     1.0f, 1.0f);
}

int beam_attn_decode_fp8(int kind, const beam_attn_params *p, int32_t B, const void *q,
                         const void *k, const void *v, const void *gate, const float *q_norm_w,
                         const float *k_norm_w, const float *gate_bias, const int64_t *pos,
                         void *k_cache, void *v_cache, const beam_kv_layout_t *layout,
                         float k_scale, float v_scale, void *out, void *workspace,
                         size_t workspace_bytes, int32_t *dev_status, beam_stream_t stream) {
  return decode_call(kind, p, B, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos, k_cache,
                     v_cache, layout, out, workspace, workspace_bytes, dev_status, stream, true,
                     k_scale, v_scale);
}

int beam_kv_layout_fp8(int kind, const beam_attn_params *p, int32_t batch,
                       int64_t capacity_tokens, beam_kv_layout_t *out) {
  int st = beam_kv_layout(kind, p, batch, capacity_tokens, out);
  if (st) return st;
  out->bytes_k = (int64_t)batch * out->stride_seq;   // one byte per element
  out->bytes_v = out->bytes_k;
  return BEAM_OK;
}

int beam_kv_append_fp8(int kind, const beam_attn_params *p, int32_t B, int32_t T, const void *k,
                       const void *v, const float *k_norm_w, const int64_t *pos0, void *k_cache,
                       void *v_cache, const beam_kv_layout_t *layout, float k_scale,
                       float v_scale, int32_t *dev_status, beam_stream_t stream) {
  int st = check_params(kind, p);
  if (st) return st;
  if (B < 0 || T < 0) return BEAM_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return BEAM_OK;
  if (!k || !v || !k_norm_w || !pos0 || !k_cache || !v_cache) return BEAM_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_norm_w) || !aligned16(k_cache) ||
      !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(pos0) & 7u))
    return BEAM_ERR_ALIGNMENT;
  if ((st = check_layout_fp8(kind, p, layout))) return st;
  if (!valid_scale(k_scale) || !valid_scale(v_scale)) return BEAM_ERR_INVALID_ARG;
  if ((int64_t)B * T > INT32_MAX) return BEAM_ERR_UNSUPPORTED;
  DeviceInfo *dev = nullptr;
  if ((st = device_info(&dev))) return st;
  PrologueArgs pa;
  memset(&pa, 0, sizeof pa);
  pa.k = static_cast<const uint16_t *>(k);
  pa.v = static_cast<const uint16_t *>(v);
  pa.kw = k_norm_w;
  pa.k_cache = static_cast<uint16_t *>(k_cache);
  pa.v_cache = static_cast<uint16_t *>(v_cache);
  pa.stride_seq = layout->stride_seq;
  pa.stride_head = layout->stride_head;
  pa.slots = layout->slots_per_seq;
  pa.pos0 = pos0;
  pa.cache_fp8 = 1;
  pa.k_scale = k_scale;
  pa.v_scale = v_scale;
  pa.status = dev_status;
  pa.T = T;
  pa.kind = kind;
  pa.window = p->window;
  pa.eps = p->rms_eps;
  fill_inv_freq(pa.inv_freq, p->rope_theta);
  prologue_kernel<<<(unsigned)((size_t)B * T), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(pa);
  return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Fixed device scratch of beam_attn_decode_noalloc.  In host code the name
// g_decode_scratch is only a host-side stand-in for the array, not its device
// address: passing it to a kernel would fault or, where the GPU can reach host
// memory, silently touch the wrong memory.  The device address is looked up
// once per device with cudaGetSymbolAddress while that device is current.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocScratchBytes];

void *g_scratch_addr[kMaxDevices];

int noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BEAM_ERR_CUDA;
  if (!g_scratch_addr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return BEAM_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return BEAM_OK;
}

}  // namespace

extern "C" {

int beam_attn_decode_noalloc(int kind, const beam_attn_params *p, int32_t B, const void *q,
                             const void *k, const void *v, const void *gate,
                             const float *q_norm_w, const float *k_norm_w,
                             const float *gate_bias, const int64_t *pos, void *k_cache,
                             void *v_cache, const beam_kv_layout_t *layout, void *out,
                             int32_t *dev_status, beam_stream_t stream) {
  int st = check_params(kind, p);
  if (st) return st;
  if (B < 0) return BEAM_ERR_INVALID_ARG;
  if (B == 0) return BEAM_OK;
  if ((st = check_layout(kind, p, layout))) return st;
  // a local (ring) decode keeps nothing in the scratch; a global one needs the
  // split-K partials of all its sequences to fit
  if (kind == BEAM_GLOBAL) {
    const size_t need = beam_decode_workspace_bytes(kind, p, B, layout);
    if (need == 0) return BEAM_ERR_CUDA;
    if (need > kNoAllocScratchBytes) return BEAM_ERR_SCRATCH_LIMIT;
  }
  void *scratch = nullptr;
  if ((st = noalloc_scratch(&scratch))) return st;
  return beam_attn_decode(kind, p, B, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos, k_cache,
                          v_cache, layout, out, scratch, kNoAllocScratchBytes, dev_status, stream);
}

const char *beam_status_string(int status) {
  switch (status) {
    case BEAM_OK: return "ok";
    case BEAM_ERR_INVALID_ARG: return "invalid argument";
    case BEAM_ERR_UNSUPPORTED: return "unsupported head layout or size";
    case BEAM_ERR_CUDA: return "CUDA launch or query failed";
    case BEAM_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case BEAM_ERR_CAPACITY: return "position does not fit the cache";
    case BEAM_ERR_WORKSPACE: return "workspace missing or too small";
    case BEAM_ERR_ALIGNMENT: return "tensor pointer or stride not 16-byte aligned";
    case BEAM_ERR_SCRATCH_LIMIT: return "call needs more than the fixed 8 MiB decode scratch";
    default: return "unknown status";
  }
}

}  // extern "C"
