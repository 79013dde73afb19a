/*
 * beam_attn.h -- C ABI of the Beam 1.0 attention core on NVIDIA B200 (sm_100a).
 *
 * The operation is the attention sublayer of "Beam 1.0: Local RoPE, Global NoPE
 * and Scalable Softmax" (flozi.net), from the post-projection tensors up to the
 * gated output that feeds W_o:
 *
 *   section "Follow the tensors, not the parameter label":
 *     - Q [B,T,48*128], K and V [B,T,8*128], gate logits G [B,T,48*128];
 *     - RMSNorm of Q and K along the 128-wide head axis, eps 1e-6, learned weight
 *       (multiplied directly); V is not normalised;
 *     - local layers rotate normalised Q and K with RoPE (theta 10000, rotate-half
 *       pairing of coordinate i with i+64, angle t * theta^(-2i/128), t 0-based);
 *     - global layers leave K unrotated and multiply only Q by the scalable-softmax
 *       factor a(p) = (1 + p/2048)^0.1, p = t + 1 the one-based absolute position;
 *     - six query heads share each KV head (query head h reads KV head h/6);
 *     - s_j = <q, k_j> / sqrt(128), softmax over the visible keys, O = sum P_j v_j;
 *     - Y = O * sigmoid(G + b_h) per coordinate; the bias b_h is one value per head.
 *   section "Two attention paths in one decoder":
 *     - a local layer sees keys t-511 .. t (the current token and 511 earlier);
 *     - a global layer sees keys 0 .. t.
 *   section "KV memory: nine growing caches, not 52":
 *     - a global layer keeps an append-only cache (4 KiB per token in bf16);
 *     - a local layer keeps a window-sized cache; here a ring of `window` slots,
 *       position j in slot j mod window.
 *
 * Conventions shared by every call:
 *   - bf16 tensors are passed as pointers to 16-bit storage; every tensor pointer
 *     is a DEVICE pointer owned by the caller and must be 16-byte aligned;
 *   - parameter and layout structs are HOST pointers, read during the call only;
 *   - calls are asynchronous on `stream`, never synchronise and never allocate;
 *   - stream order holds as usual: the decode and chunk calls launch their kernels
 *     with programmatic stream serialization, so a kernel may be scheduled while
 *     the one before it on the stream finishes; the first kernel of a call waits for
 *     the kernel before it to complete before it touches any caller buffer or
 *     workspace, and a later kernel of the call waits for the earlier ones before it
 *     reads what they wrote;
 *   - errors found on the host (bad kind, sizes, null or misaligned pointers, a
 *     workspace that is too small) return before any launch, writing nothing;
 *   - launch failures return BEAM_ERR_CUDA;
 *   - conditions only the device can see (a position past a cache's capacity, a
 *     bounded wait that ran out) are written to `dev_status`, a caller-owned
 *     device int32 (nullable).  The library only ever writes error codes into it
 *     and never clears it: the caller sets it to 0 and reads it after the stream.
 *     The kernel that finds the condition skips the affected work and returns.
 *   - the library keeps no state besides cached per-device attributes.
 */
#ifndef BEAM_ATTN_H
#define BEAM_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BEAM_API __attribute__((visibility("default")))
#else
#define BEAM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *beam_stream_t; /* the same type as cudaStream_t */

typedef enum { BEAM_LOCAL = 0, BEAM_GLOBAL = 1 } beam_kind;

typedef enum {
  BEAM_OK = 0,
  BEAM_ERR_INVALID_ARG = -1,    /* null pointer, bad kind, negative size, bad layout */
  BEAM_ERR_UNSUPPORTED = -2,    /* head layout other than 48 / 8 / 128 */
  BEAM_ERR_CUDA = -3,           /* a CUDA launch or query failed */
  BEAM_ERR_DEVICE_TIMEOUT = -4, /* device side: a bounded wait ran out */
  BEAM_ERR_CAPACITY = -5,       /* a position does not fit the cache (host or device) */
  BEAM_ERR_WORKSPACE = -6,      /* workspace null or smaller than the query function says */
  BEAM_ERR_ALIGNMENT = -7,      /* a tensor pointer is not 16-byte aligned */
  BEAM_ERR_SCRATCH_LIMIT = -8   /* beam_attn_decode_noalloc: the call needs more scratch than
                                   the library's fixed device array holds */
} beam_status;

/* Sublayer hyper-parameters.  The kernels are built for 48 query heads, 8 KV
 * heads and head_dim 128 (any other value returns BEAM_ERR_UNSUPPORTED); the
 * window (>= 1), theta, epsilon, the a(p) base and exponent and the softmax
 * scale are runtime values. */
typedef struct {
  int32_t n_q_heads;     /* 48 */
  int32_t n_kv_heads;    /* 8 */
  int32_t head_dim;      /* 128 */
  int32_t window;        /* 512: keys t-window+1 .. t visible in a local layer */
  float rope_theta;      /* 10000 */
  float rms_eps;         /* 1e-6 */
  float ssmax_base;      /* 2048 */
  float ssmax_exp;       /* 0.1 */
  float softmax_scale;   /* 1/sqrt(128) */
} beam_attn_params;

/* Fills the values above. */
BEAM_API void beam_default_params(beam_attn_params *p);

/* KV cache geometry of one layer for a batch.  Rows are head-major:
 * element (b, g, slot, i) sits at b*stride_seq + g*stride_head + slot*stride_slot + i
 * (in elements of 2 bytes).  K and V caches are two separate buffers of bytes_k
 * and bytes_v bytes. */
typedef struct {
  int64_t slots_per_seq; /* local: window; global: capacity in tokens */
  int64_t stride_seq;
  int64_t stride_head;
  int64_t stride_slot;
  int64_t bytes_k;
  int64_t bytes_v;
} beam_kv_layout_t;

/* Pure host function.  A local layer gets `window` slots per sequence whatever
 * capacity_tokens says; a global layer gets capacity_tokens slots (>= 1).
 * The byte counts reproduce the pages' budget: 2 * 8 * 128 * 2 B = 4 KiB per
 * token per global layer in bf16 (section "KV memory"). */
BEAM_API int beam_kv_layout(int kind, const beam_attn_params *p, int32_t batch, int64_t capacity_tokens,
                   beam_kv_layout_t *out);

/* Workspace the prefill call needs for B sequences of T tokens (bytes): the
 * normalised (local: rotated) keys in bf16 and a table of the RoPE cos/sin values
 * of positions 0 .. T-1.  16-byte aligned workspace required. */
BEAM_API size_t beam_prefill_workspace_bytes(const beam_attn_params *p, int32_t B, int32_t T);

/* Prefill of one layer: B sequences of T new tokens at positions 0 .. T-1.
 *   q, gate : [B][T][48*128] bf16     k, v : [B][T][8*128] bf16
 *   q_norm_w, k_norm_w : [128] float32    gate_bias : [48] float32
 *   out : [B][T][48*128] bf16, the gated attention output before W_o.
 *   k_cache, v_cache : both null, or both set together with `layout` (host):
 *     the call also writes the normalised (local: rotated) keys and the raw
 *     values into the cache -- a global cache at slot t, a local ring the last
 *     min(T, window) tokens at slot t mod window.  A global cache must hold T
 *     slots (else BEAM_ERR_CAPACITY before any launch).
 *   workspace : device buffer of at least beam_prefill_workspace_bytes().
 * B = 0 or T = 0 is a no-op that returns BEAM_OK.
 * Every wait inside the attention kernel gives up after about one second of
 * device time: it then writes BEAM_ERR_DEVICE_TIMEOUT to dev_status, lets its
 * in-flight copies and MMAs finish, leaves that part of `out` unwritten and
 * returns, so the CUDA context stays usable.  For tests of that path only, the
 * environment variable BEAM_FAULT_INJECT=prefill_wait_stall (read at each call)
 * makes the kernel start with a wait that nothing satisfies. */
BEAM_API int beam_attn_prefill(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                      const void *q, const void *k, const void *v, const void *gate,
                      const float *q_norm_w, const float *k_norm_w, const float *gate_bias,
                      void *out, void *k_cache, void *v_cache, const beam_kv_layout_t *layout,
                      void *workspace, size_t workspace_bytes, int32_t *dev_status,
                      beam_stream_t stream);

/* Workspace beam_attn_prefill_chunk needs (bytes) for B sequences of T new
 * tokens and the cache `layout`: for a local layer the keys and values
 * [B][window-1+T][8*128] bf16 (the ring rows the chunk still sees, then the new
 * ones) and a RoPE table [B][T][128] fp32; for T <= 16 also the split-K partial
 * results of the few-token path (sized from the layout's slots).  A global
 * chunk of more than 16 tokens needs none (0). */
BEAM_API size_t beam_prefill_chunk_workspace_bytes(int kind, const beam_attn_params *p, int32_t B,
                                                   int32_t T, const beam_kv_layout_t *layout);

/* Chunked prefill of one layer against an existing cache (section "KV memory":
 * a call that continues a sequence reads the earlier keys from the global cache
 * or the local ring).  Sequence b adds T new tokens at positions
 * pos0[b] .. pos0[b]+T-1 (pos0: device int64 [B], 8-byte aligned) after pos0[b]
 * tokens already in k_cache / v_cache (required; `layout` as for decode).  Query
 * row i is position t = pos0[b] + i: RoPE (local) and a(t+1) (global) use t, and
 * it sees every earlier key in its window (local) or all of them (global), plus
 * the chunk's own keys up to t.  Tensors as in beam_attn_prefill; the new keys
 * and values are appended as there, at their own positions (a local ring keeps
 * the last min(T, window) of them).  pos0 = 0 everywhere is a plain prefill.
 * A global call also zeroes the value slots from pos0[b]+T up to the next
 * multiple of 128 below the capacity: they hold no token yet.  A sequence with
 * pos0[b] < 0, or (global) pos0[b] + T > slots_per_seq, sets BEAM_ERR_CAPACITY
 * in dev_status and is neither appended nor written to `out`; the others are
 * unaffected.  T > slots_per_seq (global) is BEAM_ERR_CAPACITY before any launch.
 * Up to 16 new tokens (multi-token decode, e.g. verifying a drafted block) run on
 * a split-K tcgen05 kernel that spreads the history over many CTAs and a merge
 * kernel; when the plan gives each (sequence, KV head) a single CTA (many
 * sequences, or a short history) that CTA applies the gate and writes `out`
 * itself.  Longer chunks run on the tcgen05 prefill kernel.  The bounded waits of both behave as in beam_attn_prefill. */
BEAM_API int beam_attn_prefill_chunk(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                                     const void *q, const void *k, const void *v, const void *gate,
                                     const float *q_norm_w, const float *k_norm_w,
                                     const float *gate_bias, const int64_t *pos0, void *out,
                                     void *k_cache, void *v_cache, const beam_kv_layout_t *layout,
                                     void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                     beam_stream_t stream);

/* Cache append without attention: T tokens per sequence at positions
 * pos0[b] .. pos0[b]+T-1 (pos0: device int64 [B]).  k, v : [B][T][8*128] bf16.
 * Keys are normalised (local: rotated at their own position) and stored in bf16;
 * values are copied.  A local ring receives only the last min(T, window)
 * tokens.  A global position >= slots_per_seq writes nothing for that token and
 * sets BEAM_ERR_CAPACITY in dev_status. */
BEAM_API int beam_kv_append(int kind, const beam_attn_params *p, int32_t B, int32_t T, const void *k,
                   const void *v, const float *k_norm_w, const int64_t *pos0, void *k_cache,
                   void *v_cache, const beam_kv_layout_t *layout, int32_t *dev_status,
                   beam_stream_t stream);

/* Workspace of one decode call (bytes): for a global layer the split-K partial
 * results, sized from the layout's slots per sequence (0: invalid arguments).  A
 * local layer's decode merges its splits on chip and needs no workspace: the
 * function returns 16 and the call accepts any workspace, null included. */
BEAM_API size_t beam_decode_workspace_bytes(int kind, const beam_attn_params *p, int32_t B,
                                   const beam_kv_layout_t *layout);

/* One decode step: each of B sequences adds one token at 0-based position
 * pos[b] (device int64 [B]; p = pos[b] + 1).
 *   q, gate : [B][48*128] bf16     k, v : [B][8*128] bf16 (raw projections)
 *   k_cache, v_cache : the layer's caches (layout on the host); the new key and
 *     value are written first (global slot t, local slot t mod window), then the
 *     query attends over keys max(0, t-window+1) .. t (local) or 0 .. t (global).
 *     Cached keys must already be normalised (and rotated, in a local ring) --
 *     exactly what this library writes.
 *   out : [B][48*128] bf16.
 * A global position t >= slots_per_seq, or t < 0, leaves that sequence's cache and
 * output untouched and sets BEAM_ERR_CAPACITY in dev_status. */
BEAM_API int beam_attn_decode(int kind, const beam_attn_params *p, int32_t B, const void *q, const void *k,
                     const void *v, const void *gate, const float *q_norm_w,
                     const float *k_norm_w, const float *gate_bias, const int64_t *pos,
                     void *k_cache, void *v_cache, const beam_kv_layout_t *layout, void *out,
                     void *workspace, size_t workspace_bytes, int32_t *dev_status,
                     beam_stream_t stream);

/* ---- FP8 E4M3 KV cache (section "KV memory": 18 KiB per token over the nine
 * global layers instead of 36 KiB in BF16).  Each element of an FP8 cache is one
 * E4M3 code (OCP FP8 E4M3: bias 7, no infinities, largest finite 448) of
 * value / scale, with one float scale per cache tensor of a layer (k_scale for
 * the keys, v_scale for the values; finite and > 0, else BEAM_ERR_INVALID_ARG).
 * Codes are the nearest, ties to even, saturating at +-448; keys are quantised
 * from their fp32 normalised (local: rotated) values, values from their raw
 * bf16 values.  A code reads back as E4M3^-1(code) * scale. */

/* Layout of an FP8 cache: the same head-major [B][8][slots][128] element order
 * and strides as beam_kv_layout, one byte per element (bytes_k, bytes_v
 * halved).  Rows must start on 16 bytes: strides multiples of 16 elements. */
BEAM_API int beam_kv_layout_fp8(int kind, const beam_attn_params *p, int32_t batch,
                                int64_t capacity_tokens, beam_kv_layout_t *out);

/* beam_kv_append into an FP8 cache (same positions, slots and capacity
 * behaviour). */
BEAM_API int beam_kv_append_fp8(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                                const void *k, const void *v, const float *k_norm_w,
                                const int64_t *pos0, void *k_cache, void *v_cache,
                                const beam_kv_layout_t *layout, float k_scale, float v_scale,
                                int32_t *dev_status, beam_stream_t stream);

/* beam_attn_decode over an FP8 cache: the new key and value are written as
 * codes, then the query attends over the cached codes read back as values (the
 * new token's too).  Workspace as for beam_attn_decode
 * (beam_decode_workspace_bytes with the FP8 layout). */
BEAM_API int beam_attn_decode_fp8(int kind, const beam_attn_params *p, int32_t B, const void *q,
                                  const void *k, const void *v, const void *gate,
                                  const float *q_norm_w, const float *k_norm_w,
                                  const float *gate_bias, const int64_t *pos, void *k_cache,
                                  void *v_cache, const beam_kv_layout_t *layout, float k_scale,
                                  float v_scale, void *out, void *workspace,
                                  size_t workspace_bytes, int32_t *dev_status,
                                  beam_stream_t stream);

/* Workspace beam_attn_prefill_chunk_fp8 needs (bytes): what
 * beam_prefill_chunk_workspace_bytes gives for the same shapes and, for a global
 * layer with T > 16, a bf16 view of the cache (keys and values, two bytes for every
 * element of the FP8 layout, 4 * bytes_k in all) at the end of the workspace. */
BEAM_API size_t beam_prefill_chunk_fp8_workspace_bytes(int kind, const beam_attn_params *p,
                                                       int32_t B, int32_t T,
                                                       const beam_kv_layout_t *layout);

/* beam_attn_prefill_chunk over FP8 E4M3 caches (layout from beam_kv_layout_fp8; one
 * scale per cache tensor as for beam_attn_decode_fp8).  The chunk's new keys and
 * values are written as codes first; the queries then attend over every visible key
 * and value read back from the cache, the new ones included (the order the FP8
 * decode takes for one new token).  The codes are read as their unscaled values
 * (exact), with k_scale folded into the score scale and v_scale into the output:
 * a local chunk widens the ring rows it sees to bf16 in the workspace, and a global
 * chunk of more than 16 tokens widens the rows before each sequence's pos0 into a
 * bf16 view of the cache, both then read by the tensor-core kernels of the bf16
 * path; a global chunk of at most 16 tokens reads the codes themselves (keys in
 * E4M3 MMAs against a two-term E4M3 split of each query row, values widened to f16
 * on chip).  Positions, status, capacity and the T <= 16 path as in
 * beam_attn_prefill_chunk. */
BEAM_API int beam_attn_prefill_chunk_fp8(int kind, const beam_attn_params *p, int32_t B, int32_t T,
                                         const void *q, const void *k, const void *v,
                                         const void *gate, const float *q_norm_w,
                                         const float *k_norm_w, const float *gate_bias,
                                         const int64_t *pos0, void *out, void *k_cache,
                                         void *v_cache, const beam_kv_layout_t *layout,
                                         float k_scale, float v_scale, void *workspace,
                                         size_t workspace_bytes, int32_t *dev_status,
                                         beam_stream_t stream);

/* Decode without any allocation, for callers that cannot call cudaMalloc.
 *
 * There is no counterpart in the paper: this is a deployment convenience.  Some
 * hosts hand a library only the buffers of its inputs and outputs and forbid
 * it any device allocation of its own -- for example a serving runtime that
 * pre-partitions all device memory into its own pools, or a latency-critical
 * loop in which an allocation (and the device synchronisation that cudaMalloc
 * and cudaFree can imply) is not acceptable -- yet beam_attn_decode needs a
 * workspace for the split-K partial results.
 *
 * This entry point computes exactly what beam_attn_decode computes, with the
 * same arguments minus the workspace.  Its scratch is a fixed array of
 * 8 MiB (8,388,608 bytes) of device memory inside the library, which every GPU
 * that loads the library holds until the process exits.  A global-layer call
 * whose beam_decode_workspace_bytes() would exceed 8 MiB returns
 * BEAM_ERR_SCRATCH_LIMIT before any launch (roughly: B * 8 * splits * 3.1 KB;
 * B = 64 at a 32K-slot cache or B = 1 at a 1M-slot cache fit).  A local-layer
 * call uses no scratch and takes any batch.
 *
 * The first call on each device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture.  The library caches per-device state (this address, the kernels'
 * shared-memory opt-ins) for the life of the process: after cudaDeviceReset
 * of a device, do not call the library on that device again in the same
 * process.  All calls share the one array and it keeps whatever the last call
 * left in it; nothing in it needs to start at zero, because every value read
 * is written earlier in the same call.  Calls whose kernels overlap on the GPU
 * (on different streams, or from several threads) race on the array: issue
 * them on one stream, one after the other.  The call allocates nothing and
 * calls no allocating routine. */
BEAM_API int beam_attn_decode_noalloc(int kind, const beam_attn_params *p, int32_t B,
                                      const void *q, const void *k, const void *v,
                                      const void *gate, const float *q_norm_w,
                                      const float *k_norm_w, const float *gate_bias,
                                      const int64_t *pos, void *k_cache, void *v_cache,
                                      const beam_kv_layout_t *layout, void *out,
                                      int32_t *dev_status, beam_stream_t stream);

/* Static description of a status code. */
BEAM_API const char *beam_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* BEAM_ATTN_H */
