/*
 * wushkv.h -- C ABI of libwushkv: the WUSH-KV append + decode-attention hot path
 * on NVIDIA B200 (sm_100a).
 *
 * The method ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms"):
 *   - append (§4.1, §4.2, §4.4, §5.3): every new post-RoPE key k of KV head h is
 *     transformed, k' = T_K k (T_K a full invertible 128x128 matrix fixed at
 *     calibration); the value v arrives already in its transformed basis (the value
 *     transform is folded into the weights, §4.5) and is stored as given.  The first
 *     s_sink positions and the newest s_keep positions stay fp16; the rest is
 *     quantized per token with a percentile-clipped asymmetric affine quantizer to
 *     2 or 4 bits, in batches of s_flush positions (Algorithm 2 prose, §4.4).
 *   - decode attention (§4.1, §4.2): each query is compensated, q' = T_K^{-T} q, so
 *     q'.k' = q.k; keys and values are dequantized on the fly and the fp16 sink and
 *     recent windows are merged in one exact softmax over all S cached positions.
 *     The output stays in the value-transform basis (the output projection undoes it).
 *
 * Conventions shared by every entry point:
 *   - head_dim d must be 128; bits must be 2 or 4; n_q_heads / n_kv_heads = g must
 *     be 1, 2, 4 or 8; query head j reads KV head j / g.
 *   - fp16 means IEEE binary16 stored as uint16; half2 means two fp16 in 4 bytes,
 *     the first (lower address) element in the low half.
 *   - All device buffers are allocated and owned by the caller (sizes from
 *     wushkv_pack_layout), must be 16-byte aligned, and stay valid until the work
 *     queued on `stream` has finished.  The library allocates nothing; its only
 *     global state is the fixed scratch array of wushkv_decode_attn_static.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *   - Calls are asynchronous: a zero return means the work was validated and
 *     queued.  Conditions only the device can see (capacity overflow, decode of an
 *     empty sequence, a bounded wait that gave up) are OR-ed into the cache's
 *     status word (below); nothing traps.
 *   - Inputs must be finite (no NaN/Inf).
 *
 * Return codes: WUSHKV_OK, or a negative WUSHKV_E* value; on error nothing is queued
 * and no buffer is touched.
 */
#ifndef WUSHKV_H
#define WUSHKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WUSHKV_OK 0
#define WUSHKV_EINVAL (-1)       /* null/misaligned pointer, bad window or percentile values */
#define WUSHKV_EUNSUPPORTED (-2) /* head_dim != 128, bits not 2/4, g not 1/2/4/8, percentiles
                                    needing more than the 4 extreme order statistics */
#define WUSHKV_ECUDA (-3)        /* a CUDA launch or query failed */
#define WUSHKV_ESINGULAR (-4)    /* wushkv_compensation: T_K is singular */
#define WUSHKV_ESCRATCH (-5)     /* wushkv_decode_attn_static: the configuration needs more scratch
                                    than WUSHKV_STATIC_SCRATCH_BYTES */

/* Size of the library-owned device scratch array behind wushkv_decode_attn_static. */
#define WUSHKV_STATIC_SCRATCH_BYTES (8u << 20)

/* Bits of the device status word (state buffer, int32 index 2*batch*n_kv_heads). */
#define WUSHKV_STATUS_OVERFLOW 1u /* an append would exceed `capacity`: that sequence was skipped */
#define WUSHKV_STATUS_EMPTY 2u    /* decode of a sequence with S == 0: its output rows are zero */
#define WUSHKV_STATUS_TIMEOUT 4u  /* a bounded in-kernel wait gave up (a library bug, not an input error) */
#define WUSHKV_STATUS_BADSTATE 8u /* a state entry was out of range (S < 0, S > capacity, S_quant outside
                                     [0, S]): that (sequence, KV head) was skipped / read as empty */
#define WUSHKV_STATUS_CHUNK_QUANTIZED 16u /* wushkv_chunk_attn on a cache whose newest n_q positions are
                                             not all fp16 (e.g. after a bulk append): quantized
                                             positions were visible to every chunk query */

/* Cache configuration; one cache holds one attention layer. */
typedef struct wushkv_config {
  int32_t batch;       /* B, sequences */
  int32_t n_kv_heads;  /* H_kv */
  int32_t n_q_heads;   /* H_q, a multiple of H_kv with H_q / H_kv in {1, 2, 4, 8} */
  int32_t head_dim;    /* d, must be 128 */
  int32_t bits;        /* 2 or 4 */
  int32_t capacity;    /* positions per sequence, >= 1 */
  int32_t s_sink;      /* S_sink >= 0: first positions kept fp16 for good */
  int32_t s_keep;      /* S_keep >= 0: newest positions kept fp16 */
  int32_t s_flush;     /* S_flush >= 1: quantization batch */
  int32_t chunk_max;   /* >= 1: appends of at most chunk_max tokens stay fp16 until the next
                          append (the pages' order: append, attend, then quantize); larger
                          appends are quantized on arrival */
  float p_lo;          /* clipping percentiles, 0 <= p_lo < p_hi <= 100; the needed order */
  float p_hi;          /* statistics must lie within 4 of either end (e.g. 1/99, 0.5/99.5) */
  int32_t transform;   /* key transform: WUSHKV_TRANSFORM_DENSE (0) reads T_K from the t_k
                          argument; WUSHKV_TRANSFORM_HADAMARD (1) applies the normalised
                          Walsh-Hadamard matrix H (H[r][i] = (-1)^popcount(r & i) / sqrt(128))
                          computed in the kernels, t_k unused (may be NULL) */
  int32_t quantizer;   /* WUSHKV_QUANT_PERCENTILE (0): percentile-clipped affine (p_lo, p_hi);
                          WUSHKV_QUANT_RMS (1): QuEST-style symmetric grid scaled by each
                          token's RMS, clipped at +-clip_alpha * RMS (p_lo, p_hi unused) */
  float clip_alpha;    /* WUSHKV_QUANT_RMS: clipping endpoint in RMS units, > 0 (the
                          Gaussian-optimal value for the bit width, e.g. 1.4936 at 2 bits) */
} wushkv_config;

#define WUSHKV_TRANSFORM_DENSE 0
#define WUSHKV_TRANSFORM_HADAMARD 1
#define WUSHKV_QUANT_PERCENTILE 0
/* WUSHKV_QUANT_RMS: per token sigma = sqrt(sum(x^2) / 128) in fp32, the squares summed in
 * four runs of 32 consecutive elements, then (g0 + g1) + (g2 + g3); s = fp16(fp32(2*alpha /
 * (2^b - 1)) * sigma), z = fp16(-fp32(alpha) * sigma); codes and storage as the affine
 * quantizer's (the decode is unchanged). */
#define WUSHKV_QUANT_RMS 1

/* Code orders of wushkv_layout.code_order.
 *  WUSHKV_CODE_ORDER_CANONICAL (0): every position's record holds code j (0..127) in byte
 *    (j*bits)/8 at bit offset (j*bits)%8, record p at byte offset p * code_bytes (K and V).
 *  WUSHKV_CODE_ORDER_VGROUP16 (1): k_codes canonical; v_codes in the 16-position group
 *    layout that wushkv_cache describes (the layout this library writes and reads). */
#define WUSHKV_CODE_ORDER_CANONICAL 0
#define WUSHKV_CODE_ORDER_VGROUP16 1

/* Byte sizes of the caller-allocated buffers (wushkv_pack_layout). */
typedef struct wushkv_layout {
  size_t codes_bytes;     /* each of k_codes, v_codes: uint8 [B][H_kv][cap_alloc][code_bytes] */
  size_t params_bytes;    /* each of k_params, v_params: half2 (s, z) [B][H_kv][cap_alloc] */
  size_t sink_bytes;      /* each of k_sink, v_sink: fp16 [B][H_kv][max(s_sink,1)][128] */
  size_t ring_bytes;      /* each of k_ring, v_ring: fp16 [B][H_kv][ring_slots][128] */
  size_t state_bytes;     /* int32 [B*H_kv][2] = (S, S_quant) per (sequence, KV head), then the
                             status word; zero it to start from an empty cache */
  size_t workspace_bytes; /* wushkv_decode_attn scratch; zero-fill it once before its first use */
  int32_t cap_alloc;      /* capacity rounded up to a multiple of 128 */
  int32_t ring_slots;     /* s_keep + s_flush - 1 + chunk_max; position p lives in slot p % ring_slots */
  int32_t code_bytes;     /* 128 * bits / 8 bytes of packed codes per token and head */
  int32_t n_splits;       /* decode work items per (sequence, KV head) over the quantized region */
  int32_t split_tokens;   /* most positions one decode work item streams (at full capacity; the
                             kernel splits each sequence's current length evenly among the
                             n_splits items, in whole multiples of 128) */
  int32_t code_order;     /* how the packed codes are ordered (WUSHKV_CODE_ORDER_*) */
  size_t chunk_workspace_bytes; /* wushkv_chunk_attn scratch (zero-fill it once before its first use) */
  int32_t decode_cluster; /* decode CTAs per thread-block cluster (1 or 2; divides n_splits) */
  int32_t decode_interleave; /* 1: the decode grid interleaves the units (n_splits >= 37) */
} wushkv_layout;

/* Device pointers of one layer's cache.
 *  codes: the packed record of position p (code_bytes bytes) holds code j (0..127) in byte
 *         (j*bits)/8 at bit offset (j*bits)%8 (little-endian within the byte); only
 *         S_sink <= p < S_quant are meaningful.
 *         k_codes: record p at byte offset p * code_bytes of the unit's array.
 *         v_codes: in groups of 16 positions (group p / 16 at byte offset (p & ~15) *
 *         code_bytes), laid out for the decode's PV operand: the 16-bit chunk c of record
 *         p (bytes 2c, 2c+1; c < 8*bits) is 16-bit half 2*w + (r >> 3) of the group,
 *         r = p % 16, t = r & 7, w = 16*(c>>1) + 4*(t&3) + 2*(c&1) + (t>>2) at 2 bits,
 *         w = 128*((c>>1)&1) + 16*(c>>2) + 4*(t&3) + 2*(c&1) + (t>>2) at 4 bits.
 *  params: (s, z) of position p; the token's values dequantize to z + s * code.
 *  sink:  k' / v of positions p < s_sink at index p.
 *  ring:  k' / v of fp16 positions p >= max(S_quant, s_sink) at slot p % ring_slots.
 *  k' (keys in the transformed basis) is what every key buffer holds. */
typedef struct wushkv_cache {
  void* k_codes;
  void* v_codes;
  void* k_params;
  void* v_params;
  void* k_sink;
  void* v_sink;
  void* k_ring;
  void* v_ring;
  int32_t* state;
} wushkv_cache;

/* Validate `cfg` and fill `out` with the buffer sizes the caller must allocate.
 * Host only; touches no device.  Returns WUSHKV_OK, WUSHKV_EINVAL or WUSHKV_EUNSUPPORTED. */
int wushkv_pack_layout(const wushkv_config* cfg, wushkv_layout* out);

/* One-time calibration helper (host only): the compensation matrix for the query side.
 * t_k:   host fp16 [n_kv_heads][128][128], T_K row-major acting on column vectors
 *        (k'[r] = sum_i T_K[r][i] k[i]).
 * t_k_inv: host fp32 [n_kv_heads][128][128] output, T_K^{-1} row-major, computed in double
 *        precision by Gauss-Jordan elimination with partial pivoting, then rounded.
 * The query compensation of §4.2, q' = T_K^{-T} q, reads it as q'[j] = sum_i t_k_inv[i][j] q[i].
 * Returns WUSHKV_OK, WUSHKV_EINVAL or WUSHKV_ESINGULAR. */
int wushkv_compensation(const uint16_t* t_k, int32_t n_kv_heads, float* t_k_inv);

/* The compensation matrix of WUSHKV_TRANSFORM_HADAMARD (host only): H is orthonormal and
 * symmetric, so T_K^{-1} = H; fills t_k_inv (fp32 [n_kv_heads][128][128]) with H rounded
 * to fp32.  The structured transform is the pages' Hadamard baseline and their
 * "cheaper structured transforms" direction.  Returns WUSHKV_OK or WUSHKV_EINVAL. */
int wushkv_hadamard(int32_t n_kv_heads, float* t_k_inv);

/* Calibration statistics (offline, before T_K is built): accumulate the per-head Gram
 * matrices of a batch of cached vectors ("WUSH-KV: KV Cache Quantization with
 * Data-Adaptive Transforms": §3, the transform is built from the Gram matrix M of the
 * quantized tensor; Appendix B.1, M = X X^T with one quantization group, here one token,
 * per column; §5.2 Setup, a calibration pass accumulates key Gram matrices after RMS
 * normalisation and RoPE, and value Gram matrices, per KV head).
 * x:     device fp16 [n_tokens][n_heads][128], 16-byte aligned: keys after head-norm and
 *        RoPE (before T_K), or values.  [B][n][H_kv][128] is the same array with
 *        n_tokens = B * n.
 * gram:  device fp64 [n_heads][128][128] row-major, 16-byte aligned, accumulated in place:
 *        gram[h] += sum_t x[t][h] x[t][h]^T.  Zero it before the first batch.
 * Precision: a block of at most 4096 tokens of one head is summed on the tensor cores
 * (exact fp16 products, fp32 sums), then added into gram with fp64 atomics.  The order of
 * those fp64 additions is not fixed, so the last bits can differ between calls.
 * n_tokens == 0 queues nothing (x may then be null).  The two buffers must not overlap.
 * Returns WUSHKV_OK, WUSHKV_EINVAL (null or misaligned pointer, n_tokens < 0, n_heads
 * outside [1, 65535], n_tokens * n_heads > 2^40) or WUSHKV_ECUDA. */
int wushkv_gram_accumulate(const void* x, int64_t n_tokens, int32_t n_heads, double* gram, void* stream);

/* Append n_new >= 0 tokens to every sequence (§4.1, §4.2, §4.4 "Full-Precision Cache
 * Window", §5.3 quantizer).
 * k_new, v_new: device fp16 [B][n_new][H_kv][128]; keys after head-norm and RoPE,
 *               values already in the value-transform basis.
 * t_k:          device fp16 [H_kv][128][128], T_K row-major; k' = fp16_rn(T_K k), fp32 accumulation.
 * Steps, per (sequence, KV head) with state (S, S_quant):
 *   if S + n_new > capacity: set WUSHKV_STATUS_OVERFLOW, leave the sequence unchanged;
 *   n_new <= chunk_max: flush under length S (closes the previous chunk), then store the
 *                       n_new tokens fp16 (sink or ring), S += n_new;
 *   n_new >  chunk_max: store, S += n_new, flush under the new S (tokens that the flush
 *                       covers are quantized straight from registers).
 *   flush under L: lo0 = max(S_quant, s_sink); e = L - s_keep - lo0; if e >= s_flush,
 *                  quantize positions [lo0, lo0 + floor(e/s_flush)*s_flush) and move S_quant.
 *   quantize one token's 128 values x (fp16): sort; lo/hi = the p_lo/p_hi percentiles,
 *     linear interpolation at rank p/100*127 in fp32 (s[i] + f*(s[i+1]-s[i]), each op
 *     rounded); s = fp16_rn((hi - lo)/(2^bits - 1)), z = fp16_rn(lo);
 *     code = clamp(round_half_even(fp32(x - z) / s), 0, 2^bits - 1), code = 0 when s == 0.
 * Returns WUSHKV_OK, WUSHKV_EINVAL, WUSHKV_EUNSUPPORTED or WUSHKV_ECUDA. */
int wushkv_append(const wushkv_config* cfg, const wushkv_cache* cache, const void* k_new,
                  const void* v_new, int32_t n_new, const void* t_k, void* stream);

/* Decode attention of one query per sequence over the whole cache (§4.1, §4.2, §4.4).
 * q:        device fp16 [B][H_q][128], after head-norm and RoPE.
 * t_k_inv:  device fp32 [H_kv][128][128], T_K^{-1} row-major (see wushkv_compensation).
 * softmax_scale: logits are softmax_scale * q.k (1/sqrt(128) for standard attention).
 * out_fp16: 0 -> out is fp32 [B][H_q][128]; 1 -> fp16.
 * workspace: device scratch of layout.workspace_bytes.  Zero-fill it once before its first
 *   use (cudaMemset): it holds the completion counters of the decode's last merge, which
 *   every call leaves at zero again -- also a call that gave up on a wait.  Calls that
 *   share one workspace must not overlap in time.
 * out[b][j] = sum_p softmax_p(softmax_scale * q'_j . khat_p) vhat_p over p < S, with
 *   q'_j = T_K^{-T} q_j, khat_p / vhat_p the stored fp16 k'/v in the windows and
 *   z + s*code in the quantized region.  S == 0 gives zeros and WUSHKV_STATUS_EMPTY.
 * Returns WUSHKV_OK, WUSHKV_EINVAL, WUSHKV_EUNSUPPORTED or WUSHKV_ECUDA. */
int wushkv_decode_attn(const wushkv_config* cfg, const wushkv_cache* cache, const void* q,
                       const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out,
                       void* workspace, void* stream);

/* One decode step: wushkv_append(k_new, v_new, n_new) followed by wushkv_decode_attn(q) on
 * the same stream, with the same arguments, buffers and results as those two calls
 * (§4.4: the new tokens are appended in full precision and serve the step's attention).
 * With n_new <= chunk_max the append also prepares the decode (the compensated queries,
 * their tensor-core fragments and the workspace's counters) and the decode kernel is
 * launched as its programmatic dependent, so the step costs two kernel launches instead of
 * three; the decode kernel then reads the quantized positions the append cannot touch while
 * the append runs, and it is the decode kernel that advances the state words, at its end
 * (the cache is in the same state as after the two separate calls once the step has
 * completed in stream order).  The decode of a
 * sequence whose append is refused (STATUS_OVERFLOW) attends over its cache unchanged.
 * Returns WUSHKV_OK, WUSHKV_EINVAL, WUSHKV_EUNSUPPORTED or WUSHKV_ECUDA. */
int wushkv_step(const wushkv_config* cfg, const wushkv_cache* cache, const void* k_new, const void* v_new,
                int32_t n_new, const void* t_k, const void* q, const float* t_k_inv, float softmax_scale,
                int32_t out_fp16, void* out, void* workspace, void* stream);

/* Chunked prefill attention (the pages' order, §4.4: a new chunk is appended in full
 * precision and computes its own attention before it is quantized): the n_q newest
 * positions of every sequence (the chunk just appended with n_q <= chunk_max, so all of it
 * is in the fp16 window) attend, each causally, over the cache: query t (position
 * S - n_q + t) sees positions 0 .. S - n_q + t.
 * q:   device fp16 [B][n_q][H_q][128] (after head-norm and RoPE); out: [B][n_q][H_q][128],
 *      fp32 or fp16 (out_fp16); t_k_inv, softmax_scale as in wushkv_decode_attn.
 * workspace: layout.chunk_workspace_bytes, zero-filled once before its first use (as for
 *   wushkv_decode_attn; one buffer of the larger size may serve both, and wushkv_step:
 *   every layout of a configuration keeps its completion counters in the same leading
 *   bytes, which every call leaves at zero).
 * The chunk's queries take blocks of up to 8 / g tokens (their query heads share the
 * kernel's per-position work); one launch pair runs up to 32 equal blocks side by side, as
 * separate grid rows of each (sequence, KV head) that stream its cache at the same time.
 * Returns WUSHKV_OK, WUSHKV_EINVAL (also n_q < 1 or n_q > chunk_max), WUSHKV_EUNSUPPORTED
 * or WUSHKV_ECUDA. */
int wushkv_chunk_attn(const wushkv_config* cfg, const wushkv_cache* cache, const void* q, int32_t n_q,
                      const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out, void* workspace,
                      void* stream);

/* The step before the path, for wushkv_step_prep: the queries and keys arrive as raw
 * projections and the library applies, per head, the RMSNorm (where the model has one,
 * as Qwen3 does) and the rotary position embedding that the path's inputs have undergone
 * (§4.1: keys are cached after head-wise normalisation and RoPE).
 *   RMSNorm: y = x / sqrt(mean(x^2) + norm_eps) * gain over the 128 head dimensions;
 *   RoPE: rotate-half pairing, dimension i < 64 with i + 64, angle pos * theta^(-i/64);
 *   each result rounded once to fp16.  Key t of an n_new-token append sits at position
 *   S + t (S = the sequence's length before the append); the query at the newest
 *   position, S + n_new - 1. */
typedef struct wushkv_prep {
  float rope_theta;        /* RoPE base, > 1 */
  const void* q_norm_gain; /* device fp16 [128] RMSNorm gain of every query head, or NULL: no query norm */
  const void* k_norm_gain; /* device fp16 [128] RMSNorm gain of every key head, or NULL: no key norm */
  float norm_eps;          /* RMSNorm epsilon, > 0 when a gain is given */
} wushkv_prep;

/* wushkv_step on raw q / k: k_raw and q_raw are the projections before the per-head
 * RMSNorm and RoPE that `prep` describes; v_new and every other argument as in
 * wushkv_step.  The normalisation and rotation run inside the step's kernels (the
 * append's key path and the decode's query preparation).  Returns WUSHKV_OK,
 * WUSHKV_EINVAL (also: prep NULL, theta <= 1, a gain without eps > 0),
 * WUSHKV_EUNSUPPORTED or WUSHKV_ECUDA. */
int wushkv_step_prep(const wushkv_config* cfg, const wushkv_cache* cache, const void* k_raw, const void* v_new,
                     int32_t n_new, const void* t_k, const void* q_raw, const float* t_k_inv, float softmax_scale,
                     int32_t out_fp16, void* out, void* workspace, const wushkv_prep* prep, void* stream);

/* Test hook for the bounded waits (not a production entry point; no counterpart in the
 * method): wushkv_decode_attn with the in-kernel wait limit shortened to wait_limit_cycles
 * (1000 .. the default of about 2 s of SM clock) and, when withhold_stage >= 0, stage
 * withhold_stage of every work item's pipeline never issued, so that its consumers give up.
 * Nothing faults or traps: a wait that gives up sets WUSHKV_STATUS_TIMEOUT, every warp of the
 * work item leaves its loop, the copies already issued land, the tensor memory is released,
 * and the item writes no partial result -- the output rows of an affected unit are not
 * written (they keep whatever the buffer held).  The cache and the workspace are left usable
 * for the next call.  Returns as wushkv_decode_attn, or WUSHKV_EINVAL for an out-of-range
 * hook argument. */
int wushkv_decode_attn_test_timeout(const wushkv_config* cfg, const wushkv_cache* cache, const void* q,
                                    const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out,
                                    void* workspace, int32_t withhold_stage, int64_t wait_limit_cycles,
                                    void* stream);

/* wushkv_decode_attn with library-owned scratch instead of a caller-allocated workspace.
 * The method has no counterpart of this call: it serves callers that cannot allocate
 * device memory when they decode (a runtime without an allocator, a step that must not
 * enter a caching allocator, a host program that owns every buffer it hands over).
 * Arguments, layouts, results and return codes are those of wushkv_decode_attn, minus
 * `workspace`; it allocates nothing.
 * Scratch: a file-scope device array of WUSHKV_STATIC_SCRATCH_BYTES that every GPU
 *   loading the library holds until the process exits.  A configuration whose
 *   layout.workspace_bytes exceeds it returns WUSHKV_ESCRATCH and queues nothing.
 * Set-up: every call looks up the array's device address in the current CUDA context
 *   (cudaGetSymbolAddress, a host-side query).  The first call in a context may load the
 *   library's device module: make it before any stream capture in that context.
 * Sharing: all calls in a context share the one array.  It starts zero-filled (a device
 *   array of the module) and every call leaves the merge's completion counters in it at
 *   zero again; every other byte is written before it is read.  Calls whose work overlaps
 *   in time (different streams, or threads without ordering) race on the array: serialise
 *   them. */
int wushkv_decode_attn_static(const wushkv_config* cfg, const wushkv_cache* cache, const void* q,
                              const float* t_k_inv, float softmax_scale, int32_t out_fp16, void* out,
                              void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WUSHKV_H */
