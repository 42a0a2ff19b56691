/*
 * mimo_attn.h — C ABI of the MiMo-V2-Flash hybrid attention layer for
 * NVIDIA B200 (sm_100a).
 *
 * One layer of the decoder's attention, as the pages describe it:
 *   - "Add Xiaomi MiMo-V2" (huggingface/transformers pull request 45144),
 *     section "Additional useful info": partial RoPE over the leading third
 *     of the QK head dim; a RoPE base that differs between sliding-window
 *     (SWA) and global (GA) layers; a KV-head count that differs between
 *     them (GQA); a V head dim decoupled from the QK head dim; V rescaled by
 *     sqrt(hidden_size / (num_attention_heads * v_head_dim)); a gpt-oss-style
 *     attention sink on SWA layers only.
 *   - "feat(models): add Xiaomi MiMo v2 (mimo_v2_flash) text model support"
 *     (lablup/mlxcel issue 842), section "Architecture, verified against
 *     upstream": hybrid_layer_pattern[idx] == 1 selects a sliding layer with
 *     a window of sliding_window_size; the RoPE base is swa_rope_theta on
 *     sliding layers and rope_theta otherwise; the rotated width is
 *     int(partial_rotary_factor * head_dim). Section "Implementation plan":
 *     sliding layers keep a rotating (ring) KV cache.
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense, row-major, in device memory (cudaMalloc or torch),
 *     in the element type given by `dtype` unless stated otherwise. The
 *     caller owns every buffer; the library never allocates device memory
 *     on these calls and keeps no pointer after a call returns.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream) and never synchronises.
 *   - Arguments are checked on the host before any launch. A bad argument
 *     returns a non-zero status and launches nothing. A failed launch
 *     returns MIMO_ATTN_ERR_CUDA. Conditions only the device can see
 *     (kv_lens out of range, a pipeline wait that timed out) set the
 *     device error word read by mimo_attn_get_device_error(); nothing traps.
 *   - Base pointers of bf16 tensors must be 16-byte aligned (TMA rule).
 */
#ifndef MIMO_ATTN_H
#define MIMO_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MIMO_ATTN_API __attribute__((visibility("default")))
#else
#define MIMO_ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MIMO_ATTN_OK = 0,
    MIMO_ATTN_ERR_INVALID_ARG = 1,  /* shape, pointer or value check failed */
    MIMO_ATTN_ERR_UNSUPPORTED = 2,  /* valid, but no kernel handles it (e.g. dims > 256) */
    MIMO_ATTN_ERR_WORKSPACE = 3,    /* workspace missing or smaller than the size query says */
    MIMO_ATTN_ERR_CUDA = 4          /* a CUDA runtime call or launch failed */
} mimo_attn_status;

/* Layer kind = the layer's hybrid_layer_pattern entry (lablup/mlxcel issue
 * 842, "Architecture, verified against upstream"). */
typedef enum { MIMO_ATTN_GLOBAL = 0, MIMO_ATTN_SWA = 1 } mimo_attn_layer_type;

/* Element type of q, k, v, out and the caches. */
typedef enum { MIMO_ATTN_BF16 = 0, MIMO_ATTN_FP32 = 1 } mimo_attn_dtype;

/* Per-layer parameters (host struct; read during the call only). */
typedef struct {
    int32_t layer_type;    /* mimo_attn_layer_type */
    int32_t num_q_heads;   /* Hq */
    int32_t num_kv_heads;  /* Hkv; Hq % Hkv == 0; query head h reads KV head h / (Hq/Hkv) */
    int32_t qk_dim;        /* Dqk, even, <= 256 */
    int32_t v_dim;         /* Dv, <= 256 (decoupled from Dqk, PR 45144) */
    int32_t rotary_dim;    /* r = int(partial_rotary_factor * qk_dim); even, 0 <= r <= Dqk */
    int32_t window;        /* SWA: keys visible to query i are i-window+1 .. i; ignored for GLOBAL */
    int32_t hidden_size;   /* V scale = sqrt(hidden_size / (Hq * Dv)); must be > 0 */
    double rope_theta;     /* base of this layer: swa_rope_theta (SWA) or rope_theta (GLOBAL); > 0 */
    float softmax_scale;   /* 0 selects 1/sqrt(Dqk) */
    const float *sinks;    /* device [Hq] fp32 sink logits, one per query head; SWA only
                              (must be NULL for GLOBAL, PR 45144); NULL = no sink */
} mimo_attn_layer;

/* Rotated width helper: int(partial_rotary_factor * qk_dim), the rule of
 * lablup/mlxcel issue 842 ("Architecture, verified against upstream"); the
 * factor is taken as a double because upstream types it as an int but uses
 * it as a multiplier. Returns -1 for a negative or non-finite product. */
MIMO_ATTN_API int mimo_attn_rotary_dim(double partial_rotary_factor, int qk_dim);

/* Bytes of workspace mimo_attn_prefill needs for this layer and shape
 * (the rotated keys when they are not written into a global cache). The
 * value does not depend on whether caches are passed; 0 means none. */
MIMO_ATTN_API size_t mimo_attn_prefill_workspace_size(const mimo_attn_layer *layer, int dtype,
                                        int batch, int seq);

/* Prefill: one layer's attention over a whole prompt.
 *   q   [batch, seq, Hq,  Dqk]  unrotated queries
 *   k   [batch, seq, Hkv, Dqk]  unrotated keys
 *   v   [batch, seq, Hkv, Dv]
 *   positions: device int32 [seq] RoPE positions, or NULL for 0..seq-1.
 *              Masking always uses the sequence index (causal, window).
 *   out [batch, seq, Hq, Dv]    out[b,i,h] = Vscale * sum_j p_ij v_j, with
 *              p the softmax over the visible keys j (GLOBAL: j <= i; SWA:
 *              i-window < j <= i) plus, on SWA with sinks, the sink term
 *              exp(sink[h]) in the denominator only.
 *   k_cache, v_cache: optional (both NULL or both set). GLOBAL: linear caches
 *              [batch, cache_capacity, Hkv, D] with cache_capacity >= seq;
 *              slots 0..seq-1 receive the rotated keys and the values.
 *              SWA: ring caches [batch, window, Hkv, D], cache_capacity ==
 *              window; token i (for i >= seq - window) lands in slot
 *              i mod window.
 *   workspace: device buffer of at least mimo_attn_prefill_workspace_size()
 *              bytes (may be NULL when that size is 0), 256-byte aligned.
 * Errors: MIMO_ATTN_ERR_INVALID_ARG for null required pointers, batch or
 * seq < 0, Hq % Hkv != 0, odd or out-of-range rotary_dim, window < 1 on SWA,
 * sinks on GLOBAL, a cache capacity that breaks the rules above, theta <= 0,
 * misaligned bf16 pointers; MIMO_ATTN_ERR_UNSUPPORTED for dims > 256;
 * MIMO_ATTN_ERR_WORKSPACE for a short workspace. batch == 0 or seq == 0 is
 * a no-op returning MIMO_ATTN_OK. */
MIMO_ATTN_API mimo_attn_status mimo_attn_prefill(const mimo_attn_layer *layer, int dtype, int batch, int seq,
                                   const void *q, const void *k, const void *v,
                                   const int32_t *positions, void *out,
                                   void *k_cache, void *v_cache, int cache_capacity,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace mimo_attn_prefill_cached needs: the RoPE table of
 * positions 0 .. max_past_len + seq - 1 and, on SWA, the per-sequence key and
 * value windows [batch, round_up(window - 1, 16) + seq, Hkv, D]. 0 on a bad
 * layer or negative sizes. */
MIMO_ATTN_API size_t mimo_attn_prefill_cached_workspace_size(const mimo_attn_layer *layer, int dtype,
                                                             int batch, int seq, int max_past_len);

/* Prefill continuing a cache (chunked prefill): a chunk of seq new tokens per
 * sequence after past_lens[b] tokens that are already in the caches. This is
 * the cache-aware prefill of the rotating cache (lablup/mlxcel issue 842,
 * "Implementation plan"; the attention itself as in mimo_attn_prefill).
 *   q [batch, seq, Hq, Dqk], k [batch, seq, Hkv, Dqk], v [batch, seq, Hkv, Dv]:
 *              the chunk, unrotated; token t of sequence b has position
 *              past_lens[b] + t (RoPE and mask).
 *   past_lens: device int32 [batch], 0 <= past_lens[b] <= max_past_len.
 *   max_past_len: host bound of past_lens (sizes the RoPE table).
 *   out [batch, seq, Hq, Dv]: token t attends every cached key and the
 *              chunk's keys up to itself (GLOBAL: positions <= its own; SWA:
 *              the last `window` positions including its own), sink on SWA.
 *   k_cache, v_cache (required; hold rotated keys, as decode and prefill
 *              leave them): GLOBAL linear [batch, cache_capacity, Hkv, D]
 *              with cache_capacity >= max_past_len + seq, position p in slot
 *              p; SWA ring [batch, window, Hkv, D], cache_capacity == window,
 *              position p in slot p mod window. On return the chunk's rotated
 *              keys and values are in their slots (on SWA the chunk's last
 *              `window` tokens).
 *   workspace: at least mimo_attn_prefill_cached_workspace_size() bytes,
 *              256-byte aligned.
 * Errors: as mimo_attn_prefill, plus MIMO_ATTN_ERR_INVALID_ARG for null
 * past_lens or caches, max_past_len < 0 or a cache capacity that breaks the
 * rules above. past_lens[b] outside [0, max_past_len] (or, on GLOBAL, beyond
 * the capacity) is caught on the device: MIMO_ATTN_DEVERR_KV_LEN is set in the
 * device error word and that sequence's cache rows are not written (its
 * outputs are undefined). */
MIMO_ATTN_API mimo_attn_status mimo_attn_prefill_cached(const mimo_attn_layer *layer, int dtype, int batch,
                                                        int seq, const void *q, const void *k, const void *v,
                                                        const int32_t *past_lens, int max_past_len, void *out,
                                                        void *k_cache, void *v_cache, int cache_capacity,
                                                        void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace mimo_attn_decode needs (split-KV partial results) for
 * this layer, batch and cache capacity. */
MIMO_ATTN_API size_t mimo_attn_decode_workspace_size(const mimo_attn_layer *layer, int dtype, int batch,
                                       int cache_capacity);

/* Decode: one new token per sequence, attending to its cache.
 *   q     [batch, Hq, Dqk], k_new [batch, Hkv, Dqk], v_new [batch, Hkv, Dv], unrotated.
 *   kv_lens: device int32 [batch]; L_b counts the new token (L_b >= 1), so the
 *          new token's position is L_b - 1. GLOBAL needs L_b <= cache_capacity.
 *   k_cache, v_cache (required, updated in place):
 *          GLOBAL: linear [batch, cache_capacity, Hkv, D]; slot p holds the
 *          rotated key / value of position p (p < L_b - 1 already filled).
 *          SWA: ring [batch, window, Hkv, D] with cache_capacity == window;
 *          slot p mod window holds position p.
 *          The call writes the new token's rotated key and value into slot
 *          L_b - 1 (GLOBAL) or (L_b - 1) mod window (SWA).
 *   out   [batch, Hq, Dv]: attention of the new token over positions
 *          0..L_b-1 (GLOBAL) or max(0, L_b-window)..L_b-1 (SWA), with the
 *          sink and V scale as in mimo_attn_prefill.
 *   workspace: at least mimo_attn_decode_workspace_size() bytes, 256-byte aligned.
 * A kv_lens entry out of range sets MIMO_ATTN_DEVERR_KV_LEN in the device
 * error word and leaves that sequence's output and cache untouched. */
MIMO_ATTN_API mimo_attn_status mimo_attn_decode(const mimo_attn_layer *layer, int dtype, int batch,
                                  const void *q, const void *k_new, const void *v_new,
                                  const int32_t *kv_lens, void *k_cache, void *v_cache,
                                  int cache_capacity, void *out, void *workspace,
                                  size_t workspace_bytes, void *stream);

/* Decode without any allocation: the same computation, arguments and
 * errors as mimo_attn_decode, but the split-KV partial results live in a
 * 16 MiB scratch array built into the library instead of a caller
 * workspace. For callers that cannot allocate device memory at all (a host
 * program whose memory pool owns the whole device, a plugin with no
 * allocator of its own, a loop that must not pay cudaMalloc's
 * synchronisation). The pages have no counterpart: this is an interface
 * convenience of this library, not a step of the layer.
 *   - Limit: mimo_attn_decode_workspace_size(layer, dtype, batch,
 *     cache_capacity) must be at most 16 MiB (16777216 bytes), else the call
 *     returns MIMO_ATTN_ERR_WORKSPACE and launches nothing. (Example: 64
 *     query heads, cache 32768, up to 31 sequences per call.)
 *   - The 16 MiB are reserved on a device when the library's device code
 *     first loads there (its first kernel launch or symbol lookup on that
 *     device) and stay reserved until the process exits.
 *   - The first call on a device looks up the array's device address there
 *     (once per device, cached); make that first call before any stream
 *     capture.
 *   - All calls share the array and it keeps the last call's contents;
 *     nothing in it has to start at zero. Calls whose kernels overlap on the
 *     GPU (concurrent streams, several host threads) race on it: serialise
 *     them. */
MIMO_ATTN_API mimo_attn_status mimo_attn_decode_static(const mimo_attn_layer *layer, int dtype, int batch,
                                         const void *q, const void *k_new, const void *v_new,
                                         const int32_t *kv_lens, void *k_cache, void *v_cache,
                                         int cache_capacity, void *out, void *stream);

/* Bytes of workspace mimo_attn_qkv_project needs: the RoPE cos/sin table of
 * positions 0 .. max_past_len + seq - 1. */
MIMO_ATTN_API size_t mimo_attn_qkv_project_workspace_size(const mimo_attn_layer *layer, int batch, int seq,
                                                          int max_past_len);

/* The step before attention, fused: the QKV projection of a chunk of tokens
 * with partial RoPE and the cache write in its epilogue.
 *   y = x W^T with W = w_qkv (no bias), then y's columns split into Hq query
 *   heads of Dqk, Hkv key heads of Dqk and Hkv value heads of Dv; query and
 *   key heads get the layer's partial RoPE at the token's position ("Add
 *   Xiaomi MiMo-V2", "Additional useful info"); values pass through.
 *   x      [batch, seq, hidden_size] bf16.
 *   w_qkv  [Hq*Dqk + Hkv*Dqk + Hkv*Dv, hidden_size] bf16: the rows of W_q,
 *          then W_k, then W_v, each in a linear layer's [out, in] layout.
 *   past_lens: device int32 [batch] or NULL (= all 0): token t of sequence b
 *          sits at position past_lens[b] + t. max_past_len >= every entry
 *          (0 when past_lens is NULL); an entry outside [0, max_past_len]
 *          sets MIMO_ATTN_DEVERR_KV_LEN and that sequence is skipped.
 *   q_out  [batch, seq, Hq, Dqk] bf16: rotated queries (required).
 *   k_out  [batch, seq, Hkv, Dqk] rotated keys, v_out [batch, seq, Hkv, Dv]
 *          values: optional (NULL = not stored).
 *   k_cache, v_cache: optional, both or neither, laid out as in
 *          mimo_attn_prefill_cached (GLOBAL: linear, cache_capacity >=
 *          max_past_len + seq; SWA: ring, cache_capacity == window, which
 *          receives the chunk's last `window` tokens).
 * The outputs are rotated already: attention over them takes a copy of the
 * layer with rotary_dim = 0 (mimo_attn_prefill, or decode-time reads of the
 * caches, which always hold rotated keys).
 * Supported: bf16; Dqk and Dv multiples of 64; rotary_dim 0 or 64;
 * hidden_size a multiple of 64 (else MIMO_ATTN_ERR_UNSUPPORTED). Pointers
 * 16-byte aligned; 32-byte aligned outputs take 32-byte stores. */
MIMO_ATTN_API mimo_attn_status mimo_attn_qkv_project(const mimo_attn_layer *layer, int batch, int seq,
                                                     const void *x, const void *w_qkv, const int32_t *past_lens,
                                                     int max_past_len, void *q_out, void *k_out, void *v_out,
                                                     void *k_cache, void *v_cache, int cache_capacity,
                                                     void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace mimo_attn_decode_fp8kv needs (the same split-KV partial
 * results as the bf16 decode). */
MIMO_ATTN_API size_t mimo_attn_decode_fp8kv_workspace_size(const mimo_attn_layer *layer, int batch,
                                                           int cache_capacity);

/* Decode over an fp8 KV cache. The pages ("Add Xiaomi MiMo-V2", section
 * "Additional useful info") note that the model ships a quantized variant
 * without saying what is quantized or how; this entry point is the plainest
 * reading for the decode hot path: the caches hold OCP FP8 E4M3 codes with
 * one scale per tensor (a cached key is k_scale * e4m3 value, a cached value
 * v_scale * e4m3 value), everything else is the bf16 decode.
 *   q [batch, Hq, Dqk], k_new [batch, Hkv, Dqk], v_new [batch, Hkv, Dv]:
 *          bf16, unrotated, as in mimo_attn_decode.
 *   kv_lens, cache_capacity, layouts: as in mimo_attn_decode, with one byte
 *          per element in k_cache / v_cache ([batch, cap, Hkv, D] uint8).
 *   k_scale, v_scale: finite, > 0.
 *   The new token's key, rotated in fp32, is divided by k_scale and
 *          stored as its E4M3 code (round to nearest even, saturating at
 *          +-448); v_new likewise with v_scale. Its own score and value use
 *          the stored codes, so the result is the attention over the cache as
 *          it stands after the call.
 *   out [batch, Hq, Dv] bf16. Scores and the PV product are computed from
 *          f16 operands (every E4M3 value is exact in f16) with fp32
 *          accumulation; the query is rounded to f16.
 * Supported: Dqk 192, Dv 128, Hq/Hkv <= 16 (else MIMO_ATTN_ERR_UNSUPPORTED).
 * q, k_new, v_new, out and both caches must be 16-byte aligned. */
MIMO_ATTN_API mimo_attn_status mimo_attn_decode_fp8kv(const mimo_attn_layer *layer, int batch, const void *q,
                                                      const void *k_new, const void *v_new,
                                                      const int32_t *kv_lens, void *k_cache, void *v_cache,
                                                      int cache_capacity, float k_scale, float v_scale,
                                                      void *out, void *workspace, size_t workspace_bytes,
                                                      void *stream);

/* dst[i] = E4M3 code of src[i] / scale for i < n (src bf16, dst uint8;
 * round to nearest even, saturating at +-448, NaN stays NaN). Fills an fp8
 * cache from bf16 keys and values (keys already rotated). scale finite, > 0. */
MIMO_ATTN_API mimo_attn_status mimo_attn_quantize_fp8(const void *src, void *dst, size_t n, float scale,
                                                      void *stream);

/* Device error word bits (sticky until read). */
#define MIMO_ATTN_DEVERR_KV_LEN 0x1u   /* a kv_lens entry was out of range */
#define MIMO_ATTN_DEVERR_TIMEOUT 0x2u  /* a kernel pipeline wait hit its iteration limit */

/* Reads and clears the device error word of the current device
 * (synchronises the device). Returns MIMO_ATTN_OK and stores the bits in
 * *bits, or MIMO_ATTN_ERR_CUDA. */
MIMO_ATTN_API mimo_attn_status mimo_attn_get_device_error(uint32_t *bits);

/* Static description of a status code. */
MIMO_ATTN_API const char *mimo_attn_status_string(mimo_attn_status status);

/* Test hook: while non-zero, every launching entry point returns
 * MIMO_ATTN_ERR_CUDA after its argument checks, without launching. Lets the
 * host-side error path be tested without provoking a GPU fault. */
MIMO_ATTN_API void mimo_attn_debug_fail_launches(int enable);

/* Test hook: sets the pipeline-wait limit of the current device, in SM clock
 * cycles; cycles <= 0 restores the default (8e9 cycles, ~4 s at 2 GHz). Every
 * bounded wait of the library's pipelined kernels (an mbarrier that a copy or
 * a tensor-core operation should complete) gives up after this many cycles,
 * sets MIMO_ATTN_DEVERR_TIMEOUT and lets its kernel tear down. Synchronises
 * the device. Returns MIMO_ATTN_OK or MIMO_ATTN_ERR_CUDA. Meant for tests of
 * the timeout path together with mimo_attn_debug_wait_probe; a short limit
 * during real work can end healthy kernels early. */
MIMO_ATTN_API mimo_attn_status mimo_attn_debug_set_wait_limit(long long cycles);

/* Test hook: launches one CTA on `stream` that waits, with the library's
 * bounded wait, on an mbarrier nothing ever arrives on. The wait ends at the
 * device's wait limit and sets MIMO_ATTN_DEVERR_TIMEOUT; no copy or
 * tensor-core operation is in flight, so the context stays usable. With the
 * default limit the kernel runs for ~4 s: shorten the limit first. */
MIMO_ATTN_API mimo_attn_status mimo_attn_debug_wait_probe(void *stream);

/* Version string of the library. */
MIMO_ATTN_API const char *mimo_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MIMO_ATTN_H */
