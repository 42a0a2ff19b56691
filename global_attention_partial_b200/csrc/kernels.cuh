// Internal launch interface of the MiMo-V2-Flash attention kernels.
#pragma once

#include "common.cuh"

#include <atomic>

namespace mimo {

// Raises `kernel`'s dynamic shared-memory limit to `bytes` once per device
// (the attribute belongs to the device's copy of the kernel). When
// `launch_regs` > 0 it first checks that the kernel was compiled with exactly
// that many registers per thread: the warp-specialised kernels split the
// block's register pool with setmaxnreg and must not launch with a smaller
// one. `done` is one bit per device ordinal (< 64), shared by the host
// threads that call the launcher.
template <typename K>
inline cudaError_t prepare_kernel_once(K kernel, int bytes, std::atomic<unsigned long long> &done, int launch_regs = 0)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit)
        return cudaSuccess;
    if (launch_regs > 0) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kernel);
        if (e != cudaSuccess)
            return e;
        if (fa.numRegs != launch_regs)
            return cudaErrorInvalidConfiguration;
    }
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        done.fetch_or(bit, std::memory_order_release);
    return e;
}


enum { kDtypeBf16 = 0, kDtypeFp32 = 1 };

// Per-layer values resolved on the host from mimo_attn_layer.
struct LayerArgs {
    int layer_type;    // 0 global, 1 sliding window
    int Hq, Hkv, G;    // G = Hq / Hkv query heads per KV head
    int Dqk, Dv;
    int window;        // sliding layers only
    float scale_log2;  // softmax scale * log2(e): scores are kept in base-2 units
    float v_scale;     // sqrt(hidden / (Hq * Dv))
    const float *sinks;  // [Hq] natural-log sink logits or nullptr
    RopeArgs rope;
};

// Rotates K at each token's position and stores it, and copies K/V into the
// caches. dst_k receives every token (row i of [B, dst_rows, Hkv, Dqk]);
// ring_k / ring_v (sliding-window ring, slot i mod window) receive the last
// `window` tokens; lin_v (global value cache [B, lin_rows, Hkv, Dv]) receives
// every token.
struct KprepArgs {
    const void *k;
    const void *v;
    const int *positions;  // nullptr: position = sequence index
    void *dst_k;
    long long dst_rows;
    void *ring_k;
    void *ring_v;
    void *lin_v;
    long long lin_rows;
    int B, S, Hkv, Dqk, Dv, window;
    float2 *rope_table;  // [S][rotary_dim/2] (cos, sin) of each token's position, built by launch_kprep
    RopeArgs rope;
};
cudaError_t launch_kprep(const KprepArgs &a, int dtype, cudaStream_t stream);

// cos / sin of positions 0..n-1 (or positions[0..n-1] when positions is not
// null) for every rotary pair: table [n][rotary_dim/2].
cudaError_t launch_rope_table(const RopeArgs &rope, float2 *table, long long n, cudaStream_t stream,
                              const int *positions = nullptr);

// The sliding-window ring of a prefill: the last `window` tokens' rotated
// keys and values into slots i mod window (a.ring_k / a.ring_v, a.rope_table
// filled); nothing else.
cudaError_t launch_kprep_ring(const KprepArgs &a, int dtype, cudaStream_t stream);

// Prefill continuing a cache: writes the chunk's rotated keys and values
// where the attention kernels read them. Global layers: cache rows
// past_lens[b] + t. Sliding layers: the key window kv_k / kv_v
// [B, key_off + S, Hkv, D] (row u = position past_lens[b] - key_off + u: old
// keys from the ring, the chunk's own rotated), then the ring takes the
// chunk's last `window` tokens. Out-of-range past_lens set the device error
// word; their rows are skipped.
struct CachedPrepArgs {
    const void *k;
    const void *v;
    const int *past_lens;
    int max_past;
    void *k_cache;
    void *v_cache;
    int cap;
    void *kv_k;
    void *kv_v;
    int key_off;
    int layer_type, B, S, Hkv, Dqk, Dv, window;
    const float2 *rope_table;
    RopeArgs rope;
    unsigned *err;
};
cudaError_t launch_cached_prep(const CachedPrepArgs &a, int dtype, cudaStream_t stream);

// Prefill attention on CUDA cores (any dims up to 256, fp32 or bf16).
// krot: rotated keys [B, krot_rows, Hkv, Dqk].
// Query token t of batch b attends the keys of index (t + key offset), the
// key offset being past_lens[b] on global layers and swa_key_off on sliding
// layers; without past_lens (plain prefill) both are 0 and queries and keys
// share the sequence index. krot / v hold key_rows / v_rows rows per batch
// (row stride krot_rows / v_rows), of which the first key_rows_valid are read.
struct PrefillArgs {
    const void *q;
    const void *krot;
    long long krot_rows;
    long long key_rows_valid;
    const void *v;
    long long v_rows;
    const int *positions;
    const float2 *rope_table;  // (cos, sin) per position: row (past_lens[b] + t) for token t
    const int *past_lens;      // [B] tokens already in the cache, or nullptr
    int max_past;              // >= every past_lens[b]: the table has max_past + S rows
    int swa_key_off;           // sliding layers: key index of query 0 (a multiple of 16)
    int k_unrotated;           // krot holds the input keys: the kernel rotates them (prefill_swa only)
    void *out;
    int B, S;
    unsigned *err;
};
cudaError_t launch_prefill_simt(const LayerArgs &L, const PrefillArgs &a, int dtype,
                                cudaStream_t stream);

// Prefill attention on the tcgen05 tensor cores (bf16, Dqk 192, Dv 128).
bool prefill_tc_supported(const LayerArgs &L);
cudaError_t launch_prefill_tc(const LayerArgs &L, const PrefillArgs &a, cudaStream_t stream);

// Global-layer prefill with two query heads of a KV group per CTA (needs an
// even number of query heads per KV head).
bool prefill_ga_supported(const LayerArgs &L);
cudaError_t launch_prefill_ga(const LayerArgs &L, const PrefillArgs &a, cudaStream_t stream);

// Sliding-window prefill whose tiles need a single key span (persistent,
// one CTA per SM); rope_table holds cos / sin per sequence index. With
// a.k_unrotated the kernel rotates the keys itself (needs swa_rotates_keys).
bool prefill_swa_supported(const LayerArgs &L);
bool swa_rotates_keys(const LayerArgs &L);
cudaError_t launch_prefill_swa(const LayerArgs &L, const PrefillArgs &a, const float2 *rope_table,
                               int num_sms, cudaStream_t stream);

// 4-D bf16 TMA map with 128-byte swizzle over [d3][d2_alloc][d1][d0] (d0
// innermost), of which the first d2 rows along dimension 2 are in bounds.
bool make_bf16_map_4d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint64_t d2_alloc, uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2);

// Decode. Caches: GLOBAL linear [B, cap, Hkv, D]; SWA ring [B, window, Hkv, D].
struct DecodeArgs {
    const void *q;
    const void *k_new;
    const void *v_new;
    const int *kv_lens;
    void *k_cache;
    void *v_cache;
    int cap;
    void *out;
    float *partial;  // workspace: [B, Hq, max_splits, Dv + 2] fp32
    int max_splits;
    int chunk;       // keys per split
    int B;
    unsigned *err;
    // E4M3 caches (bytes): a cached value is scale * e4m3(code); the new
    // token's rotated key and value are stored as e4m3(x / scale). The
    // scales also multiply the scores (k_scale) and the output (v_scale):
    // the caller folds them into the layer's softmax and V scales.
    int fp8_cache;
    float k_scale, v_scale;
};
// QKV projection with the fused RoPE / store epilogue (csrc/qkv_proj.cu).
// x [B*S, hidden] and w [Hq*Dqk + Hkv*(Dqk+Dv), hidden] bf16; q [B, S, Hq,
// Dqk], k / v [B, S, Hkv, D] (k, v may be null), caches as in the cached
// prefill (both or neither). rope_table: max_past + S rows of 32 (cos, sin)
// pairs, filled here.
struct QkvArgs {
    const void *x;
    const void *w;
    const int *past_lens;  // nullptr: position = sequence index
    int max_past;
    void *q, *k, *v;
    void *k_cache, *v_cache;
    int cap;
    int B, S, hidden;
    float2 *rope_table;
    unsigned *err;
};
bool qkv_proj_supported(const LayerArgs &L, int hidden);
cudaError_t launch_qkv_proj(const LayerArgs &L, const QkvArgs &a, int num_sms, cudaStream_t stream);

// dst[i] = e4m3(src[i] / scale) (bf16 in, E4M3 codes out; nearest, saturating).
cudaError_t launch_quantize_e4m3(const void *src, void *dst, size_t n, float scale, cudaStream_t stream);
int decode_chunk_keys(const LayerArgs &L, int dtype);
int decode_max_splits(const LayerArgs &L, int dtype, int cap);
cudaError_t launch_decode(const LayerArgs &L, const DecodeArgs &a, int dtype, cudaStream_t stream);

// One CTA that waits on an mbarrier nothing arrives on, until the device's
// wait limit ends the wait (timeout bit set in *err). Test probe only.
cudaError_t launch_wait_probe(unsigned *err, cudaStream_t stream);

} // namespace mimo
