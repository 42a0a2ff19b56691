// C ABI of the MiMo-V2-Flash attention library (declared in include/mimo_attn.h).
//
// Host side only: argument checks (all before any launch), per-layer
// parameter resolution (softmax scale, V scale sqrt(hidden/(Hq*Dv)), RoPE
// inverse frequencies theta^(-2j/r) in double precision), workspace layout,
// and the launches. No device memory is allocated here.
#include "../../include/mimo_attn.h"
#include "kernels.cuh"

#include <math.h>
#include <string.h>

#include <mutex>

namespace {

// Device status block: the error word (sticky bits set by kernels: kv_lens
// out of range, wait timeouts), read by mimo_attn_get_device_error(), and the
// pipeline-wait limit the kernels read beside it. One copy per device.
__device__ mimo::DeviceStatus g_device_status;

int g_fail_launches = 0;

constexpr int kMaxDevices = 64;

// Device addresses looked up once per device and cached: the status block
// here, the decode scratch array further down. One lock guards both caches,
// so host threads that make their first call on a device at the same time
// never race on them.
std::mutex g_symbol_mutex;
unsigned *g_err_ptr[kMaxDevices];

unsigned *device_error_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_symbol_mutex);
    if (g_err_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess)
            return nullptr;
        g_err_ptr[dev] = &static_cast<mimo::DeviceStatus *>(p)->error;
    }
    return g_err_ptr[dev];
}

int g_num_sms[kMaxDevices];

// Streaming multiprocessors of the current device (cached per device).
int num_sms()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return 148;
    if (g_num_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        g_num_sms[dev] = n;
    }
    return g_num_sms[dev];
}

size_t elem_size(int dtype) { return dtype == MIMO_ATTN_BF16 ? 2 : 4; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the per-layer struct; fills the resolved arguments.
mimo_attn_status resolve_layer(const mimo_attn_layer *layer, int dtype, mimo::LayerArgs *out)
{
    if (layer == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (dtype != MIMO_ATTN_BF16 && dtype != MIMO_ATTN_FP32)
        return MIMO_ATTN_ERR_INVALID_ARG;
    const mimo_attn_layer &l = *layer;
    if (l.layer_type != MIMO_ATTN_GLOBAL && l.layer_type != MIMO_ATTN_SWA)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (l.num_q_heads < 1 || l.num_kv_heads < 1 || l.num_q_heads % l.num_kv_heads != 0)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (l.qk_dim < 2 || l.v_dim < 1 || (l.qk_dim % 2) != 0)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (l.rotary_dim < 0 || l.rotary_dim > l.qk_dim || (l.rotary_dim % 2) != 0)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (l.layer_type == MIMO_ATTN_SWA && l.window < 1)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (l.layer_type == MIMO_ATTN_GLOBAL && l.sinks != nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (l.hidden_size < 1 || !(l.rope_theta > 0.0) || !isfinite(l.rope_theta))
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (!(l.softmax_scale >= 0.f) || !isfinite(l.softmax_scale))
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (l.qk_dim > 256 || l.v_dim > 256)
        return MIMO_ATTN_ERR_UNSUPPORTED;

    mimo::LayerArgs &L = *out;
    memset(&L, 0, sizeof(L));
    L.layer_type = l.layer_type;
    L.Hq = l.num_q_heads;
    L.Hkv = l.num_kv_heads;
    L.G = l.num_q_heads / l.num_kv_heads;
    L.Dqk = l.qk_dim;
    L.Dv = l.v_dim;
    L.window = l.layer_type == MIMO_ATTN_SWA ? l.window : 0;
    const double scale = l.softmax_scale > 0.f ? (double)l.softmax_scale : 1.0 / sqrt((double)l.qk_dim);
    L.scale_log2 = (float)(scale * 1.4426950408889634074);
    L.v_scale = (float)sqrt((double)l.hidden_size / ((double)l.num_q_heads * (double)l.v_dim));
    L.sinks = l.sinks;
    L.rope.rotary_dim = l.rotary_dim;
    L.rope.half = l.rotary_dim / 2;
    for (int j = 0; j < L.rope.half; ++j)
        L.rope.inv_freq[j] = pow(l.rope_theta, -2.0 * (double)j / (double)l.rotary_dim);
    return MIMO_ATTN_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Continuing a cache on a sliding layer: window row of query 0. At least the
// window - 1 older positions precede it; a multiple of 16 keeps the 16-key
// blocks of the tensor-core kernel aligned with the queries' spans.
int cached_key_off(const mimo::LayerArgs &L) { return (int)round_up((size_t)(L.window - 1), 16); }

// A sliding layer whose keys the tensor-core kernel rotates itself: no
// rotated copy of K is written, the workspace holds only the RoPE table.
bool swa_fused_keys(const mimo::LayerArgs &L, int dtype)
{
    return dtype == MIMO_ATTN_BF16 && mimo::prefill_swa_supported(L) &&
           (L.rope.half == 0 || mimo::swa_rotates_keys(L));
}

} // namespace

extern "C" {

int mimo_attn_rotary_dim(double partial_rotary_factor, int qk_dim)
{
    const double r = partial_rotary_factor * (double)qk_dim;
    if (!isfinite(r) || r < 0.0 || r > 2147483647.0)
        return -1;
    return (int)r;  // truncation toward zero: Python int() of a non-negative float
}

size_t mimo_attn_prefill_workspace_size(const mimo_attn_layer *layer, int dtype, int batch, int seq)
{
    mimo::LayerArgs L;
    if (resolve_layer(layer, dtype, &L) != MIMO_ATTN_OK || batch < 0 || seq < 0)
        return 0;
    // the RoPE cos/sin table [S, r/2], then the rotated keys [B, S, Hkv, Dqk]
    // (none when the sliding-window kernel rotates the keys itself)
    const size_t table = round_up((size_t)seq * L.rope.half * sizeof(float2), 256);
    if (swa_fused_keys(L, dtype))
        return table;
    return table + round_up((size_t)batch * seq * L.Hkv * L.Dqk * elem_size(dtype), 256);
}

mimo_attn_status mimo_attn_prefill(const mimo_attn_layer *layer, int dtype, int batch, int seq,
                                   const void *q, const void *k, const void *v,
                                   const int32_t *positions, void *out, void *k_cache,
                                   void *v_cache, int cache_capacity, void *workspace,
                                   size_t workspace_bytes, void *stream)
{
    mimo::LayerArgs L;
    mimo_attn_status st = resolve_layer(layer, dtype, &L);
    if (st != MIMO_ATTN_OK)
        return st;
    if (batch < 0 || seq < 0)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if ((k_cache == nullptr) != (v_cache == nullptr))
        return MIMO_ATTN_ERR_INVALID_ARG;
    const bool has_cache = k_cache != nullptr;
    if (has_cache) {
        if (L.layer_type == MIMO_ATTN_SWA && cache_capacity != L.window)
            return MIMO_ATTN_ERR_INVALID_ARG;
        if (L.layer_type == MIMO_ATTN_GLOBAL && cache_capacity < seq)
            return MIMO_ATTN_ERR_INVALID_ARG;
    }
    if (batch == 0 || seq == 0)
        return MIMO_ATTN_OK;
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (dtype == MIMO_ATTN_BF16 &&
        !(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out) && aligned16(k_cache) &&
          aligned16(v_cache) && aligned16(workspace)))
        return MIMO_ATTN_ERR_INVALID_ARG;
    // Workspace: the RoPE cos/sin table [S, r/2] first, then the rotated keys
    // (which go straight into a global cache when the caller passes one).
    const bool keys_in_cache = has_cache && L.layer_type == MIMO_ATTN_GLOBAL;
    const bool use_swa_kernel = dtype == MIMO_ATTN_BF16 && mimo::prefill_swa_supported(L);
    const size_t table_bytes = round_up((size_t)seq * L.rope.half * sizeof(float2), 256);
    const size_t need = keys_in_cache ? table_bytes : mimo_attn_prefill_workspace_size(layer, dtype, batch, seq);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return MIMO_ATTN_ERR_WORKSPACE;
    if (g_fail_launches)
        return MIMO_ATTN_ERR_CUDA;
    unsigned *err = device_error_ptr();
    if (err == nullptr)
        return MIMO_ATTN_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (swa_fused_keys(L, dtype)) {
        // Sliding layer on the tensor-core kernel, which rotates K in shared
        // memory: the RoPE table, the ring (when asked for), the attention.
        float2 *table = L.rope.half > 0 ? reinterpret_cast<float2 *>(workspace) : nullptr;
        if (mimo::launch_rope_table(L.rope, table, seq, s, positions) != cudaSuccess)
            return MIMO_ATTN_ERR_CUDA;
        if (has_cache) {
            mimo::KprepArgs kr;
            memset(&kr, 0, sizeof(kr));
            kr.k = k;
            kr.v = v;
            kr.ring_k = k_cache;
            kr.ring_v = v_cache;
            kr.B = batch;
            kr.S = seq;
            kr.Hkv = L.Hkv;
            kr.Dqk = L.Dqk;
            kr.Dv = L.Dv;
            kr.window = L.window;
            kr.rope_table = table;
            kr.rope = L.rope;
            if (mimo::launch_kprep_ring(kr, dtype, s) != cudaSuccess)
                return MIMO_ATTN_ERR_CUDA;
        }
        mimo::PrefillArgs pa;
        memset(&pa, 0, sizeof(pa));
        pa.q = q;
        pa.krot = k;
        pa.krot_rows = seq;
        pa.key_rows_valid = seq;
        pa.k_unrotated = L.rope.half > 0;
        pa.v = v;
        pa.v_rows = seq;
        pa.positions = positions;
        pa.rope_table = table;
        pa.out = out;
        pa.B = batch;
        pa.S = seq;
        pa.err = err;
        return mimo::launch_prefill_swa(L, pa, table, num_sms(), s) == cudaSuccess ? MIMO_ATTN_OK
                                                                                    : MIMO_ATTN_ERR_CUDA;
    }

    mimo::KprepArgs kp;
    memset(&kp, 0, sizeof(kp));
    kp.k = k;
    kp.v = v;
    kp.positions = positions;
    kp.dst_k = keys_in_cache ? k_cache : static_cast<void *>(static_cast<char *>(workspace) + table_bytes);
    kp.dst_rows = keys_in_cache ? cache_capacity : seq;
    if (has_cache && L.layer_type == MIMO_ATTN_SWA) {
        kp.ring_k = k_cache;
        kp.ring_v = v_cache;
    }
    if (keys_in_cache) {
        kp.lin_v = v_cache;
        kp.lin_rows = cache_capacity;
    }
    kp.B = batch;
    kp.S = seq;
    kp.Hkv = L.Hkv;
    kp.Dqk = L.Dqk;
    kp.Dv = L.Dv;
    kp.window = L.layer_type == MIMO_ATTN_SWA ? L.window : 0;
    kp.rope_table = L.rope.half > 0 ? reinterpret_cast<float2 *>(workspace) : nullptr;
    kp.rope = L.rope;
    if (mimo::launch_kprep(kp, dtype, s) != cudaSuccess)
        return MIMO_ATTN_ERR_CUDA;

    mimo::PrefillArgs pa;
    memset(&pa, 0, sizeof(pa));
    pa.q = q;
    pa.krot = kp.dst_k;
    pa.krot_rows = kp.dst_rows;
    pa.key_rows_valid = seq;
    pa.v = v;
    pa.v_rows = seq;
    pa.positions = positions;
    pa.rope_table = kp.rope_table;
    pa.out = out;
    pa.B = batch;
    pa.S = seq;
    pa.err = err;
    cudaError_t e;
    if (use_swa_kernel)
        e = mimo::launch_prefill_swa(L, pa, pa.rope_table, num_sms(), s);
    else if (dtype == MIMO_ATTN_BF16 && mimo::prefill_ga_supported(L))
        e = mimo::launch_prefill_ga(L, pa, s);
    else if (dtype == MIMO_ATTN_BF16 && mimo::prefill_tc_supported(L))
        e = mimo::launch_prefill_tc(L, pa, s);
    else
        e = mimo::launch_prefill_simt(L, pa, dtype, s);
    return e == cudaSuccess ? MIMO_ATTN_OK : MIMO_ATTN_ERR_CUDA;
}

size_t mimo_attn_prefill_cached_workspace_size(const mimo_attn_layer *layer, int dtype, int batch, int seq,
                                               int max_past_len)
{
    mimo::LayerArgs L;
    if (resolve_layer(layer, dtype, &L) != MIMO_ATTN_OK || batch < 0 || seq < 0 || max_past_len < 0)
        return 0;
    // the RoPE table of positions 0 .. max_past + seq - 1, then (SWA) the key
    // and value windows [B, key_off + seq, Hkv, D]
    size_t bytes = round_up(((size_t)max_past_len + seq) * L.rope.half * sizeof(float2), 256);
    if (L.layer_type == MIMO_ATTN_SWA) {
        const size_t rows = (size_t)batch * (cached_key_off(L) + seq) * L.Hkv;
        bytes += round_up(rows * L.Dqk * elem_size(dtype), 256) + round_up(rows * L.Dv * elem_size(dtype), 256);
    }
    return bytes;
}

mimo_attn_status mimo_attn_prefill_cached(const mimo_attn_layer *layer, int dtype, int batch, int seq,
                                          const void *q, const void *k, const void *v, const int32_t *past_lens,
                                          int max_past_len, void *out, void *k_cache, void *v_cache,
                                          int cache_capacity, void *workspace, size_t workspace_bytes,
                                          void *stream)
{
    mimo::LayerArgs L;
    mimo_attn_status st = resolve_layer(layer, dtype, &L);
    if (st != MIMO_ATTN_OK)
        return st;
    if (batch < 0 || seq < 0 || max_past_len < 0)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (k_cache == nullptr || v_cache == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (L.layer_type == MIMO_ATTN_SWA && cache_capacity != L.window)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (L.layer_type == MIMO_ATTN_GLOBAL && (long long)cache_capacity < (long long)max_past_len + seq)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (batch == 0 || seq == 0)
        return MIMO_ATTN_OK;
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || past_lens == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (dtype == MIMO_ATTN_BF16 &&
        !(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out) && aligned16(k_cache) &&
          aligned16(v_cache) && aligned16(workspace)))
        return MIMO_ATTN_ERR_INVALID_ARG;
    const size_t need = mimo_attn_prefill_cached_workspace_size(layer, dtype, batch, seq, max_past_len);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return MIMO_ATTN_ERR_WORKSPACE;
    if (g_fail_launches)
        return MIMO_ATTN_ERR_CUDA;
    unsigned *err = device_error_ptr();
    if (err == nullptr)
        return MIMO_ATTN_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    const bool swa = L.layer_type == MIMO_ATTN_SWA;
    const int key_off = swa ? cached_key_off(L) : 0;
    const size_t table_bytes = round_up(((size_t)max_past_len + seq) * L.rope.half * sizeof(float2), 256);
    float2 *table = L.rope.half > 0 ? reinterpret_cast<float2 *>(workspace) : nullptr;
    char *win = static_cast<char *>(workspace) + table_bytes;
    const size_t win_rows = (size_t)batch * (key_off + seq) * L.Hkv;
    void *win_k = swa ? static_cast<void *>(win) : nullptr;
    void *win_v = swa ? static_cast<void *>(win + round_up(win_rows * L.Dqk * elem_size(dtype), 256)) : nullptr;
    if (mimo::launch_rope_table(L.rope, table, (long long)max_past_len + seq, s) != cudaSuccess)
        return MIMO_ATTN_ERR_CUDA;

    mimo::CachedPrepArgs cp;
    memset(&cp, 0, sizeof(cp));
    cp.k = k;
    cp.v = v;
    cp.past_lens = past_lens;
    cp.max_past = max_past_len;
    cp.k_cache = k_cache;
    cp.v_cache = v_cache;
    cp.cap = cache_capacity;
    cp.kv_k = win_k;
    cp.kv_v = win_v;
    cp.key_off = key_off;
    cp.layer_type = L.layer_type;
    cp.B = batch;
    cp.S = seq;
    cp.Hkv = L.Hkv;
    cp.Dqk = L.Dqk;
    cp.Dv = L.Dv;
    cp.window = L.window;
    cp.rope_table = table;
    cp.rope = L.rope;
    cp.err = err;
    if (mimo::launch_cached_prep(cp, dtype, s) != cudaSuccess)
        return MIMO_ATTN_ERR_CUDA;

    // Keys and values: the global cache itself, or the SWA windows.
    mimo::PrefillArgs pa;
    memset(&pa, 0, sizeof(pa));
    pa.q = q;
    pa.krot = swa ? win_k : k_cache;
    pa.krot_rows = swa ? key_off + seq : cache_capacity;
    pa.key_rows_valid = pa.krot_rows;
    pa.v = swa ? win_v : v_cache;
    pa.v_rows = pa.krot_rows;
    pa.rope_table = table;
    pa.past_lens = past_lens;
    pa.max_past = max_past_len;
    pa.swa_key_off = key_off;
    pa.out = out;
    pa.B = batch;
    pa.S = seq;
    pa.err = err;
    cudaError_t e;
    if (dtype == MIMO_ATTN_BF16 && swa && mimo::prefill_swa_supported(L))
        e = mimo::launch_prefill_swa(L, pa, table, num_sms(), s);
    else if (dtype == MIMO_ATTN_BF16 && !swa && mimo::prefill_ga_supported(L))
        e = mimo::launch_prefill_ga(L, pa, s);
    else
        e = mimo::launch_prefill_simt(L, pa, dtype, s);
    return e == cudaSuccess ? MIMO_ATTN_OK : MIMO_ATTN_ERR_CUDA;
}

size_t mimo_attn_decode_workspace_size(const mimo_attn_layer *layer, int dtype, int batch,
                                       int cache_capacity)
{
    mimo::LayerArgs L;
    if (resolve_layer(layer, dtype, &L) != MIMO_ATTN_OK || batch < 0 || cache_capacity < 1)
        return 0;
    const int splits = mimo::decode_max_splits(L, dtype, cache_capacity);
    if (splits <= 1)
        return 0;
    return round_up((size_t)batch * L.Hq * splits * (L.Dv + 2) * sizeof(float), 256);
}

mimo_attn_status mimo_attn_decode(const mimo_attn_layer *layer, int dtype, int batch,
                                  const void *q, const void *k_new, const void *v_new,
                                  const int32_t *kv_lens, void *k_cache, void *v_cache,
                                  int cache_capacity, void *out, void *workspace,
                                  size_t workspace_bytes, void *stream)
{
    mimo::LayerArgs L;
    mimo_attn_status st = resolve_layer(layer, dtype, &L);
    if (st != MIMO_ATTN_OK)
        return st;
    if (batch < 0 || cache_capacity < 1)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (L.layer_type == MIMO_ATTN_SWA && cache_capacity != L.window)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (batch == 0)
        return MIMO_ATTN_OK;
    if (q == nullptr || k_new == nullptr || v_new == nullptr || kv_lens == nullptr ||
        k_cache == nullptr || v_cache == nullptr || out == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (dtype == MIMO_ATTN_BF16 &&
        !(aligned16(q) && aligned16(k_new) && aligned16(v_new) && aligned16(k_cache) &&
          aligned16(v_cache) && aligned16(out)))
        return MIMO_ATTN_ERR_INVALID_ARG;
    const size_t need = mimo_attn_decode_workspace_size(layer, dtype, batch, cache_capacity);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return MIMO_ATTN_ERR_WORKSPACE;
    if (g_fail_launches)
        return MIMO_ATTN_ERR_CUDA;
    unsigned *err = device_error_ptr();
    if (err == nullptr)
        return MIMO_ATTN_ERR_CUDA;

    mimo::DecodeArgs da;
    memset(&da, 0, sizeof(da));
    da.q = q;
    da.k_new = k_new;
    da.v_new = v_new;
    da.kv_lens = kv_lens;
    da.k_cache = k_cache;
    da.v_cache = v_cache;
    da.cap = cache_capacity;
    da.out = out;
    da.partial = static_cast<float *>(workspace);
    da.max_splits = mimo::decode_max_splits(L, dtype, cache_capacity);
    da.chunk = mimo::decode_chunk_keys(L, dtype);
    da.B = batch;
    da.err = err;
    cudaError_t e = mimo::launch_decode(L, da, dtype, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MIMO_ATTN_OK : MIMO_ATTN_ERR_CUDA;
}

size_t mimo_attn_qkv_project_workspace_size(const mimo_attn_layer *layer, int batch, int seq, int max_past_len)
{
    mimo::LayerArgs L;
    if (resolve_layer(layer, MIMO_ATTN_BF16, &L) != MIMO_ATTN_OK || batch < 0 || seq < 0 || max_past_len < 0)
        return 0;
    // the RoPE table of positions 0 .. max_past + seq - 1
    return round_up(((size_t)max_past_len + seq) * L.rope.half * sizeof(float2), 256);
}

mimo_attn_status mimo_attn_qkv_project(const mimo_attn_layer *layer, int batch, int seq, const void *x,
                                       const void *w_qkv, const int32_t *past_lens, int max_past_len, void *q_out,
                                       void *k_out, void *v_out, void *k_cache, void *v_cache, int cache_capacity,
                                       void *workspace, size_t workspace_bytes, void *stream)
{
    mimo::LayerArgs L;
    mimo_attn_status st = resolve_layer(layer, MIMO_ATTN_BF16, &L);
    if (st != MIMO_ATTN_OK)
        return st;
    if (batch < 0 || seq < 0 || max_past_len < 0)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (past_lens == nullptr && max_past_len != 0)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if ((k_cache == nullptr) != (v_cache == nullptr))
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (k_cache != nullptr) {
        if (L.layer_type == MIMO_ATTN_SWA && cache_capacity != L.window)
            return MIMO_ATTN_ERR_INVALID_ARG;
        if (L.layer_type == MIMO_ATTN_GLOBAL && (cache_capacity < 1 || (long long)max_past_len + seq > cache_capacity))
            return MIMO_ATTN_ERR_INVALID_ARG;
    }
    if (!mimo::qkv_proj_supported(L, layer->hidden_size))
        return MIMO_ATTN_ERR_UNSUPPORTED;
    if (batch == 0 || seq == 0)
        return MIMO_ATTN_OK;
    if (x == nullptr || w_qkv == nullptr || q_out == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (!(aligned16(x) && aligned16(w_qkv) && aligned16(q_out) && aligned16(k_out) && aligned16(v_out) &&
          aligned16(k_cache) && aligned16(v_cache)))
        return MIMO_ATTN_ERR_INVALID_ARG;
    const size_t need = mimo_attn_qkv_project_workspace_size(layer, batch, seq, max_past_len);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return MIMO_ATTN_ERR_WORKSPACE;
    if (g_fail_launches)
        return MIMO_ATTN_ERR_CUDA;
    unsigned *err = device_error_ptr();
    if (err == nullptr)
        return MIMO_ATTN_ERR_CUDA;
    mimo::QkvArgs a;
    memset(&a, 0, sizeof(a));
    a.x = x;
    a.w = w_qkv;
    a.past_lens = past_lens;
    a.max_past = max_past_len;
    a.q = q_out;
    a.k = k_out;
    a.v = v_out;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.cap = cache_capacity;
    a.B = batch;
    a.S = seq;
    a.hidden = layer->hidden_size;
    a.rope_table = L.rope.half > 0 ? static_cast<float2 *>(workspace) : nullptr;
    a.err = err;
    cudaError_t e = mimo::launch_qkv_proj(L, a, num_sms(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MIMO_ATTN_OK : MIMO_ATTN_ERR_CUDA;
}

size_t mimo_attn_decode_fp8kv_workspace_size(const mimo_attn_layer *layer, int batch, int cache_capacity)
{
    return mimo_attn_decode_workspace_size(layer, MIMO_ATTN_BF16, batch, cache_capacity);
}

mimo_attn_status mimo_attn_decode_fp8kv(const mimo_attn_layer *layer, int batch, const void *q, const void *k_new,
                                        const void *v_new, const int32_t *kv_lens, void *k_cache, void *v_cache,
                                        int cache_capacity, float k_scale, float v_scale, void *out,
                                        void *workspace, size_t workspace_bytes, void *stream)
{
    mimo::LayerArgs L;
    mimo_attn_status st = resolve_layer(layer, MIMO_ATTN_BF16, &L);
    if (st != MIMO_ATTN_OK)
        return st;
    if (batch < 0 || cache_capacity < 1)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (L.layer_type == MIMO_ATTN_SWA && cache_capacity != L.window)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(k_scale) || !isfinite(v_scale))
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (L.Dqk != 192 || L.Dv != 128 || L.G > 16)
        return MIMO_ATTN_ERR_UNSUPPORTED;
    if (batch == 0)
        return MIMO_ATTN_OK;
    if (q == nullptr || k_new == nullptr || v_new == nullptr || kv_lens == nullptr || k_cache == nullptr ||
        v_cache == nullptr || out == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (!(aligned16(q) && aligned16(k_new) && aligned16(v_new) && aligned16(k_cache) && aligned16(v_cache) &&
          aligned16(out)))
        return MIMO_ATTN_ERR_INVALID_ARG;
    const size_t need = mimo_attn_decode_fp8kv_workspace_size(layer, batch, cache_capacity);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return MIMO_ATTN_ERR_WORKSPACE;
    if (g_fail_launches)
        return MIMO_ATTN_ERR_CUDA;
    unsigned *err = device_error_ptr();
    if (err == nullptr)
        return MIMO_ATTN_ERR_CUDA;
    // a cached value is scale * code value: the key scale multiplies every
    // score, the value scale the output
    L.scale_log2 *= k_scale;
    L.v_scale *= v_scale;
    mimo::DecodeArgs da;
    memset(&da, 0, sizeof(da));
    da.q = q;
    da.k_new = k_new;
    da.v_new = v_new;
    da.kv_lens = kv_lens;
    da.k_cache = k_cache;
    da.v_cache = v_cache;
    da.cap = cache_capacity;
    da.out = out;
    da.partial = static_cast<float *>(workspace);
    da.max_splits = mimo::decode_max_splits(L, MIMO_ATTN_BF16, cache_capacity);
    da.chunk = mimo::decode_chunk_keys(L, MIMO_ATTN_BF16);
    da.B = batch;
    da.err = err;
    da.fp8_cache = 1;
    da.k_scale = k_scale;
    da.v_scale = v_scale;
    cudaError_t e = mimo::launch_decode(L, da, MIMO_ATTN_BF16, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MIMO_ATTN_OK : MIMO_ATTN_ERR_CUDA;
}

mimo_attn_status mimo_attn_quantize_fp8(const void *src, void *dst, size_t n, float scale, void *stream)
{
    if (!(scale > 0.f) || !isfinite(scale))
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (n == 0)
        return MIMO_ATTN_OK;
    if (src == nullptr || dst == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    if (g_fail_launches)
        return MIMO_ATTN_ERR_CUDA;
    return mimo::launch_quantize_e4m3(src, dst, n, scale, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MIMO_ATTN_OK
               : MIMO_ATTN_ERR_CUDA;
}

mimo_attn_status mimo_attn_get_device_error(uint32_t *bits)
{
    if (bits == nullptr)
        return MIMO_ATTN_ERR_INVALID_ARG;
    unsigned host = 0;
    const unsigned zero = 0;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyFromSymbol(&host, g_device_status, sizeof(host), offsetof(mimo::DeviceStatus, error)) !=
            cudaSuccess ||
        cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero), offsetof(mimo::DeviceStatus, error)) !=
            cudaSuccess)
        return MIMO_ATTN_ERR_CUDA;
    *bits = host;
    return MIMO_ATTN_OK;
}

mimo_attn_status mimo_attn_debug_set_wait_limit(long long cycles)
{
    const long long v = cycles > 0 ? cycles : 0;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyToSymbol(g_device_status, &v, sizeof(v), offsetof(mimo::DeviceStatus, wait_limit)) !=
            cudaSuccess)
        return MIMO_ATTN_ERR_CUDA;
    return MIMO_ATTN_OK;
}

mimo_attn_status mimo_attn_debug_wait_probe(void *stream)
{
    if (g_fail_launches)
        return MIMO_ATTN_ERR_CUDA;
    unsigned *err = device_error_ptr();
    if (err == nullptr)
        return MIMO_ATTN_ERR_CUDA;
    return mimo::launch_wait_probe(err, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MIMO_ATTN_OK
                                                                                           : MIMO_ATTN_ERR_CUDA;
}

const char *mimo_attn_status_string(mimo_attn_status status)
{
    switch (status) {
    case MIMO_ATTN_OK:
        return "ok";
    case MIMO_ATTN_ERR_INVALID_ARG:
        return "invalid argument";
    case MIMO_ATTN_ERR_UNSUPPORTED:
        return "unsupported configuration";
    case MIMO_ATTN_ERR_WORKSPACE:
        return "workspace missing or too small";
    case MIMO_ATTN_ERR_CUDA:
        return "CUDA error";
    }
    return "unknown status";
}

void mimo_attn_debug_fail_launches(int enable) { g_fail_launches = enable != 0; }

const char *mimo_attn_version(void) { return "mimo_attn 0.1.0 (sm_100a)"; }

} // extern "C"

// ------------------------------------------------------ decode without allocation
// mimo_attn_decode_static keeps the split-KV partial results in this
// file-scope device array instead of a caller workspace, for callers that
// cannot allocate device memory. The array is part of the library's device
// image: every GPU that loads the library holds these 16 MiB until the
// process exits. Every call shares it and it keeps the previous call's
// contents; nothing in it needs to start at zero, because each call writes
// every partial it later reads. Calls whose kernels overlap on the GPU (other
// streams, other host threads) race on it.
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;
static __device__ __align__(256) float g_decode_scratch[kStaticScratchBytes / sizeof(float)];

float *g_scratch_ptr[kMaxDevices];

// Device address of g_decode_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
float *static_scratch_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_symbol_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        float *ptr = nullptr;
        if (cudaGetSymbolAddress((void **)&ptr, g_decode_scratch) != cudaSuccess)
            return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

} // namespace

extern "C" mimo_attn_status mimo_attn_decode_static(const mimo_attn_layer *layer, int dtype, int batch,
                                                    const void *q, const void *k_new, const void *v_new,
                                                    const int32_t *kv_lens, void *k_cache, void *v_cache,
                                                    int cache_capacity, void *out, void *stream)
{
    const size_t need = mimo_attn_decode_workspace_size(layer, dtype, batch, cache_capacity);
    if (need > kStaticScratchBytes)
        return MIMO_ATTN_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0) {  // a valid layer that splits the keys: partials go to the array
        if (g_fail_launches)
            return MIMO_ATTN_ERR_CUDA;
        scratch = static_scratch_ptr();
        if (scratch == nullptr)
            return MIMO_ATTN_ERR_CUDA;
    }
    return mimo_attn_decode(layer, dtype, batch, q, k_new, v_new, kv_lens, k_cache, v_cache,
                            cache_capacity, out, scratch, need, stream);
}
