// Preparation of a prefill that continues a cache (a chunk of S new tokens
// after past_lens[b] cached ones): the chunk's keys are rotated at their
// positions and its keys and values are put where the attention kernels read
// them. See CachedPrepArgs in kernels.cuh.
//
// Global layers: the linear cache holds position p in row p, so the chunk is
// written into rows past + t and the attention reads the cache itself.
//
// Sliding layers: the ring holds only the last `window` positions and the
// chunk may overwrite slots its own first queries still need, so the keys a
// query can see are first gathered into a window in the workspace, row u =
// position past - key_off + u: rows before position 0, or too old for any of
// the chunk's queries, are zero (never visible); older rows come from the
// ring, the chunk's own rows are rotated here. A second kernel then stores the
// chunk's last `window` tokens into the ring.
#include "kernels.cuh"

namespace mimo {
namespace {

// One warp rotates one key row (partial RoPE, cos/sin from the table row of
// its position) from src into dst.
template <typename T>
__device__ __forceinline__ void rotate_row(const T *src, T *dst, int Dqk, int rotary_dim, int half,
                                           const float2 *cs, int lane)
{
    for (int e = lane; e < Dqk; e += 32) {
        float y;
        if (e < rotary_dim) {
            const int j = e < half ? e : e - half;
            const float2 c = __ldg(cs + j);
            const float xa = to_f32<T>(src[j]);
            const float xb = to_f32<T>(src[j + half]);
            y = e < half ? xa * c.x - xb * c.y : xb * c.x + xa * c.y;
        } else {
            y = to_f32<T>(src[e]);
        }
        dst[e] = from_f32<T>(y);
    }
}

template <typename T>
__device__ __forceinline__ void copy_row(const T *src, T *dst, int n, int lane)
{
    for (int e = lane; e < n; e += 32)
        dst[e] = src[e];
}

template <typename T>
__device__ __forceinline__ void zero_row(T *dst, int n, int lane)
{
    for (int e = lane; e < n; e += 32)
        dst[e] = from_f32<T>(0.f);
}

// Global layers: one warp per chunk row (b, t, kv head) -> cache row past + t.
template <typename T>
__global__ void cached_global_kernel(const __grid_constant__ CachedPrepArgs a)
{
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (long long)a.B * a.S * a.Hkv)
        return;
    const int kvh = (int)(w % a.Hkv);
    const long long bt = w / a.Hkv;  // b * S + t
    const int t = (int)(bt % a.S);
    const int b = (int)(bt / a.S);
    const int past = __ldg(a.past_lens + b);
    if (past < 0 || past > a.max_past || past + a.S > a.cap) {
        if (lane == 0 && t == 0 && kvh == 0)
            atomicOr(a.err, kErrKvLen);
        return;
    }
    const int pos = past + t;
    const size_t dst_row = ((size_t)b * a.cap + pos) * a.Hkv + kvh;
    rotate_row<T>(reinterpret_cast<const T *>(a.k) + (size_t)w * a.Dqk,
                  reinterpret_cast<T *>(a.k_cache) + dst_row * a.Dqk, a.Dqk, a.rope.rotary_dim, a.rope.half,
                  a.rope_table + (size_t)pos * a.rope.half, lane);
    copy_row<T>(reinterpret_cast<const T *>(a.v) + (size_t)w * a.Dv,
                reinterpret_cast<T *>(a.v_cache) + dst_row * a.Dv, a.Dv, lane);
}

// Sliding layers: one warp per window row (b, u, kv head).
template <typename T>
__global__ void cached_swa_gather_kernel(const __grid_constant__ CachedPrepArgs a)
{
    const int n_rows = a.key_off + a.S;
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (long long)a.B * n_rows * a.Hkv)
        return;
    const int kvh = (int)(w % a.Hkv);
    const long long bu = w / a.Hkv;  // b * n_rows + u
    const int u = (int)(bu % n_rows);
    const int b = (int)(bu / n_rows);
    int past = __ldg(a.past_lens + b);
    if (past < 0 || past > a.max_past) {
        if (lane == 0 && u == 0 && kvh == 0)
            atomicOr(a.err, kErrKvLen);
        past = min(max(past, 0), a.max_past);
    }
    const int pos = past - a.key_off + u;
    T *kd = reinterpret_cast<T *>(a.kv_k) + (size_t)w * a.Dqk;
    T *vd = reinterpret_cast<T *>(a.kv_v) + (size_t)w * a.Dv;
    if (pos < max(0, past - (a.window - 1))) {
        zero_row<T>(kd, a.Dqk, lane);
        zero_row<T>(vd, a.Dv, lane);
    } else if (pos < past) {
        const size_t src_row = ((size_t)b * a.window + pos % a.window) * a.Hkv + kvh;
        copy_row<T>(reinterpret_cast<const T *>(a.k_cache) + src_row * a.Dqk, kd, a.Dqk, lane);
        copy_row<T>(reinterpret_cast<const T *>(a.v_cache) + src_row * a.Dv, vd, a.Dv, lane);
    } else {
        const size_t src_row = ((size_t)b * a.S + (pos - past)) * a.Hkv + kvh;
        rotate_row<T>(reinterpret_cast<const T *>(a.k) + src_row * a.Dqk, kd, a.Dqk, a.rope.rotary_dim,
                      a.rope.half, a.rope_table + (size_t)pos * a.rope.half, lane);
        copy_row<T>(reinterpret_cast<const T *>(a.v) + src_row * a.Dv, vd, a.Dv, lane);
    }
}

// Sliding layers, after the gather: the chunk's last `window` tokens (distinct
// slots) go into the ring.
template <typename T>
__global__ void cached_swa_ring_kernel(const __grid_constant__ CachedPrepArgs a)
{
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (long long)a.B * a.S * a.Hkv)
        return;
    const int kvh = (int)(w % a.Hkv);
    const long long bt = w / a.Hkv;
    const int t = (int)(bt % a.S);
    const int b = (int)(bt / a.S);
    if (t < a.S - a.window)
        return;  // a later token of the chunk takes this slot
    const int past = min(max(__ldg(a.past_lens + b), 0), a.max_past);
    const size_t src_row = ((size_t)b * (a.key_off + a.S) + a.key_off + t) * a.Hkv + kvh;
    const size_t dst_row = ((size_t)b * a.window + (past + t) % a.window) * a.Hkv + kvh;
    copy_row<T>(reinterpret_cast<const T *>(a.kv_k) + src_row * a.Dqk,
                reinterpret_cast<T *>(a.k_cache) + dst_row * a.Dqk, a.Dqk, lane);
    copy_row<T>(reinterpret_cast<const T *>(a.kv_v) + src_row * a.Dv,
                reinterpret_cast<T *>(a.v_cache) + dst_row * a.Dv, a.Dv, lane);
}

template <typename T> cudaError_t launch_typed(const CachedPrepArgs &a, cudaStream_t stream)
{
    constexpr int kThreads = 256;
    auto grid = [](long long rows) { return (unsigned)((rows * 32 + kThreads - 1) / kThreads); };
    const long long chunk_rows = (long long)a.B * a.S * a.Hkv;
    if (a.layer_type == 0) {
        cached_global_kernel<T><<<grid(chunk_rows), kThreads, 0, stream>>>(a);
    } else {
        cached_swa_gather_kernel<T><<<grid((long long)a.B * (a.key_off + a.S) * a.Hkv), kThreads, 0, stream>>>(a);
        cached_swa_ring_kernel<T><<<grid(chunk_rows), kThreads, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_cached_prep(const CachedPrepArgs &a, int dtype, cudaStream_t stream)
{
    if ((long long)a.B * a.S * a.Hkv == 0)
        return cudaSuccess;
    return dtype == kDtypeBf16 ? launch_typed<__nv_bfloat16>(a, stream) : launch_typed<float>(a, stream);
}

} // namespace mimo
