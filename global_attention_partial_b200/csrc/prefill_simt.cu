// Key preparation and the CUDA-core prefill path of the MiMo-V2-Flash layer.
//
// kprep: builds the RoPE cos/sin table of every (position, pair) once, then
// rotates every key at its token's position (fp32 arithmetic on the table's
// values, angles formed in double precision) once per layer, and writes it where
// the attention kernels read it (the global cache itself, or a workspace),
// plus the caches: the global value cache, or the sliding-window ring (slot
// i mod window for the last `window` tokens). Rotating K once per layer,
// rather than once per (query tile, key tile) pair, keeps the rotation off
// the attention kernels' inner loop.
//
// prefill_simt: one warp per query row on CUDA cores, fp32 arithmetic; the
// path for fp32 inputs and for head dims the tensor-core kernel does not
// take.
#include "kernels.cuh"

#include <math.h>

namespace mimo {
namespace {

// cos / sin of every (position, pair): table[i][j] for pair j of token i.
// The inverse frequencies are staged in shared memory, so lanes that need
// different pairs never serialise on the kernel-parameter bank.
__global__ void rope_table_kernel(const __grid_constant__ KprepArgs a)
{
    __shared__ double inv_freq[kMaxHalfRotary];
    const int half = a.rope.half;
    for (int j = threadIdx.x; j < half; j += blockDim.x)
        inv_freq[j] = a.rope.inv_freq[j];
    __syncthreads();
    const long long total = (long long)a.S * half;
    for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < total;
         u += (long long)gridDim.x * blockDim.x) {
        const int i = (int)(u / half);
        const int j = (int)(u - (long long)i * half);
        const double pos = a.positions ? (double)__ldg(a.positions + i) : (double)i;
        float c, s;
        rope_cos_sin(pos, inv_freq[j], c, s);
        a.rope_table[u] = make_float2(c, s);
    }
}

// One warp per key row (b, i, kv); any dims / dtype. Reads cos/sin from the table.
template <typename T>
__global__ void kprep_kernel(const __grid_constant__ KprepArgs a)
{
    const int warps = blockDim.x >> 5;
    const long long row = (long long)blockIdx.x * warps + (threadIdx.x >> 5);
    const long long total = (long long)a.B * a.S * a.Hkv;
    if (row >= total)
        return;
    const int lane = threadIdx.x & 31;
    const int kv = (int)(row % a.Hkv);
    const long long bi = row / a.Hkv;
    const int i = (int)(bi % a.S);
    const int b = (int)(bi / a.S);
    const int half = a.rope.half;
    const float2 *cs = a.rope_table + (long long)i * half;
    const T *k = reinterpret_cast<const T *>(a.k) + row * a.Dqk;
    T *dk = reinterpret_cast<T *>(a.dst_k) + (((long long)b * a.dst_rows + i) * a.Hkv + kv) * a.Dqk;
    const bool to_ring = a.ring_k != nullptr && a.window > 0 && i >= a.S - a.window;
    const long long ring_off = to_ring ? ((long long)b * a.window + i % a.window) * a.Hkv + kv : 0;
    T *rk = to_ring ? reinterpret_cast<T *>(a.ring_k) + ring_off * a.Dqk : nullptr;
    for (int e = lane; e < a.Dqk; e += 32) {
        float y;
        if (e < a.rope.rotary_dim) {
            const int j = e < half ? e : e - half;
            const float2 c = __ldg(cs + j);
            const float xa = to_f32<T>(k[j]);
            const float xb = to_f32<T>(k[j + half]);
            y = e < half ? xa * c.x - xb * c.y : xb * c.x + xa * c.y;
        } else {
            y = to_f32<T>(k[e]);
        }
        const T yt = from_f32<T>(y);
        dk[e] = yt;
        if (rk)
            rk[e] = yt;
    }
    T *rv = to_ring ? reinterpret_cast<T *>(a.ring_v) + ring_off * a.Dv : nullptr;
    T *lv = a.lin_v ? reinterpret_cast<T *>(a.lin_v) + (((long long)b * a.lin_rows + i) * a.Hkv + kv) * a.Dv
                    : nullptr;
    if (rv || lv) {
        const T *v = reinterpret_cast<const T *>(a.v) + row * a.Dv;
        for (int e = lane; e < a.Dv; e += 32) {
            const T x = v[e];
            if (rv)
                rv[e] = x;
            if (lv)
                lv[e] = x;
        }
    }
}

// The sliding-window ring only: one warp per (b, token, kv) row of the last
// min(S, window) tokens; rotates the key (table values) into ring slot
// i mod window and copies the value. Used when the attention kernel rotates
// the keys itself, so no other key copy is written.
template <typename T>
__global__ void kprep_ring_kernel(const __grid_constant__ KprepArgs a)
{
    const int warps = blockDim.x >> 5;
    const long long row = (long long)blockIdx.x * warps + (threadIdx.x >> 5);
    const int nring = a.S < a.window ? a.S : a.window;
    const long long total = (long long)a.B * nring * a.Hkv;
    if (row >= total)
        return;
    const int lane = threadIdx.x & 31;
    const int kv = (int)(row % a.Hkv);
    const long long br = row / a.Hkv;
    const int i = a.S - nring + (int)(br % nring);
    const int b = (int)(br / nring);
    const int half = a.rope.half;
    const float2 *cs = a.rope_table + (long long)i * half;
    const long long src = ((long long)b * a.S + i) * a.Hkv + kv;
    const long long dst = ((long long)b * a.window + i % a.window) * a.Hkv + kv;
    const T *k = reinterpret_cast<const T *>(a.k) + src * a.Dqk;
    T *rk = reinterpret_cast<T *>(a.ring_k) + dst * a.Dqk;
    for (int e = lane; e < a.Dqk; e += 32) {
        float y;
        if (e < a.rope.rotary_dim) {
            const int j = e < half ? e : e - half;
            const float2 c = __ldg(cs + j);
            const float xa = to_f32<T>(k[j]);
            const float xb = to_f32<T>(k[j + half]);
            y = e < half ? xa * c.x - xb * c.y : xb * c.x + xa * c.y;
        } else {
            y = to_f32<T>(k[e]);
        }
        rk[e] = from_f32<T>(y);
    }
    const T *v = reinterpret_cast<const T *>(a.v) + src * a.Dv;
    T *rv = reinterpret_cast<T *>(a.ring_v) + dst * a.Dv;
    for (int e = lane; e < a.Dv; e += 32)
        rv[e] = v[e];
}

// bf16 rows in 16-byte units (8 elements): a lane takes either a pair of
// rotary chunks (c, c + half/8), a pass-through K chunk, or a V chunk.
// Needs rotary_dim % 16 == 0, Dqk % 8 == 0, Dv % 8 == 0.
__global__ void kprep_bf16_vec_kernel(const __grid_constant__ KprepArgs a)
{
    const int warps = blockDim.x >> 5;
    const long long row = (long long)blockIdx.x * warps + (threadIdx.x >> 5);
    const long long total = (long long)a.B * a.S * a.Hkv;
    if (row >= total)
        return;
    const int lane = threadIdx.x & 31;
    const int kv = (int)(row % a.Hkv);
    const long long bi = row / a.Hkv;
    const int i = (int)(bi % a.S);
    const int b = (int)(bi / a.S);
    const int npair = a.rope.half / 8;
    const int ncopy = (a.Dqk - a.rope.rotary_dim) / 8;
    const bool with_v = a.ring_v != nullptr || a.lin_v != nullptr;
    const int nv = with_v ? a.Dv / 8 : 0;
    const bool to_ring = a.ring_k != nullptr && a.window > 0 && i >= a.S - a.window;
    const long long ring_off = to_ring ? ((long long)b * a.window + i % a.window) * a.Hkv + kv : 0;
    const uint4 *k = reinterpret_cast<const uint4 *>(a.k) + row * (a.Dqk / 8);
    uint4 *dk = reinterpret_cast<uint4 *>(a.dst_k) + (((long long)b * a.dst_rows + i) * a.Hkv + kv) * (a.Dqk / 8);
    uint4 *rk = to_ring ? reinterpret_cast<uint4 *>(a.ring_k) + ring_off * (a.Dqk / 8) : nullptr;
    for (int u = lane; u < npair + ncopy + nv; u += 32) {
        if (u < npair) {
            const uint4 xa = __ldg(k + u);
            const uint4 xb = __ldg(k + u + npair);
            const float4 *cs = reinterpret_cast<const float4 *>(a.rope_table + (long long)i * a.rope.half + u * 8);
            const uint32_t *pa = reinterpret_cast<const uint32_t *>(&xa);
            const uint32_t *pb = reinterpret_cast<const uint32_t *>(&xb);
            uint4 ya, yb;
            uint32_t *qa = reinterpret_cast<uint32_t *>(&ya);
            uint32_t *qb = reinterpret_cast<uint32_t *>(&yb);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 c = __ldg(cs + w);  // (cos, sin) of pairs 8u+2w and 8u+2w+1
                const float2 va = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pa[w]));
                const float2 vb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pb[w]));
                qa[w] = pack_bf16x2(va.x * c.x - vb.x * c.y, va.y * c.z - vb.y * c.w);
                qb[w] = pack_bf16x2(vb.x * c.x + va.x * c.y, vb.y * c.z + va.y * c.w);
            }
            dk[u] = ya;
            dk[u + npair] = yb;
            if (rk) {
                rk[u] = ya;
                rk[u + npair] = yb;
            }
        } else if (u < npair + ncopy) {
            const int c = 2 * npair + (u - npair);
            const uint4 x = __ldg(k + c);
            dk[c] = x;
            if (rk)
                rk[c] = x;
        } else {
            const int c = u - npair - ncopy;
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(a.v) + row * (a.Dv / 8) + c);
            if (to_ring)
                reinterpret_cast<uint4 *>(a.ring_v)[ring_off * (a.Dv / 8) + c] = x;
            if (a.lin_v)
                reinterpret_cast<uint4 *>(a.lin_v)[(((long long)b * a.lin_rows + i) * a.Hkv + kv) * (a.Dv / 8) + c] = x;
        }
    }
}

// K rows of 192 bf16 (24 chunks of 16 bytes) with rotary_dim 64, rotated
// into dst_k only (no cache copies): the rows are one flat array of chunks,
// 32 consecutive chunks per warp, four per thread in flight. A row starts at
// a multiple of 8 chunks, so its 8 rotary chunks (dims 0-63: chunk c < 4
// pairs with c + 4) sit in one aligned group of 8 lanes and a lane gets its
// partner chunk from lane ^ 4 by shuffle.
constexpr int kKprepChunks = 24;
constexpr int kKprepUnroll = 4;
__global__ void kprep_r64_kernel(const __grid_constant__ KprepArgs a)
{
    const long long total = (long long)a.B * a.S * a.Hkv * kKprepChunks;
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.k);
    uint4 *dst = reinterpret_cast<uint4 *>(a.dst_k);
    for (long long w = warp0 * kKprepUnroll; w * 32 < total; w += nwarps * kKprepUnroll) {
        uint4 x[kKprepUnroll];
#pragma unroll
        for (int u = 0; u < kKprepUnroll; ++u) {
            const long long g = (w + u) * 32 + lane;
            x[u] = g < total ? __ldg(src + g) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kKprepUnroll; ++u) {
            const long long g = (w + u) * 32 + lane;
            const long long row = g / kKprepChunks;
            const int c = (int)(g - row * kKprepChunks);
            // partner chunk of the rotary half (meaningful for c < 8 only);
            // every lane takes part in the shuffles
            uint4 y;
            y.x = __shfl_xor_sync(0xffffffffu, x[u].x, 4);
            y.y = __shfl_xor_sync(0xffffffffu, x[u].y, 4);
            y.z = __shfl_xor_sync(0xffffffffu, x[u].z, 4);
            y.w = __shfl_xor_sync(0xffffffffu, x[u].w, 4);
            if (g >= total)
                continue;
            const long long bi = row / a.Hkv;
            const int i = (int)(bi % a.S);
            const int b = (int)(bi / a.S);
            const int kv = (int)(row - bi * a.Hkv);
            uint4 out = x[u];
            if (c < 8) {
                const bool first = c < 4;
                // own dims are 8c.. (first half) or 32 + 8(c-4).. (second half):
                // pairs 8(c & 3) .. 8(c & 3) + 7
                const float4 *cs = reinterpret_cast<const float4 *>(a.rope_table + (long long)i * 32 + (c & 3) * 8);
                const uint32_t *own = reinterpret_cast<const uint32_t *>(&x[u]);
                const uint32_t *oth = reinterpret_cast<const uint32_t *>(&y);
                uint32_t *o = reinterpret_cast<uint32_t *>(&out);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 cc = __ldg(cs + e);  // (cos, sin) of pairs 2e and 2e + 1 of the chunk
                    const float2 xa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(first ? &own[e] : &oth[e]));
                    const float2 xb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(first ? &oth[e] : &own[e]));
                    o[e] = first ? pack_bf16x2(xa.x * cc.x - xb.x * cc.y, xa.y * cc.z - xb.y * cc.w)
                                 : pack_bf16x2(xb.x * cc.x + xa.x * cc.y, xb.y * cc.z + xa.y * cc.w);
                }
            }
            dst[(((long long)b * a.dst_rows + i) * a.Hkv + kv) * kKprepChunks + c] = out;
        }
    }
}

template <typename T>
__global__ void prefill_simt_kernel(const __grid_constant__ LayerArgs L, const __grid_constant__ PrefillArgs a)
{
    __shared__ float qs[4][256];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * 4 + warp;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    if (i >= a.S)
        return;
    // Query i is the token at position past + i and key index past + i
    // (global) or swa_key_off + i (sliding window); past = 0 for a plain prefill.
    const int past = a.past_lens != nullptr ? min(max(__ldg(a.past_lens + b), 0), a.max_past) : 0;
    const int key_off = a.past_lens == nullptr ? 0 : (L.layer_type == 1 ? a.swa_key_off : past);
    const int ki = i + key_off;
    if (ki >= a.key_rows_valid)  // out-of-range past_lens: reported by the cache prep
        return;
    const int half = L.rope.half;
    const float2 *cs = a.rope_table + (size_t)(past + i) * half;
    const T *q = reinterpret_cast<const T *>(a.q) + (((size_t)b * a.S + i) * L.Hq + h) * L.Dqk;
    for (int e = lane; e < L.Dqk; e += 32) {
        float y;
        if (e < L.rope.rotary_dim) {
            const int j = e < half ? e : e - half;
            const float2 c = __ldg(cs + j);
            const float xa = to_f32<T>(q[j]);
            const float xb = to_f32<T>(q[j + half]);
            y = e < half ? xa * c.x - xb * c.y : xb * c.x + xa * c.y;
        } else {
            y = to_f32<T>(q[e]);
        }
        qs[warp][e] = y;
    }
    __syncwarp();
    const int kvh = h / L.G;
    const int lo = L.layer_type == 1 ? max(max(0, key_off - past), ki - L.window + 1) : 0;
    float m = -INFINITY, l = 0.f;
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t)
        acc[t] = 0.f;
    for (int j = lo; j <= ki; ++j) {
        const T *kr = reinterpret_cast<const T *>(a.krot) + (((size_t)b * a.krot_rows + j) * L.Hkv + kvh) * L.Dqk;
        float part = 0.f;
        for (int e = lane; e < L.Dqk; e += 32)
            part += qs[warp][e] * to_f32<T>(kr[e]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            part += __shfl_xor_sync(0xffffffffu, part, off);
        const float x = part * L.scale_log2;
        const float mn = fmaxf(m, x);
        const float c = (m == -INFINITY) ? 0.f : exp2f(m - mn);
        const float pj = exp2f(x - mn);
        l = l * c + pj;
        const T *vr = reinterpret_cast<const T *>(a.v) + (((size_t)b * a.v_rows + j) * L.Hkv + kvh) * L.Dv;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int e = lane + 32 * t;
            if (e < L.Dv)
                acc[t] = acc[t] * c + pj * to_f32<T>(vr[e]);
        }
        m = mn;
    }
    float scale;
    if (L.sinks != nullptr) {
        const float s2 = __ldg(L.sinks + h) * kLog2e;
        const float mf = fmaxf(m, s2);
        const float al = exp2f(m - mf);
        scale = al * L.v_scale / (l * al + exp2f(s2 - mf));
    } else {
        scale = L.v_scale / l;
    }
    T *dst = reinterpret_cast<T *>(a.out) + (((size_t)b * a.S + i) * L.Hq + h) * L.Dv;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const int e = lane + 32 * t;
        if (e < L.Dv)
            dst[e] = from_f32<T>(acc[t] * scale);
    }
}

} // namespace

cudaError_t launch_kprep(const KprepArgs &a, int dtype, cudaStream_t stream)
{
    const long long rows = (long long)a.B * a.S * a.Hkv;
    if (rows == 0)
        return cudaSuccess;
    if (a.rope.half > 0) {
        const long long entries = (long long)a.S * a.rope.half;
        const long long tb = (entries + 255) / 256;
        rope_table_kernel<<<(unsigned)(tb < 4096 ? tb : 4096), 256, 0, stream>>>(a);
    }
    const int threads = 256;
    if (dtype == kDtypeBf16 && a.rope.rotary_dim == 64 && a.Dqk == 192 && a.ring_k == nullptr &&
        a.ring_v == nullptr && a.lin_v == nullptr) {
        const long long warps = (rows * kKprepChunks + 32 * kKprepUnroll - 1) / (32 * kKprepUnroll);
        const long long need = (warps + threads / 32 - 1) / (threads / 32);
        const long long cap = 148LL * 16;  // grid-stride beyond 16 blocks per SM
        kprep_r64_kernel<<<(unsigned)(need < cap ? need : cap), threads, 0, stream>>>(a);
        return cudaGetLastError();
    }
    const long long blocks = (rows + (threads / 32) - 1) / (threads / 32);
    const bool vec = dtype == kDtypeBf16 && a.rope.rotary_dim % 16 == 0 && a.Dqk % 8 == 0 && a.Dv % 8 == 0 &&
                     (a.rope.half / 8) + (a.Dqk - a.rope.rotary_dim) / 8 + a.Dv / 8 <= 32 * 64;
    if (vec)
        kprep_bf16_vec_kernel<<<(unsigned)blocks, threads, 0, stream>>>(a);
    else if (dtype == kDtypeBf16)
        kprep_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, stream>>>(a);
    else
        kprep_kernel<float><<<(unsigned)blocks, threads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_kprep_ring(const KprepArgs &a, int dtype, cudaStream_t stream)
{
    const int nring = a.S < a.window ? a.S : a.window;
    const long long rows = (long long)a.B * nring * a.Hkv;
    if (rows == 0)
        return cudaSuccess;
    const int threads = 256;
    const long long blocks = (rows + (threads / 32) - 1) / (threads / 32);
    if (dtype == kDtypeBf16)
        kprep_ring_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, stream>>>(a);
    else
        kprep_ring_kernel<float><<<(unsigned)blocks, threads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_rope_table(const RopeArgs &rope, float2 *table, long long n, cudaStream_t stream,
                              const int *positions)
{
    if (rope.half == 0 || n == 0)
        return cudaSuccess;
    KprepArgs a;
    memset(&a, 0, sizeof(a));
    a.S = (int)n;
    a.positions = positions;
    a.rope_table = table;
    a.rope = rope;
    const long long tb = (n * rope.half + 255) / 256;
    rope_table_kernel<<<(unsigned)(tb < 4096 ? tb : 4096), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_prefill_simt(const LayerArgs &L, const PrefillArgs &a, int dtype, cudaStream_t stream)
{
    dim3 grid((a.S + 3) / 4, L.Hq, a.B);
    if (dtype == kDtypeBf16)
        prefill_simt_kernel<__nv_bfloat16><<<grid, 128, 0, stream>>>(L, a);
    else
        prefill_simt_kernel<float><<<grid, 128, 0, stream>>>(L, a);
    return cudaGetLastError();
}

} // namespace mimo
