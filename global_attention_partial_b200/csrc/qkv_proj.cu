// QKV projection of one MiMo-V2-Flash attention layer with its epilogue
// fused: y = x W^T on the tcgen05 tensor cores (bf16 operands staged by TMA,
// fp32 accumulators in TMEM), then, per 64-column block of y, the layer's
// partial RoPE on query and key heads at the token's position, bf16 rounding
// and the stores to q / k / v and to the key and value caches. The pages'
// attention ("Add Xiaomi MiMo-V2", "Additional useful info": partial RoPE,
// decoupled V head dim, per-layer KV heads) starts from these tensors.
//
// Persistent kernel, one CTA per SM, 192 threads:
//   warp 0      TMA producer: x tile 128 tokens x 64 hidden (16 KB) and W tile
//               256 features x 64 hidden (32 KB) per stage, 4-stage ring;
//   warp 1      allocates 512 TMEM columns; one lane issues the MMAs
//               (128 x 256 x 16, four per stage) into one of two 256-column
//               accumulators and commits stage and tile completions;
//   warps 2-5   epilogue: thread r owns token row r of the tile (TMEM lane
//               r), drains one accumulator while the MMAs fill the other.
// Tiles are rastered in groups of 16 token tiles that sweep every feature
// tile together, so the x rows and the W rows a wave reads stay in L2.
#include "kernels.cuh"

namespace mimo {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBN * kBK * 2;
constexpr int kThreads = 192;
constexpr int kTmemCols = 2 * kBN;
constexpr int kGroupM = 16;

struct QkvBars {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint32_t tmem_base;
    int abort;
};

constexpr int kSmemBytes = 1024 + kStages * (kABytes + kBBytes) + (int)sizeof(QkvBars) + 64;
static_assert(kSmemBytes <= 232448, "shared memory");

struct QkvParams {
    CUtensorMap tm_x;  // [T, hidden]  box {64, 128}
    CUtensorMap tm_w;  // [N, hidden]  box {64, 256}
    int T, S, kblocks, n_total, tiles_m, tiles_n;
    int Hq, Hkv, Dqk, Dv, n_q, n_k;
    int rotate;        // rotary_dim == 64: pairs (j, j + 32) of each head's first 64 columns
    int layer_type, window, cap, max_past;
    const int *past_lens;        // nullptr: position = sequence index
    const float2 *rope_table;    // [max_past + S][32] (cos, sin)
    __nv_bfloat16 *q, *k, *v;    // k, v may be null
    __nv_bfloat16 *k_cache, *v_cache;  // both or neither
    int v8;                      // every destination is 32-byte aligned
    unsigned *err;
};

__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int &m, int &n)
{
    const int per_group = kGroupM * tiles_n;
    const int g = tile / per_group;
    const int first_m = g * kGroupM;
    const int gm = min(kGroupM, tiles_m - first_m);
    const int r = tile - g * per_group;
    m = first_m + r % gm;
    n = r / gm;
}

// 64 fp32 values (w0: columns 0-31, w1: 32-63) to 32 bf16x2 words.
__device__ __forceinline__ void pack_block(const uint32_t (&w0)[32], const uint32_t (&w1)[32], uint32_t (&o)[32])
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        o[i] = pack_bf16x2(__uint_as_float(w0[2 * i]), __uint_as_float(w0[2 * i + 1]));
        o[16 + i] = pack_bf16x2(__uint_as_float(w1[2 * i]), __uint_as_float(w1[2 * i + 1]));
    }
}

__device__ __forceinline__ void store_block(__nv_bfloat16 *dst, const uint32_t (&o)[32], bool v8)
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w[i] = o[c * 8 + i];
        st_global_32B(dst + c * 16, w, v8);
    }
}

__global__ void __launch_bounds__(kThreads, 1) qkv_proj_kernel(const __grid_constant__ QkvParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * kABytes;
    QkvBars *bars = reinterpret_cast<QkvBars *>(sB + kStages * kBBytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&bars->acc_full[a], 1);
            mbar_init(&bars->acc_empty[a], 128);
        }
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort = &bars->abort;
    const int total = p.tiles_m * p.tiles_n;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_x);
            tma_prefetch_desc(&p.tm_w);
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                int m, n;
                tile_coords(tile, p.tiles_m, p.tiles_n, m, n);
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    const int s = it % kStages;
                    if (!mbar_wait(&bars->empty[s], ((it / kStages) & 1) ^ 1, abort, p.err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->full[s], kABytes + kBBytes);
                    tma_load_4d(sA + s * kABytes, &p.tm_x, &bars->full[s], kb * kBK, m * kBM, 0, 0);
                    tma_load_4d(sB + s * kBBytes, &p.tm_w, &bars->full[s], kb * kBK, n * kBN, 0, 0);
                    ++it;
                }
            }
            // The CTA never exits under a load: wait for the last armed
            // stage loads (already complete on the normal path).
            for (uint32_t j = it > (uint32_t)kStages ? it - kStages : 0; j < it; ++j)
                mbar_drain(&bars->full[j % kStages], (j / kStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kBM, kBN, false, false);
            const uint32_t a_lo = sdesc_lo(smem_u32(sA), 16);
            const uint32_t b_lo = sdesc_lo(smem_u32(sB), 16);
            uint32_t it = 0;
            int lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++lt) {
                const int a = lt & 1;
                if (!mbar_wait(&bars->acc_empty[a], ((lt >> 1) & 1) ^ 1, abort, p.err))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(a * kBN);
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    const int s = it % kStages;
                    if (!mbar_wait(&bars->full[s], (it / kStages) & 1, abort, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ab = a_lo + (uint32_t)s * (kABytes >> 4);
                    const uint32_t bb = b_lo + (uint32_t)s * (kBBytes >> 4);
                    umma_ss_lo(d, ab, bb, idesc, kb > 0 ? 1u : 0u);
                    umma_ss_lo(d, ab + 2, bb + 2, idesc, 1u);
                    umma_ss_lo(d, ab + 4, bb + 4, idesc, 1u);
                    umma_ss_lo(d, ab + 6, bb + 6, idesc, 1u);
                    umma_commit(&bars->empty[s]);
                    ++it;
                }
                if (ok)
                    umma_commit(&bars->acc_full[a]);
            }
            // MMAs of one thread complete in order: the last stage commit
            // covers every MMA issued.
            if (it > 0)
                mbar_drain(&bars->empty[(it - 1) % kStages], ((it - 1) / kStages) & 1);
        }
    } else {
        const int q4 = warp & 3;  // TMEM lanes 32*q4 .. 32*q4+31
        const int row = q4 * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        const bool v8 = p.v8 != 0;
        int lt = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++lt) {
            int m, n;
            tile_coords(tile, p.tiles_m, p.tiles_n, m, n);
            const int a = lt & 1;
            if (!mbar_wait(&bars->acc_full[a], (lt >> 1) & 1, abort, p.err))
                break;
            tc_fence_after();
            const int t = m * kBM + row;
            bool valid = t < p.T;
            int b = 0, s = 0, pos = 0;
            if (valid) {
                b = t / p.S;
                s = t - b * p.S;
                const int past = p.past_lens ? __ldg(p.past_lens + b) : 0;
                if (past < 0 || past > p.max_past) {
                    if (n == 0)
                        atomicOr(p.err, kErrKvLen);
                    valid = false;
                }
                pos = past + s;
            }
            // the ring keeps only the chunk's last `window` tokens
            const bool to_cache = valid && p.k_cache != nullptr && (p.layer_type == 0 || s >= p.S - p.window);
            const int slot = p.layer_type == 1 ? pos % p.window : pos;
#pragma unroll 1
            for (int cb = 0; cb < kBN / 64; ++cb) {
                uint32_t w0[32], w1[32];
                tmem_ld32(lane_base + (uint32_t)(a * kBN + cb * 64), w0);
                tmem_ld32(lane_base + (uint32_t)(a * kBN + cb * 64 + 32), w1);
                tmem_wait_ld(w0);
                tmem_tie(w1);
                const int col = n * kBN + cb * 64;
                if (!valid || col >= p.n_total)
                    continue;
                int seg, head, off;
                if (col < p.n_q) {
                    seg = 0;
                    head = col / p.Dqk;
                    off = col - head * p.Dqk;
                } else if (col < p.n_q + p.n_k) {
                    seg = 1;
                    head = (col - p.n_q) / p.Dqk;
                    off = col - p.n_q - head * p.Dqk;
                } else {
                    seg = 2;
                    head = (col - p.n_q - p.n_k) / p.Dv;
                    off = col - p.n_q - p.n_k - head * p.Dv;
                }
                if (seg < 2 && off == 0 && p.rotate) {
                    const float4 *cs = reinterpret_cast<const float4 *>(p.rope_table + (size_t)pos * 32);
#pragma unroll
                    for (int j2 = 0; j2 < 16; ++j2) {
                        const float4 c = __ldg(cs + j2);  // pairs 2*j2 and 2*j2+1
                        const float xa0 = __uint_as_float(w0[2 * j2]), xb0 = __uint_as_float(w1[2 * j2]);
                        const float xa1 = __uint_as_float(w0[2 * j2 + 1]), xb1 = __uint_as_float(w1[2 * j2 + 1]);
                        w0[2 * j2] = __float_as_uint(xa0 * c.x - xb0 * c.y);
                        w1[2 * j2] = __float_as_uint(xb0 * c.x + xa0 * c.y);
                        w0[2 * j2 + 1] = __float_as_uint(xa1 * c.z - xb1 * c.w);
                        w1[2 * j2 + 1] = __float_as_uint(xb1 * c.z + xa1 * c.w);
                    }
                }
                uint32_t o[32];
                pack_block(w0, w1, o);
                if (seg == 0) {
                    store_block(p.q + ((size_t)t * p.Hq + head) * p.Dqk + off, o, v8);
                } else if (seg == 1) {
                    if (p.k)
                        store_block(p.k + ((size_t)t * p.Hkv + head) * p.Dqk + off, o, v8);
                    if (to_cache)
                        store_block(p.k_cache + (((size_t)b * p.cap + slot) * p.Hkv + head) * p.Dqk + off, o, v8);
                } else {
                    if (p.v)
                        store_block(p.v + ((size_t)t * p.Hkv + head) * p.Dv + off, o, v8);
                    if (to_cache)
                        store_block(p.v_cache + (((size_t)b * p.cap + slot) * p.Hkv + head) * p.Dv + off, o, v8);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->acc_empty[a]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

bool aligned32(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 31u) == 0; }

} // namespace

bool qkv_proj_supported(const LayerArgs &L, int hidden)
{
    return L.Dqk % 64 == 0 && L.Dv % 64 == 0 && hidden % kBK == 0 && hidden > 0 &&
           (L.rope.rotary_dim == 0 || L.rope.rotary_dim == 64);
}

cudaError_t launch_qkv_proj(const LayerArgs &L, const QkvArgs &a, int num_sms, cudaStream_t stream)
{
    const long long T = (long long)a.B * a.S;
    if (T == 0)
        return cudaSuccess;
    QkvParams p;
    memset(&p, 0, sizeof(p));
    const int n_total = L.Hq * L.Dqk + L.Hkv * (L.Dqk + L.Dv);
    if (!make_bf16_map_4d(&p.tm_x, a.x, a.hidden, T, 1, 1, 1, kBK, kBM, 1) ||
        !make_bf16_map_4d(&p.tm_w, a.w, a.hidden, n_total, 1, 1, 1, kBK, kBN, 1))
        return cudaErrorInvalidValue;
    if (L.rope.rotary_dim > 0) {
        cudaError_t e = launch_rope_table(L.rope, a.rope_table, (long long)a.max_past + a.S, stream);
        if (e != cudaSuccess)
            return e;
    }
    p.T = (int)T;
    p.S = a.S;
    p.kblocks = a.hidden / kBK;
    p.n_total = n_total;
    p.tiles_m = (int)((T + kBM - 1) / kBM);
    p.tiles_n = (n_total + kBN - 1) / kBN;
    p.Hq = L.Hq;
    p.Hkv = L.Hkv;
    p.Dqk = L.Dqk;
    p.Dv = L.Dv;
    p.n_q = L.Hq * L.Dqk;
    p.n_k = L.Hkv * L.Dqk;
    p.rotate = L.rope.rotary_dim == 64;
    p.layer_type = L.layer_type;
    p.window = L.window;
    p.cap = a.cap;
    p.max_past = a.max_past;
    p.past_lens = a.past_lens;
    p.rope_table = a.rope_table;
    p.q = reinterpret_cast<__nv_bfloat16 *>(a.q);
    p.k = reinterpret_cast<__nv_bfloat16 *>(a.k);
    p.v = reinterpret_cast<__nv_bfloat16 *>(a.v);
    p.k_cache = reinterpret_cast<__nv_bfloat16 *>(a.k_cache);
    p.v_cache = reinterpret_cast<__nv_bfloat16 *>(a.v_cache);
    p.v8 = aligned32(a.q) && aligned32(a.k) && aligned32(a.v) && aligned32(a.k_cache) && aligned32(a.v_cache);
    p.err = a.err;
    static std::atomic<unsigned long long> prepared{0};
    cudaError_t e = prepare_kernel_once(qkv_proj_kernel, kSmemBytes, prepared);
    if (e != cudaSuccess)
        return e;
    const long long tiles = (long long)p.tiles_m * p.tiles_n;
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    qkv_proj_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

} // namespace mimo
