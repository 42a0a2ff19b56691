// Decode attention of one MiMo-V2-Flash layer: one new token per sequence.
//
// bf16, Dqk 192, Dv 128, G <= 16 query heads per KV head: split-KV kernel.
//   grid (split, kv head, batch); 4 warps. The CTA rotates the G query heads
//   of its KV group at position L-1 (partial RoPE) into shared memory; the CTA
//   whose key range holds the new token's slot also rotates the new key,
//   writes key and value into the cache slot (L-1 for a global cache,
//   (L-1) mod window for a sliding-window ring) and uses its own copy.
//   K/V tiles of 64 keys stream through a multi-stage cp.async pipeline with
//   16-byte coalesced loads (all stages go out as soon as kv_lens, the first
//   load of the kernel, has arrived); each warp takes 16 keys of a tile and
//   runs S = Q K^T and O += P V on mma.sync m16n8k16 (query heads on M, keys
//   on N), with the row max / sum reduced by warp shuffles. Warps are merged
//   through shared memory; a sequence with one split is finished in place
//   (sink folded, V scale applied), otherwise the (m, l, O) partials go to the
//   workspace and a combine kernel merges them, one warp per query head.
// fp8 (E4M3) caches, same kernel with kFp8: each warp streams its own 16 keys
//   of every tile through a private cp.async ring and builds its f16 mma
//   operands from the landed bytes in registers (QK over a permuted order of
//   the 192 dims, PV with permuted output dims, undone at the merge); the new
//   token is quantized into its slot and read back as codes. Sliding layers
//   with a ring of at most two tiles take a slim form (query fragments read
//   from shared memory per k-step, 2 stages, 4 CTAs per SM), so one wave
//   holds every (sequence, KV head) of a B64 batch.
// Other dtypes / dims: a CUDA-core path (one warp per query head) after a
// separate new-token write.
#include "kernels.cuh"

#include <math.h>

namespace mimo {
namespace {

constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kThreads = 128;
constexpr int kTileKeys = 64;
constexpr int kKStride = kDqk + 8;  // elements; 400-byte rows keep ldmatrix conflict-free
constexpr int kVStride = kDv + 8;   // 272-byte rows
constexpr int kQStride = kDqk + 8;
constexpr int kChunkKeys = 2048;    // keys per split on global layers
constexpr int kStageElems = kTileKeys * (kKStride + kVStride);
// Ring depth x CTAs per SM: the bytes in flight per SM, (stages - 1) x 43 KB x
// CTAs, must cover the HBM latency at full bandwidth.
// fp8 (E4M3) caches: each warp streams its own 16 keys of every tile as dense
// 320-byte rows (K then V) through a private ring and builds its mma operands
// straight from those bytes (every E4M3 value is exact in f16), so the loop
// has no CTA barrier and no widening pass.
constexpr int kLandRow = kDqk + kDv;             // bytes per key
constexpr int kWarpLand = 16 * kLandRow;         // one warp's 16 keys: 5120
constexpr int kLandBytes = kTileKeys * kLandRow;  // one stage of the CTA: 20480
// SLIM: the query fragments stay in shared memory and are read per k-step
// instead of held in 48 registers, so 4 CTAs fit per SM (128 registers; fp8:
// 2 stages of 20 KB, bf16: 1 stage of 43 KB): the 512 CTAs of a 128-slot
// sliding layer at B64 run in one wave.
template <int ST, bool F8 = false, bool SLIM = false> struct DecodeCfg {
    static constexpr int kSmemBytes = F8 ? (16 * kQStride + kDqk + kDv) * 2 + kLandRow + ST * kLandBytes
                                         : (16 * kQStride + ST * kStageElems + kDqk + kDv) * 2;
    static constexpr int kCtasPerSm = SLIM ? 4 : F8 ? (ST <= 3 ? 3 : 2) : (ST <= 2 ? 2 : 1);
};

// 16-bit operand type of the tensor-core path: bf16 for bf16 caches, f16 for
// fp8 caches (their e4m3 values, the f16 query and the probabilities).
template <bool F8> __device__ __forceinline__ uint32_t pack16(float lo, float hi)
{
    return F8 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}
// 8 bf16 (a 16-byte chunk) as 8 f16.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v)
{
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        w[i] = pack_f16x2(f.x, f.y);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
constexpr int kDecodeStages = 2;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kDecodeStagesFp8 = 3;  // 5 KB per warp and stage; 69 KB per CTA: 3 CTAs (12 warps) per SM
static_assert(DecodeCfg<kDecodeStagesFp8, true>::kSmemBytes <= 72 * 1024, "3 CTAs per SM");
constexpr int kDecodeStagesSlim = 2;  // fp8: 48 KB per CTA: 4 CTAs per SM
static_assert(DecodeCfg<kDecodeStagesSlim, true, true>::kSmemBytes <= 55 * 1024, "4 CTAs per SM");
constexpr int kDecodeStagesSlimBf16 = 1;  // bf16: 49 KB per CTA: 4 CTAs per SM
static_assert(DecodeCfg<kDecodeStagesSlimBf16, false, true>::kSmemBytes <= 55 * 1024, "4 CTAs per SM");

struct DecodeSmem {
    float wm[4][16];
    float wl[4][16];
};
// Row stride (floats) of the per-warp O slices of the final merge, which
// reuse the stage buffers: 4 x 16 rows x 136 floats = 34 KB.
constexpr int kMergeStride = kDv + 8;
static_assert(4 * 16 * kMergeStride * 4 <= kStageElems * 2, "merge slices fit in one stage buffer");
static_assert(4 * 16 * kMergeStride * 4 <= kDecodeStagesSlim * kLandBytes, "merge slices fit in the fp8 rings");

__device__ __forceinline__ int visible_count(int layer_type, int Lb, int window)
{
    return layer_type == 1 ? min(Lb, window) : Lb;
}

__device__ __forceinline__ bool kv_len_ok(int layer_type, int Lb, int cap)
{
    return Lb >= 1 && (layer_type == 1 || Lb <= cap);
}

template <int kStages, bool kFp8 = false, bool kSlim = false>
__global__ void __launch_bounds__(kThreads, DecodeCfg<kStages, kFp8, kSlim>::kCtasPerSm)
    decode_mma_kernel(const __grid_constant__ LayerArgs L, const __grid_constant__ DecodeArgs a)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // Query rows: bf16, or f16 with fp8 caches. bf16: then the K/V stage
    // ring and the raw new k/v. fp8: the raw new k/v, the new token's codes
    // (K then V) and the per-warp landing rings (warp w, stage s at
    // (w * kStages + s) * kWarpLand).
    __nv_bfloat16 *sQ = reinterpret_cast<__nv_bfloat16 *>(smem_raw);
    __nv_bfloat16 *sStage = sQ + 16 * kQStride;
    __nv_bfloat16 *sKnew = sStage + (kFp8 ? 0 : kStages * kStageElems);
    __nv_bfloat16 *sVnew = sKnew + kDqk;
    uint8_t *sNew8 = reinterpret_cast<uint8_t *>(sVnew + kDv);
    uint8_t *sLand = sNew8 + kLandRow;
    __shared__ DecodeSmem red;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int split = blockIdx.x;
    const int kvh = blockIdx.y;
    const int b = blockIdx.z;
    const int G = L.G;
    const int half = L.rope.half;
    // kv_lens goes out first: every later step waits for it, and loads issued
    // after the K/V tile copies would queue behind them.
    const int Lb = __ldg(a.kv_lens + b);

    // The query rows of this KV group and the new token's k/v do not depend
    // on kv_lens: their loads go out beside it, instead of one dependent
    // round trip after another.
    const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                              ((size_t)b * L.Hq + (size_t)kvh * G) * kDqk;
    const bool vec_rope = L.rope.rotary_dim % 16 == 0;
    // Rotary unit: a 16-byte chunk pair (c, c + r/16); copy unit: one
    // pass-through chunk.
    const int npair = half / 8;
    const int per_row = npair + (kDqk - L.rope.rotary_dim) / 8;
    uint4 va[3], vb[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int u = tid + k * kThreads;
        const int r = u / per_row;
        const int w = u - r * per_row;
        va[k] = make_uint4(0, 0, 0, 0);
        vb[k] = make_uint4(0, 0, 0, 0);
        if (vec_rope && r < G && r < 16) {
            const uint4 *qr = reinterpret_cast<const uint4 *>(qg + (size_t)r * kDqk);
            if (w < npair) {
                va[k] = __ldg(qr + w);
                vb[k] = __ldg(qr + w + npair);
            } else {
                va[k] = __ldg(qr + npair + w);
            }
        }
    }
    const __nv_bfloat16 *kn = reinterpret_cast<const __nv_bfloat16 *>(a.k_new) + ((size_t)b * L.Hkv + kvh) * kDqk;
    const __nv_bfloat16 *vn = reinterpret_cast<const __nv_bfloat16 *>(a.v_new) + ((size_t)b * L.Hkv + kvh) * kDv;
    uint4 nv = make_uint4(0, 0, 0, 0);  // chunk tid of k_new (tid < 24) or v_new (24 <= tid < 40)
    if (tid < 24)
        nv = __ldg(reinterpret_cast<const uint4 *>(kn) + tid);
    else if (tid < 40)
        nv = __ldg(reinterpret_cast<const uint4 *>(vn) + (tid - 24));
    // The sink logits of the group's heads are read now, not in the epilogue.
    const float sink_in = (L.sinks != nullptr && tid < G) ? __ldg(L.sinks + kvh * G + tid) : 0.f;

    const size_t kv_row = (size_t)L.Hkv;  // rows of the cache are [slot][Hkv][D]
    const uint8_t *kc8 = reinterpret_cast<const uint8_t *>(a.k_cache) + ((size_t)b * a.cap * kv_row + kvh) * kDqk;
    const uint8_t *vc8 = reinterpret_cast<const uint8_t *>(a.v_cache) + ((size_t)b * a.cap * kv_row + kvh) * kDv;
    const __nv_bfloat16 *kc = reinterpret_cast<const __nv_bfloat16 *>(a.k_cache) +
                              ((size_t)b * a.cap * kv_row + kvh) * kDqk;
    const __nv_bfloat16 *vc = reinterpret_cast<const __nv_bfloat16 *>(a.v_cache) +
                              ((size_t)b * a.cap * kv_row + kvh) * kDv;

    if (!kv_len_ok(L.layer_type, Lb, a.cap)) {
        if (split == 0 && kvh == 0 && tid == 0)
            atomicOr(a.err, kErrKvLen);
        return;
    }
    const int n_vis = visible_count(L.layer_type, Lb, L.window);
    const int nsplit = (n_vis + a.chunk - 1) / a.chunk;
    if (split >= nsplit)
        return;
    const int key_begin = split * a.chunk;
    const int key_end = min(n_vis, key_begin + a.chunk);
    const int slot_new = L.layer_type == 1 ? (Lb - 1) % L.window : Lb - 1;
    const bool owns_new = slot_new >= key_begin && slot_new < key_end;
    const double pos = (double)(Lb - 1);

    // The K/V tiles go out before the query preparation below: the whole
    // ring of kStages tiles. Rows past the range and the new token's slot are
    // zero-filled (the new token comes from its own copy; a slot past the
    // range may hold any bits).
    const int n_tiles = (key_end - key_begin + kTileKeys - 1) / kTileKeys;
    // Each thread copies a fixed pattern of 16-byte chunks in every tile, so
    // the shared-memory offsets are compile-time steps from one base and only
    // the key rows change per tile. bf16: K rows are 24 chunks: thread (key
    // kr + 16i, chunk kch + 8j); V rows are 16 chunks: thread (key vr + 8i,
    // chunk vch). fp8, per warp and its 16 keys: K rows are 12 chunks: lane
    // (key fr + 8i, chunk fch + 4j); V rows are 8 chunks: lane (key gr + 4i,
    // chunk gch).
    const int kr = tid >> 3, kch = tid & 7;
    const int vr = tid >> 4, vch = tid & 15;
    const int fr = lane >> 2, fch = lane & 3;
    const int gr = lane >> 3, gch = lane & 7;
    const size_t k_rstride = kv_row * kDqk;  // elements (bf16) or bytes (fp8) between key rows
    const size_t v_rstride = kv_row * kDv;
    auto row_of = [&](int key) { return (size_t)(key < key_end && key != slot_new ? key : key_begin); };
    auto ok_of = [&](int key) { return key < key_end && key != slot_new ? 16u : 0u; };
    auto issue = [&](int t) {
        const int base_key = key_begin + t * kTileKeys;
        if (kFp8) {
            const int wkey = base_key + warp * 16;
            uint8_t *land = sLand + (warp * kStages + t % kStages) * kWarpLand;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int key = wkey + fr + 8 * i;
                const uint8_t *src = kc8 + row_of(key) * k_rstride + fch * 16;
                const uint32_t n = ok_of(key);
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    cp_async16(land + (fr + 8 * i) * kLandRow + (fch + 4 * j) * 16, src + j * 64, n);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int key = wkey + gr + 4 * i;
                cp_async16(land + (gr + 4 * i) * kLandRow + kDqk + gch * 16,
                           vc8 + row_of(key) * v_rstride + gch * 16, ok_of(key));
            }
            return;
        }
        __nv_bfloat16 *st = sStage + (t % kStages) * kStageElems;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int key = base_key + kr + 16 * i;
            const __nv_bfloat16 *src = kc + row_of(key) * k_rstride + kch * 8;
            const uint32_t n = ok_of(key);
#pragma unroll
            for (int j = 0; j < 3; ++j)
                cp_async16(st + (kr + 16 * i) * kKStride + (kch + 8 * j) * 8, src + j * 64, n);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int key = base_key + vr + 8 * i;
            cp_async16(st + kTileKeys * kKStride + (vr + 8 * i) * kVStride + vch * 8,
                       vc + row_of(key) * v_rstride + vch * 8, ok_of(key));
        }
    };
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
        if (s < n_tiles)
            issue(s);
        cp_async_commit();
    }

    // cos/sin of the new token's position for every rotary pair, once per CTA;
    // the raw new k/v chunks go to shared memory.
    __shared__ float2 s_cs[kMaxHalfRotary];
    __shared__ float s_sink[16];
    for (int j = tid; j < half; j += kThreads) {
        float c, s;
        rope_cos_sin(pos, L.rope.inv_freq[j], c, s);
        s_cs[j] = make_float2(c, s);
    }
    if (tid < 16)
        s_sink[tid] = sink_in;
    if (tid < 24)
        reinterpret_cast<uint4 *>(sKnew)[tid] = nv;
    else if (tid < 40)
        reinterpret_cast<uint4 *>(sVnew)[tid - 24] = nv;
    __syncthreads();

    if (vec_rope) {
        // Query heads of this KV group rotated at position L-1 (rows >= G are 0).
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int u = tid + k * kThreads;
            const int r = u / per_row;
            const int w = u - r * per_row;
            if (r >= 16)
                continue;
            uint4 *dst = reinterpret_cast<uint4 *>(sQ + r * kQStride);
            if (w < npair) {
                uint4 ya, yb;
                const uint32_t *pa = reinterpret_cast<const uint32_t *>(&va[k]);
                const uint32_t *pb = reinterpret_cast<const uint32_t *>(&vb[k]);
                uint32_t *qa = reinterpret_cast<uint32_t *>(&ya);
                uint32_t *qb = reinterpret_cast<uint32_t *>(&yb);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 c0 = s_cs[w * 8 + 2 * e];
                    const float2 c1 = s_cs[w * 8 + 2 * e + 1];
                    const float2 xa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pa[e]));
                    const float2 xb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&pb[e]));
                    qa[e] = pack16<kFp8>(xa.x * c0.x - xb.x * c0.y, xa.y * c1.x - xb.y * c1.y);
                    qb[e] = pack16<kFp8>(xb.x * c0.x + xa.x * c0.y, xb.y * c1.x + xa.y * c1.y);
                }
                dst[w] = ya;
                dst[w + npair] = yb;
            } else {
                dst[npair + w] = kFp8 ? bf16x8_to_f16x8(va[k]) : va[k];
            }
        }
    } else {
        for (int idx = tid; idx < 16 * kDqk; idx += kThreads) {
            const int r = idx / kDqk;
            const int e = idx - r * kDqk;
            float y = 0.f;
            if (r < G) {
                const __nv_bfloat16 *qr = qg + (size_t)r * kDqk;
                if (e < L.rope.rotary_dim) {
                    const int j = e < half ? e : e - half;
                    const float2 cs = s_cs[j];
                    const float xa = __bfloat162float(qr[j]);
                    const float xb = __bfloat162float(qr[j + half]);
                    y = e < half ? xa * cs.x - xb * cs.y : xb * cs.x + xa * cs.y;
                } else {
                    y = __bfloat162float(qr[e]);
                }
            }
            if (kFp8)
                reinterpret_cast<__half *>(sQ)[r * kQStride + e] = __float2half_rn(y);
            else
                sQ[r * kQStride + e] = __float2bfloat16_rn(y);
        }
    }
    // New token (CTA-uniform branch): rotate k from its raw copy, then write k
    // and v into the cache slot and keep the rotated copy for the tile.
    // rotated element e of the new key, from its raw copy in sKnew
    auto rot_new_k = [&](int e) -> float {
        if (e < L.rope.rotary_dim) {
            const int j = e < half ? e : e - half;
            const float2 cs = s_cs[j];
            const float xa = __bfloat162float(sKnew[j]);
            const float xb = __bfloat162float(sKnew[j + half]);
            return e < half ? xa * cs.x - xb * cs.y : xb * cs.x + xa * cs.y;
        }
        return __bfloat162float(sKnew[e]);
    };
    if (owns_new && kFp8) {
        // fp8 caches: the rotated key and the value are quantized (divided by
        // their scales, nearest E4M3, saturating) two elements at a time; the
        // tile uses the stored codes' values, as every other cached key.
        uint8_t *kdst = reinterpret_cast<uint8_t *>(a.k_cache) + (((size_t)b * a.cap + slot_new) * kv_row + kvh) * kDqk;
        uint8_t *vdst = reinterpret_cast<uint8_t *>(a.v_cache) + (((size_t)b * a.cap + slot_new) * kv_row + kvh) * kDv;
        uint16_t kq = 0, vq = 0;
        if (tid < kDqk / 2)
            kq = f32x2_to_e4m3x2(rot_new_k(2 * tid) / a.k_scale, rot_new_k(2 * tid + 1) / a.k_scale);
        if (tid < kDv / 2)
            vq = f32x2_to_e4m3x2(__bfloat162float(sVnew[2 * tid]) / a.v_scale,
                                 __bfloat162float(sVnew[2 * tid + 1]) / a.v_scale);
        __syncthreads();  // every raw element read before any is overwritten
        if (tid < kDqk / 2) {
            reinterpret_cast<uint16_t *>(kdst)[tid] = kq;
            reinterpret_cast<uint16_t *>(sNew8)[tid] = kq;
        }
        if (tid < kDv / 2) {
            reinterpret_cast<uint16_t *>(vdst)[tid] = vq;
            reinterpret_cast<uint16_t *>(sNew8 + kDqk)[tid] = vq;
        }
    } else if (owns_new) {
        __nv_bfloat16 *kdst = reinterpret_cast<__nv_bfloat16 *>(a.k_cache) +
                              (((size_t)b * a.cap + slot_new) * kv_row + kvh) * kDqk;
        __nv_bfloat16 *vdst = reinterpret_cast<__nv_bfloat16 *>(a.v_cache) +
                              (((size_t)b * a.cap + slot_new) * kv_row + kvh) * kDv;
        __nv_bfloat16 yk[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int e = tid + k * kThreads;
            yk[k] = __float2bfloat16_rn(e < kDqk ? rot_new_k(e) : 0.f);
        }
        __syncthreads();  // every raw element read before any is overwritten
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int e = tid + k * kThreads;
            if (e < kDqk) {
                sKnew[e] = yk[k];
                kdst[e] = yk[k];
            }
        }
        if (tid < kDv)
            vdst[tid] = sVnew[tid];
    }
    __syncthreads();

    const int g = lane >> 2;  // row (head) g and g + 8
    const int tq = lane & 3;
    // Query fragments (A operand, 16 heads x 192) for the 12 k-steps. fp8:
    // the QK dot product runs over a permutation of the 192 dims that lets a
    // lane read its key operands as whole words: in k-step ks, lane (g, tq)
    // holds dims tq*48 + 4*ks + {0, 1} (fragment k = 2tq, 2tq+1) and
    // tq*48 + 4*ks + {2, 3} (k = 2tq+8, 2tq+9), for the query as for the key.
    uint32_t qa[kSlim ? 1 : 12][4];
    // fp8: the two words of k-step ks in rows g and g + 8 (64-bit reads)
    const uint2 *q0w = reinterpret_cast<const uint2 *>(sQ + g * kQStride + tq * 48);
    const uint2 *q1w = reinterpret_cast<const uint2 *>(sQ + (g + 8) * kQStride + tq * 48);
    // bf16: ldmatrix base of the query fragments (rows and 8-column halves by lane)
    const uint32_t q_ldm = smem_u32(sQ) + (uint32_t)((((lane & 7) + ((lane >> 3) & 1) * 8) * kQStride +
                                                     (lane >> 4) * 8) * 2u);
    if constexpr (kSlim) {
    } else if constexpr (kFp8) {
        const uint32_t *q0 = reinterpret_cast<const uint32_t *>(q0w);
        const uint32_t *q1 = reinterpret_cast<const uint32_t *>(q1w);
#pragma unroll
        for (int ks = 0; ks < 12; ++ks) {
            qa[ks][0] = q0[2 * ks];
            qa[ks][1] = q1[2 * ks];
            qa[ks][2] = q0[2 * ks + 1];
            qa[ks][3] = q1[2 * ks + 1];
        }
    } else {
#pragma unroll
        for (int ks = 0; ks < 12; ++ks)
            ldmatrix_x4(q_ldm + ks * 32, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
    }
    float m0 = -INFINITY, m1 = -INFINITY;  // running max of rows g, g+8 (base 2)
    float l0 = 0.f, l1 = 0.f;              // this thread's partial sums
    float o[16][4];
#pragma unroll
    for (int d = 0; d < 16; ++d)
        o[d][0] = o[d][1] = o[d][2] = o[d][3] = 0.f;

    for (int t = 0; t < n_tiles; ++t) {
        const int base_key = key_begin + t * kTileKeys;
        const int kb = warp * 16;  // this warp's 16 keys within the tile
        // Two accumulators per n-tile (even and odd k-steps), so the 12
        // dependent MMAs of a score tile form two chains of 6.
        float s_acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float s_odd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const uint8_t *land = nullptr;       // fp8: this warp's landed rows of tile t
        const __nv_bfloat16 *st = nullptr;   // bf16: the CTA's stage of tile t
        if constexpr (kFp8) {
            // The warp refills the ring entry of tile t - 1 once all its lanes
            // are done with it, then waits for its own copies of tile t. The
            // first kStages tiles went out before the loop, so tile t is
            // always commit group t.
            __syncwarp();
            if (t > 0) {
                if (t + kStages - 1 < n_tiles)
                    issue(t + kStages - 1);
                cp_async_commit();
            }
            cp_async_wait<kStages - 1>();
            __syncwarp();
            if (base_key + kb >= key_end)
                continue;
            land = sLand + (warp * kStages + t % kStages) * kWarpLand;
            if (owns_new && slot_new >= base_key + kb && slot_new < base_key + kb + 16) {
                if (lane < kLandRow / 16)
                    *reinterpret_cast<uint4 *>(const_cast<uint8_t *>(land) + (slot_new - base_key - kb) * kLandRow +
                                               lane * 16) = *reinterpret_cast<const uint4 *>(sNew8 + lane * 16);
                __syncwarp();
            }
            // S = Q K^T: lane (g, tq) reads its 48 key bytes tq*48 .. of key
            // g (n-tile 0) and 8 + g (n-tile 1); word ks holds the four dims of
            // k-step ks (low half: b0, high half: b1).
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const uint4 *kr4 = reinterpret_cast<const uint4 *>(land + (nt * 8 + g) * kLandRow + tq * 48);
                const uint4 w0 = kr4[0], w1 = kr4[1], w2 = kr4[2];
                const uint32_t kw[12] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w, w2.x, w2.y, w2.z, w2.w};
#pragma unroll
                for (int ks = 0; ks < 12; ++ks) {
                    uint32_t qf[4];
                    if constexpr (kSlim) {
                        const uint2 x0 = q0w[ks], x1 = q1w[ks];
                        qf[0] = x0.x;
                        qf[1] = x1.x;
                        qf[2] = x0.y;
                        qf[3] = x1.y;
                    } else {
                        qf[0] = qa[ks][0];
                        qf[1] = qa[ks][1];
                        qf[2] = qa[ks][2];
                        qf[3] = qa[ks][3];
                    }
                    // (the slim form keeps one chain per n-tile: registers)
                    mma_f16_16816((ks & 1) && !kSlim ? s_odd[nt] : s_acc[nt], qf,
                                  e4m3x2_to_f16x2((uint16_t)(kw[ks] & 0xFFFFu)),
                                  e4m3x2_to_f16x2((uint16_t)(kw[ks] >> 16)));
                }
            }
        } else {
            // Tile t + kStages - 1 goes out before the wait for tile t, so
            // kStages tiles are in flight during it; the barrier first makes
            // sure every warp is done with the buffer it refills (tile t - 1's).
            // The first kStages tiles went out before the loop, so tile t is
            // always commit group t.
            if (t > 0) {
                __syncthreads();
                if (t + kStages - 1 < n_tiles)
                    issue(t + kStages - 1);
                cp_async_commit();
            }
            cp_async_wait<kStages - 1>();
            __syncthreads();
            __nv_bfloat16 *stw = sStage + (t % kStages) * kStageElems;
            if (owns_new && slot_new >= base_key && slot_new < base_key + kTileKeys) {
                const int r = slot_new - base_key;
                if (tid < 24)
                    *reinterpret_cast<uint4 *>(stw + r * kKStride + tid * 8) =
                        *reinterpret_cast<const uint4 *>(sKnew + tid * 8);
                else if (tid < 40)
                    *reinterpret_cast<uint4 *>(stw + kTileKeys * kKStride + r * kVStride + (tid - 24) * 8) =
                        *reinterpret_cast<const uint4 *>(sVnew + (tid - 24) * 8);
                __syncthreads();
            }
            st = stw;
            if (base_key + kb >= key_end)
                continue;
            // S = Q K^T for 16 heads x 16 keys.
            const int mi = lane >> 3;
            const int key = kb + (mi >> 1) * 8 + (lane & 7);
            const uint32_t base = smem_u32(st) + (uint32_t)(key * kKStride + (mi & 1) * 8) * 2u;
#pragma unroll
            for (int ks = 0; ks < 12; ++ks) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(base + ks * 32, b0, b1, b2, b3);
                uint32_t qf[4];
                if constexpr (kSlim) {
                    ldmatrix_x4(q_ldm + ks * 32, qf[0], qf[1], qf[2], qf[3]);
                } else {
                    qf[0] = qa[ks][0];
                    qf[1] = qa[ks][1];
                    qf[2] = qa[ks][2];
                    qf[3] = qa[ks][3];
                }
                mma_bf16_16816((ks & 1) && !kSlim ? s_odd[0] : s_acc[0], qf, b0, b1);
                mma_bf16_16816((ks & 1) && !kSlim ? s_odd[1] : s_acc[1], qf, b2, b3);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                s_acc[nt][e] += kSlim ? 0.f : s_odd[nt][e];
        // Scale, mask keys past the end of the range (only the range's last
        // tile has any), online softmax.
        float mx0 = -INFINITY, mx1 = -INFINITY;
        const bool full_tile = base_key + kTileKeys <= key_end;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int key = base_key + kb + nt * 8 + 2 * tq + e;
                const bool valid = full_tile || key < key_end;
                s_acc[nt][e] = valid ? s_acc[nt][e] * L.scale_log2 : -INFINITY;
                s_acc[nt][2 + e] = valid ? s_acc[nt][2 + e] * L.scale_log2 : -INFINITY;
                mx0 = fmaxf(mx0, s_acc[nt][e]);
                mx1 = fmaxf(mx1, s_acc[nt][2 + e]);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        // The reference max of a row only moves when the block's max exceeds
        // it by more than 2^8 (probabilities stay <= 256, exact in the 16-bit
        // operand types), so O is rescaled rarely: m and l always describe the
        // same reference, and the merge / combine use them as they are.
        const bool up0 = mx0 > m0 + kRescaleThreshold || (m0 == -INFINITY && mx0 > -INFINITY);
        const bool up1 = mx1 > m1 + kRescaleThreshold || (m1 == -INFINITY && mx1 > -INFINITY);
        const float c0 = up0 && m0 != -INFINITY ? exp2f(m0 - mx0) : 1.f;
        const float c1 = up1 && m1 != -INFINITY ? exp2f(m1 - mx1) : 1.f;
        if (up0)
            m0 = mx0;
        if (up1)
            m1 = mx1;
        const float u0 = (m0 == -INFINITY) ? 0.f : m0;
        const float u1 = (m1 == -INFINITY) ? 0.f : m1;
        float p[2][4];
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            p[nt][0] = fast_exp2(s_acc[nt][0] - u0);
            p[nt][1] = fast_exp2(s_acc[nt][1] - u0);
            p[nt][2] = fast_exp2(s_acc[nt][2] - u1);
            p[nt][3] = fast_exp2(s_acc[nt][3] - u1);
            rs0 += p[nt][0] + p[nt][1];
            rs1 += p[nt][2] + p[nt][3];
        }
        l0 = l0 * c0 + rs0;
        l1 = l1 * c1 + rs1;
        if (__any_sync(0xffffffffu, c0 != 1.f || c1 != 1.f)) {
#pragma unroll
            for (int d = 0; d < 16; ++d) {
                o[d][0] *= c0;
                o[d][1] *= c0;
                o[d][2] *= c1;
                o[d][3] *= c1;
            }
        }
        uint32_t pa[4];
        pa[0] = pack16<kFp8>(p[0][0], p[0][1]);
        pa[1] = pack16<kFp8>(p[0][2], p[0][3]);
        pa[2] = pack16<kFp8>(p[1][0], p[1][1]);
        pa[3] = pack16<kFp8>(p[1][2], p[1][3]);
        // O += P V over these 16 keys.
        if constexpr (kFp8) {
            // Output dims are permuted: n-tile dp, column n holds dim n*16 + dp.
            // Lane (g, tq) reads value bytes g*16 .. g*16+15 of keys 2tq, 2tq+1
            // (b0) and 2tq+8, 2tq+9 (b1); prmt pairs the two keys' bytes of one
            // dim, lower key in the low byte.
            const uint8_t *vb = land + kDqk + g * 16;
            const uint4 va = *reinterpret_cast<const uint4 *>(vb + (2 * tq) * kLandRow);
            const uint4 vb1 = *reinterpret_cast<const uint4 *>(vb + (2 * tq + 1) * kLandRow);
            const uint4 vc2 = *reinterpret_cast<const uint4 *>(vb + (2 * tq + 8) * kLandRow);
            const uint4 vd3 = *reinterpret_cast<const uint4 *>(vb + (2 * tq + 9) * kLandRow);
            const uint32_t A[4] = {va.x, va.y, va.z, va.w}, B[4] = {vb1.x, vb1.y, vb1.z, vb1.w};
            const uint32_t C[4] = {vc2.x, vc2.y, vc2.z, vc2.w}, D[4] = {vd3.x, vd3.y, vd3.z, vd3.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t lo01 = __byte_perm(A[w], B[w], 0x5140u), hi01 = __byte_perm(C[w], D[w], 0x5140u);
                const uint32_t lo23 = __byte_perm(A[w], B[w], 0x7362u), hi23 = __byte_perm(C[w], D[w], 0x7362u);
                mma_f16_16816(o[4 * w], pa, e4m3x2_to_f16x2((uint16_t)(lo01 & 0xFFFFu)),
                              e4m3x2_to_f16x2((uint16_t)(hi01 & 0xFFFFu)));
                mma_f16_16816(o[4 * w + 1], pa, e4m3x2_to_f16x2((uint16_t)(lo01 >> 16)),
                              e4m3x2_to_f16x2((uint16_t)(hi01 >> 16)));
                mma_f16_16816(o[4 * w + 2], pa, e4m3x2_to_f16x2((uint16_t)(lo23 & 0xFFFFu)),
                              e4m3x2_to_f16x2((uint16_t)(hi23 & 0xFFFFu)));
                mma_f16_16816(o[4 * w + 3], pa, e4m3x2_to_f16x2((uint16_t)(lo23 >> 16)),
                              e4m3x2_to_f16x2((uint16_t)(hi23 >> 16)));
            }
        } else {
            const int mi = lane >> 3;
            const int key = kb + (mi & 1) * 8 + (lane & 7);
            const uint32_t base = smem_u32(st + kTileKeys * kKStride) +
                                  (uint32_t)(key * kVStride + (mi >> 1) * 8) * 2u;
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(base + dp * 32, b0, b1, b2, b3);
                mma_bf16_16816(o[2 * dp], pa, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
            }
        }
    }
    cp_async_wait<0>();

    // Merge the four warps.
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (tq == 0) {
        red.wm[warp][g] = m0;
        red.wm[warp][g + 8] = m1;
        red.wl[warp][g] = l0;
        red.wl[warp][g + 8] = l1;
    }
    __syncthreads();  // every warp is past its last tile: the stage buffers are free
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        M0 = fmaxf(M0, red.wm[w][g]);
        M1 = fmaxf(M1, red.wm[w][g + 8]);
    }
    const float f0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M0);
    const float f1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M1);
    // Each warp writes its rescaled partial O into its own slice in fragment
    // order (column 8d + n holds n-tile d, column n; rows padded to
    // kMergeStride floats so the 8 rows of a warp's access fall in different
    // banks), then one pass sums the four slices. With fp8 caches n-tile d,
    // column n is output dim 16n + d: the summing pass undoes that.
    float *slices = reinterpret_cast<float *>(kFp8 ? sLand : reinterpret_cast<uint8_t *>(sStage));
    {
        float *sl = slices + warp * 16 * kMergeStride;
#pragma unroll
        for (int d = 0; d < 16; ++d) {
            const int col = d * 8 + 2 * tq;
            *reinterpret_cast<float2 *>(sl + g * kMergeStride + col) = make_float2(o[d][0] * f0, o[d][1] * f0);
            *reinterpret_cast<float2 *>(sl + (g + 8) * kMergeStride + col) = make_float2(o[d][2] * f1, o[d][3] * f1);
        }
    }
    __syncthreads();

    // Row r = query head kvh*G + r; thread -> (row, 16 columns).
    for (int idx = tid; idx < G * (kDv / 16); idx += kThreads) {
        const int r = idx / (kDv / 16);
        const int c0 = (idx % (kDv / 16)) * 16;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w)
            M = fmaxf(M, red.wm[w][r]);
        float Ls = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w)
            Ls += (red.wm[w][r] == -INFINITY) ? 0.f : red.wl[w][r] * exp2f(red.wm[w][r] - M);
        // this row's 16 columns, summed over the four warps' slices
        float v[16];
        if constexpr (kFp8) {
            // output dims c0 + j = 16n + d with n = c0 / 16, d = j: column 8j + n
            const int n = c0 >> 4;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float acc = slices[r * kMergeStride + 8 * j + n];
#pragma unroll
                for (int w = 1; w < 4; ++w)
                    acc += slices[(w * 16 + r) * kMergeStride + 8 * j + n];
                v[j] = acc;
            }
        } else {
#pragma unroll
            for (int c = 0; c < 16; c += 4) {
                float4 acc = *reinterpret_cast<const float4 *>(slices + r * kMergeStride + c0 + c);
#pragma unroll
                for (int w = 1; w < 4; ++w) {
                    const float4 x = *reinterpret_cast<const float4 *>(slices + (w * 16 + r) * kMergeStride + c0 + c);
                    acc.x += x.x;
                    acc.y += x.y;
                    acc.z += x.z;
                    acc.w += x.w;
                }
                v[c] = acc.x;
                v[c + 1] = acc.y;
                v[c + 2] = acc.z;
                v[c + 3] = acc.w;
            }
        }
        const int h = kvh * G + r;
        if (nsplit == 1) {
            float scale;
            if (L.sinks != nullptr) {
                const float s2 = s_sink[r] * kLog2e;
                const float mf = fmaxf(M, s2);
                const float al = exp2f(M - mf);
                scale = al * L.v_scale / (Ls * al + exp2f(s2 - mf));
            } else {
                scale = L.v_scale / Ls;
            }
            __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.out) + ((size_t)b * L.Hq + h) * kDv + c0;
            uint4 w0, w1;
            w0.x = pack_bf16x2(v[0] * scale, v[1] * scale);
            w0.y = pack_bf16x2(v[2] * scale, v[3] * scale);
            w0.z = pack_bf16x2(v[4] * scale, v[5] * scale);
            w0.w = pack_bf16x2(v[6] * scale, v[7] * scale);
            w1.x = pack_bf16x2(v[8] * scale, v[9] * scale);
            w1.y = pack_bf16x2(v[10] * scale, v[11] * scale);
            w1.z = pack_bf16x2(v[12] * scale, v[13] * scale);
            w1.w = pack_bf16x2(v[14] * scale, v[15] * scale);
            reinterpret_cast<uint4 *>(dst)[0] = w0;
            reinterpret_cast<uint4 *>(dst)[1] = w1;
        } else {
            float *part = a.partial + (((size_t)b * L.Hq + h) * a.max_splits + split) * (kDv + 2);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                part[c0 + c] = v[c];
            if (c0 == 0) {
                part[kDv] = M;
                part[kDv + 1] = Ls;
            }
        }
    }
}

// Merges the split partials of one (batch, query head) per warp (Dv 128):
// log-sum-exp merge, sink folded into the denominator, V scale applied. grid
// (Hq / 4, batch), 4 warps. Lane s holds split s's (m, l) (more splits:
// strided loops); each lane takes four output dims as two float2 reads of
// every split's partial O (8-byte aligned: rows of Dv + 2 floats).
template <typename T>
__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ LayerArgs L,
                                                             const __grid_constant__ DecodeArgs a)
{
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x * 4 + warp;
    const int b = blockIdx.y;
    if (h >= L.Hq)
        return;
    const int Lb = __ldg(a.kv_lens + b);
    if (!kv_len_ok(L.layer_type, Lb, a.cap))
        return;
    const int n_vis = visible_count(L.layer_type, Lb, L.window);
    const int nsplit = (n_vis + a.chunk - 1) / a.chunk;
    if (nsplit <= 1)
        return;
    const int stride = L.Dv + 2;
    const float *part = a.partial + ((size_t)b * L.Hq + h) * a.max_splits * stride;
    const float s2 = L.sinks != nullptr ? __ldg(L.sinks + h) * kLog2e : -INFINITY;
    // every split holds at least one key, so its m is finite
    float m_l = -INFINITY, l_l = 0.f;
    if (lane < nsplit) {
        m_l = part[(size_t)lane * stride + L.Dv];
        l_l = part[(size_t)lane * stride + L.Dv + 1];
    }
    float M = fmaxf(m_l, s2);
    for (int s = lane + 32; s < nsplit; s += 32)
        M = fmaxf(M, part[(size_t)s * stride + L.Dv]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w_l = lane < nsplit ? exp2f(m_l - M) : 0.f;  // weight of split `lane`
    float Ls = w_l * l_l;
    for (int s = lane + 32; s < nsplit; s += 32) {
        const float *ps = part + (size_t)s * stride;
        Ls += ps[L.Dv + 1] * exp2f(ps[L.Dv] - M);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    if (L.sinks != nullptr)
        Ls += exp2f(s2 - M);
    const float scale = L.v_scale / Ls;
    // dims 2 lane, 2 lane + 1 and 64 + 2 lane, 65 + 2 lane (Dv 128), splits
    // in batches of 8 whose loads all go out before the sums
    T *out = reinterpret_cast<T *>(a.out) + ((size_t)b * L.Hq + h) * kDv;
    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
    for (int s0 = 0; s0 < nsplit; s0 += 8) {
        float2 o0[8], o1[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float *ps = part + (size_t)(s0 + j) * stride + 2 * lane;
            o0[j] = s0 + j < nsplit ? *reinterpret_cast<const float2 *>(ps) : make_float2(0.f, 0.f);
            o1[j] = s0 + j < nsplit ? *reinterpret_cast<const float2 *>(ps + 64) : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int s = s0 + j;
            float w;
            if (s < 32)
                w = __shfl_sync(0xffffffffu, w_l, s);
            else
                w = s < nsplit ? exp2f(part[(size_t)s * stride + kDv] - M) : 0.f;
            acc0.x += w * o0[j].x;
            acc0.y += w * o0[j].y;
            acc1.x += w * o1[j].x;
            acc1.y += w * o1[j].y;
        }
    }
    out[2 * lane] = from_f32<T>(acc0.x * scale);
    out[2 * lane + 1] = from_f32<T>(acc0.y * scale);
    out[64 + 2 * lane] = from_f32<T>(acc1.x * scale);
    out[65 + 2 * lane] = from_f32<T>(acc1.y * scale);
}

// ------------------------------------------------------- CUDA-core path
// Writes the new token (rotated key, value) into its cache slot.
template <typename T>
__global__ void decode_write_new_kernel(const __grid_constant__ LayerArgs L, const __grid_constant__ DecodeArgs a)
{
    const int kvh = blockIdx.x;
    const int b = blockIdx.y;
    const int Lb = __ldg(a.kv_lens + b);
    if (!kv_len_ok(L.layer_type, Lb, a.cap)) {
        if (kvh == 0 && threadIdx.x == 0)
            atomicOr(a.err, kErrKvLen);
        return;
    }
    const int slot = L.layer_type == 1 ? (Lb - 1) % L.window : Lb - 1;
    const double pos = (double)(Lb - 1);
    const int half = L.rope.half;
    __shared__ float2 s_cs[kMaxHalfRotary];
    for (int j = threadIdx.x; j < half; j += blockDim.x) {
        float c, s;
        rope_cos_sin(pos, L.rope.inv_freq[j], c, s);
        s_cs[j] = make_float2(c, s);
    }
    __syncthreads();
    const T *kn = reinterpret_cast<const T *>(a.k_new) + ((size_t)b * L.Hkv + kvh) * L.Dqk;
    const T *vn = reinterpret_cast<const T *>(a.v_new) + ((size_t)b * L.Hkv + kvh) * L.Dv;
    T *kd = reinterpret_cast<T *>(a.k_cache) + (((size_t)b * a.cap + slot) * L.Hkv + kvh) * L.Dqk;
    T *vd = reinterpret_cast<T *>(a.v_cache) + (((size_t)b * a.cap + slot) * L.Hkv + kvh) * L.Dv;
    for (int e = threadIdx.x; e < L.Dqk; e += blockDim.x) {
        float y;
        if (e < L.rope.rotary_dim) {
            const int j = e < half ? e : e - half;
            const float2 cs = s_cs[j];
            const float xa = to_f32<T>(kn[j]);
            const float xb = to_f32<T>(kn[j + half]);
            y = e < half ? xa * cs.x - xb * cs.y : xb * cs.x + xa * cs.y;
        } else {
            y = to_f32<T>(kn[e]);
        }
        kd[e] = from_f32<T>(y);
    }
    for (int e = threadIdx.x; e < L.Dv; e += blockDim.x)
        vd[e] = vn[e];
}

// One warp per (batch, query head) over the visible cache slots.
template <typename T>
__global__ void decode_simt_kernel(const __grid_constant__ LayerArgs L, const __grid_constant__ DecodeArgs a)
{
    __shared__ float qs[4][256];
    __shared__ float2 s_cs[kMaxHalfRotary];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x * 4 + warp;
    const int b = blockIdx.y;
    const int Lb = __ldg(a.kv_lens + b);
    if (!kv_len_ok(L.layer_type, Lb, a.cap))
        return;
    const double pos = (double)(Lb - 1);
    const int half = L.rope.half;
    for (int j = threadIdx.x; j < half; j += blockDim.x) {
        float c, s;
        rope_cos_sin(pos, L.rope.inv_freq[j], c, s);
        s_cs[j] = make_float2(c, s);
    }
    __syncthreads();
    if (h >= L.Hq)
        return;
    const int n_vis = visible_count(L.layer_type, Lb, L.window);
    const T *q = reinterpret_cast<const T *>(a.q) + ((size_t)b * L.Hq + h) * L.Dqk;
    for (int e = lane; e < L.Dqk; e += 32) {
        float y;
        if (e < L.rope.rotary_dim) {
            const int j = e < half ? e : e - half;
            const float2 cs = s_cs[j];
            const float xa = to_f32<T>(q[j]);
            const float xb = to_f32<T>(q[j + half]);
            y = e < half ? xa * cs.x - xb * cs.y : xb * cs.x + xa * cs.y;
        } else {
            y = to_f32<T>(q[e]);
        }
        qs[warp][e] = y;
    }
    __syncwarp();
    const int kvh = h / L.G;
    float m = -INFINITY, l = 0.f;
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t)
        acc[t] = 0.f;
    for (int slot = 0; slot < n_vis; ++slot) {
        const T *kr = reinterpret_cast<const T *>(a.k_cache) + (((size_t)b * a.cap + slot) * L.Hkv + kvh) * L.Dqk;
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
        const T *vr = reinterpret_cast<const T *>(a.v_cache) + (((size_t)b * a.cap + slot) * L.Hkv + kvh) * L.Dv;
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
    T *dst = reinterpret_cast<T *>(a.out) + ((size_t)b * L.Hq + h) * L.Dv;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const int e = lane + 32 * t;
        if (e < L.Dv)
            dst[e] = from_f32<T>(acc[t] * scale);
    }
}

bool decode_mma_supported(const LayerArgs &L, int dtype)
{
    return dtype == kDtypeBf16 && L.Dqk == kDqk && L.Dv == kDv && L.G >= 1 && L.G <= 16;
}

} // namespace

int decode_chunk_keys(const LayerArgs &L, int dtype)
{
    if (!decode_mma_supported(L, dtype))
        return 1 << 30;
    return L.layer_type == 1 ? max(L.window, 1) : kChunkKeys;
}

int decode_max_splits(const LayerArgs &L, int dtype, int cap)
{
    const int chunk = decode_chunk_keys(L, dtype);
    return (cap + chunk - 1) / chunk;
}

namespace {
__global__ void quantize_e4m3_kernel(const __nv_bfloat16 *src, uint8_t *dst, size_t n, float scale)
{
    for (size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 2; i < n; i += (size_t)gridDim.x * blockDim.x * 2) {
        const float x0 = __bfloat162float(src[i]) / scale;
        if (i + 1 < n) {
            const uint16_t c = f32x2_to_e4m3x2(x0, __bfloat162float(src[i + 1]) / scale);
            dst[i] = (uint8_t)(c & 0xFF);
            dst[i + 1] = (uint8_t)(c >> 8);
        } else {
            dst[i] = (uint8_t)(f32x2_to_e4m3x2(x0, 0.f) & 0xFF);
        }
    }
}
} // namespace

cudaError_t launch_quantize_e4m3(const void *src, void *dst, size_t n, float scale, cudaStream_t stream)
{
    const size_t pairs = (n + 1) / 2;
    const size_t blocks = (pairs + 255) / 256;
    quantize_e4m3_kernel<<<(unsigned)(blocks < 65536 ? blocks : 65536), 256, 0, stream>>>(
        reinterpret_cast<const __nv_bfloat16 *>(src), reinterpret_cast<uint8_t *>(dst), n, scale);
    return cudaGetLastError();
}

cudaError_t launch_decode(const LayerArgs &L, const DecodeArgs &a, int dtype, cudaStream_t stream)
{
    if (a.fp8_cache && !decode_mma_supported(L, dtype))
        return cudaErrorInvalidValue;
    if (decode_mma_supported(L, dtype)) {
        static std::atomic<unsigned long long> prepared[4] = {{0}, {0}, {0}, {0}};
        // sliding layers whose ring is at most two tiles take the slim forms
        const bool slim = L.layer_type == 1 && L.window <= 2 * kTileKeys;
        const int f = a.fp8_cache ? (slim ? 2 : 1) : (slim ? 3 : 0);
        {
            cudaError_t e =
                f == 3 ? prepare_kernel_once(decode_mma_kernel<kDecodeStagesSlimBf16, false, true>,
                                             DecodeCfg<kDecodeStagesSlimBf16, false, true>::kSmemBytes, prepared[3])
                : f == 2 ? prepare_kernel_once(decode_mma_kernel<kDecodeStagesSlim, true, true>,
                                               DecodeCfg<kDecodeStagesSlim, true, true>::kSmemBytes, prepared[2])
                : f == 1 ? prepare_kernel_once(decode_mma_kernel<kDecodeStagesFp8, true>,
                                               DecodeCfg<kDecodeStagesFp8, true>::kSmemBytes, prepared[1])
                         : prepare_kernel_once(decode_mma_kernel<kDecodeStages, false>,
                                               DecodeCfg<kDecodeStages, false>::kSmemBytes, prepared[0]);
            if (e != cudaSuccess)
                return e;
        }
        dim3 grid(a.max_splits, L.Hkv, a.B);
        if (f == 3)
            decode_mma_kernel<kDecodeStagesSlimBf16, false, true>
                <<<grid, kThreads, DecodeCfg<kDecodeStagesSlimBf16, false, true>::kSmemBytes, stream>>>(L, a);
        else if (f == 2)
            decode_mma_kernel<kDecodeStagesSlim, true, true>
                <<<grid, kThreads, DecodeCfg<kDecodeStagesSlim, true, true>::kSmemBytes, stream>>>(L, a);
        else if (f == 1)
            decode_mma_kernel<kDecodeStagesFp8, true>
                <<<grid, kThreads, DecodeCfg<kDecodeStagesFp8, true>::kSmemBytes, stream>>>(L, a);
        else
            decode_mma_kernel<kDecodeStages, false>
                <<<grid, kThreads, DecodeCfg<kDecodeStages, false>::kSmemBytes, stream>>>(L, a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess || a.max_splits <= 1)
            return e;
        decode_combine_kernel<__nv_bfloat16><<<dim3((L.Hq + 3) / 4, a.B), 128, 0, stream>>>(L, a);
        return cudaGetLastError();
    }
    dim3 g1(L.Hkv, a.B);
    dim3 g2((L.Hq + 3) / 4, a.B);
    if (dtype == kDtypeBf16) {
        decode_write_new_kernel<__nv_bfloat16><<<g1, 128, 0, stream>>>(L, a);
        decode_simt_kernel<__nv_bfloat16><<<g2, 128, 0, stream>>>(L, a);
    } else {
        decode_write_new_kernel<float><<<g1, 128, 0, stream>>>(L, a);
        decode_simt_kernel<float><<<g2, 128, 0, stream>>>(L, a);
    }
    return cudaGetLastError();
}

} // namespace mimo
