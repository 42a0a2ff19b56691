// Prefill attention of one MiMo-V2-Flash layer on the sm_100a tensor cores.
//
// One CTA computes one tile of 128 query rows. A row is (sequence index i,
// query head h); a tile packs `gp` consecutive query heads of one KV group
// for P = 128 / gp consecutive positions (gp = 1 for global layers; gp = G on
// sliding-window layers so that the key span of a tile is P + window - 1
// keys rather than 128 + window - 1).
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread r owns row r of S and O in TMEM. It also
//              rotates its row of Q in shared memory (partial RoPE fused into
//              the Q tile load), applies the causal / window mask, keeps the
//              running max and sum, writes P (bf16) back into TMEM over the
//              S columns it has read, rescales O when the max grows by more
//              than 2^8, and in the epilogue folds the sink, normalises,
//              applies the V scale and stores O.
//   warp 4     TMA producer: Q once, then K/V tiles of BLOCK_N keys through
//              KST-stage rings. Tiles wholly outside the causal window are
//              never loaded (the key range of the tile is computed first).
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM
//              S buffers, then O += P_{j-1} V_{j-1} with P read from TMEM.
//
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384) of a 512-column
// allocation (one CTA per SM: shared memory use is ~210 KB).
//
// Shared memory: every operand is stored as 128-byte-swizzled rows of 64
// bf16 (the TMA SWIZZLE_128B layout), one 1024-byte-aligned block per 64
// columns: Q = 3 blocks of 128 rows, K stage = 3 blocks of BLOCK_N rows,
// V stage = 2 blocks of BLOCK_N rows (V is read MN-major by the MMA).
#include "kernels.cuh"

#include <math.h>

namespace mimo {
namespace {

constexpr int kBlockM = 128;
constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kThreads = 192;
constexpr int kQBytes = kBlockM * kDqk * 2;       // 49152
constexpr int kTmemCols = 512;

// Key tile of BN keys, ST-deep K and V rings. Smaller tiles with more stages
// keep more bytes in flight per SM for the same shared memory.
template <int BN, int ST> struct TileCfg {
    static constexpr int kKStageBytes = BN * kDqk * 2;
    static constexpr int kVStageBytes = BN * kDv * 2;
    static constexpr int kSmemBytes = 1024 + kQBytes + ST * (kKStageBytes + kVStageBytes) + 256;
    static_assert(BN % 16 == 0 && BN <= 128, "key tile");
    static_assert((BN * 128) % 1024 == 0, "swizzle atoms must stay 1024-byte aligned");
    static_assert(kSmemBytes <= 232448, "shared memory");
};
constexpr int kBN = 128;     // keys per tile
constexpr int kStages = 2;   // K/V ring depth
constexpr int kColS0 = 0;
constexpr int kColS1 = 128;
constexpr int kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct TcParams {
    CUtensorMap tm_q;  // [B, S, Hq, Dqk]    box {64, gp, P, 1}
    CUtensorMap tm_k;  // [B, rows, Hkv, Dqk] box {64, 1, BLOCK_N, 1}
    CUtensorMap tm_v;  // [B, S, Hkv, Dv]    box {64, 1, BLOCK_N, 1}
    __nv_bfloat16 *out;
    const int *positions;
    const float *sinks;
    unsigned *err;
    int S, Hq, G, gp, P, window, is_swa;
    int num_p_tiles, num_g_tiles;
    float scale_log2;
    float v_scale;
    RopeArgs rope;
};

template <int ST> struct SmemBars {
    uint64_t q_full, q_ready;
    uint64_t k_full[ST], k_empty[ST];
    uint64_t v_full[ST], v_empty[ST];
    uint64_t s_full[2], p_full[2];
    uint64_t o_done;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};


// Byte offset of element e of row `row` in a 128B-swizzled operand whose
// 64-column blocks are `block_bytes` apart.
__device__ __forceinline__ uint32_t swz_offset(int row, int e, int block_bytes)
{
    int blk = e >> 6;
    int chunk = (e & 63) >> 3;
    return (uint32_t)(blk * block_bytes + row * 128 + ((chunk ^ (row & 7)) << 4) + ((e & 7) << 1));
}

template <int BN, int ST>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ TcParams p)
{
    using Cfg = TileCfg<BN, ST>;
    constexpr int kBlockN = BN;
    constexpr int kKStages = ST;
    constexpr int kKStageBytes = Cfg::kKStageBytes;
    constexpr int kVStageBytes = Cfg::kVStageBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = smem;
    uint8_t *sK = sQ + kQBytes;
    uint8_t *sV = sK + kKStages * kKStageBytes;
    SmemBars<ST> *bars = reinterpret_cast<SmemBars<ST> *>(sV + kKStages * kVStageBytes);
    volatile int *abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Heaviest causal tiles first.
    const int pt = p.num_p_tiles - 1 - (int)blockIdx.x;
    const int kvh = (int)blockIdx.y / p.num_g_tiles;
    const int gt = (int)blockIdx.y % p.num_g_tiles;
    const int b = (int)blockIdx.z;
    const int p0 = pt * p.P;
    const int h0 = kvh * p.G + gt * p.gp;
    const int q_last = min(p0 + p.P, p.S) - 1;
    const int k_lo = p.is_swa ? max(0, p0 - p.window + 1) : 0;
    const int n_tiles = (q_last - k_lo) / kBlockN + 1;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_ready, 128);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->p_full[s], 128);
        }
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 5) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 4) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int last_k[kKStages], last_v[kKStages];
            for (int s = 0; s < kKStages; ++s)
                last_k[s] = last_v[s] = -1;
            tma_prefetch_desc(&p.tm_q);
            tma_prefetch_desc(&p.tm_k);
            tma_prefetch_desc(&p.tm_v);
            mbar_arrive_expect_tx(&bars->q_full, kQBytes);
            for (int a = 0; a < 3; ++a)
                tma_load_4d(sQ + a * (kBlockM * 128), &p.tm_q, &bars->q_full, a * 64, h0, p0, b);
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % kKStages;
                const uint32_t ph = (uint32_t)(j / kKStages) & 1u;
                const int k0 = k_lo + j * kBlockN;
                if (!mbar_wait(&bars->k_empty[s], ph ^ 1u, abort_flag, p.err))
                    break;
                mbar_arrive_expect_tx(&bars->k_full[s], kKStageBytes);
                uint8_t *dk = sK + s * kKStageBytes;
                for (int a = 0; a < 3; ++a)
                    tma_load_4d(dk + a * (kBlockN * 128), &p.tm_k, &bars->k_full[s], a * 64, kvh, k0, b);
                last_k[s] = j;
                if (!mbar_wait(&bars->v_empty[s], ph ^ 1u, abort_flag, p.err))
                    break;
                mbar_arrive_expect_tx(&bars->v_full[s], kVStageBytes);
                uint8_t *dv = sV + s * kVStageBytes;
                for (int a = 0; a < 2; ++a)
                    tma_load_4d(dv + a * (kBlockN * 128), &p.tm_v, &bars->v_full[s], a * 64, kvh, k0, b);
                last_v[s] = j;
            }
            if (*abort_flag) {
                // Let every copy still in flight land before the CTA exits:
                // only the latest load of each stage can be outstanding.
                mbar_drain(&bars->q_full, 0);
                for (int s = 0; s < kKStages; ++s) {
                    if (last_k[s] >= 0)
                        mbar_drain(&bars->k_full[s], (uint32_t)(last_k[s] / kKStages) & 1u);
                    if (last_v[s] >= 0)
                        mbar_drain(&bars->v_full[s], (uint32_t)(last_v[s] / kKStages) & 1u);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false, false);
            const uint32_t idesc_pv = idesc_bf16_f32(kBlockM, kDv, false, true);
            const uint32_t q_addr = smem_u32(sQ);
            bool ok = mbar_wait(&bars->q_ready, 0, abort_flag, p.err);
            tc_fence_after();
            auto issue_pv = [&](int jj) -> bool {
                const int s = jj % kKStages;
                const uint32_t ph = (uint32_t)(jj / kKStages) & 1u;
                const int pb = jj & 1;
                if (!mbar_wait(&bars->p_full[pb], (uint32_t)(jj >> 1) & 1u, abort_flag, p.err))
                    return false;
                if (!mbar_wait(&bars->v_full[s], ph, abort_flag, p.err))
                    return false;
                tc_fence_after();
                const uint32_t v_addr = smem_u32(sV + s * kVStageBytes);
                const uint32_t p_col = tmem + (pb ? kColS1 : kColS0);
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk) {
                    const uint64_t bdesc = sdesc_sw128(v_addr + kk * 2048, kBlockN * 128, 1024);
                    umma_ts(tmem + kColO, p_col + kk * 8, bdesc, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars->o_done);
                umma_commit(&bars->v_empty[s]);
                return true;
            };
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int s = j % kKStages;
                const uint32_t ph = (uint32_t)(j / kKStages) & 1u;
                if (!mbar_wait(&bars->k_full[s], ph, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t k_addr = smem_u32(sK + s * kKStageBytes);
                const uint32_t s_col = tmem + ((j & 1) ? kColS1 : kColS0);
#pragma unroll
                for (int kk = 0; kk < kDqk / 16; ++kk) {
                    const int blk = kk >> 2;
                    const uint32_t off = (uint32_t)(kk & 3) * 32u;
                    const uint64_t adesc = sdesc_sw128(q_addr + blk * (kBlockM * 128) + off, 16, 1024);
                    const uint64_t bdesc = sdesc_sw128(k_addr + blk * (kBlockN * 128) + off, 16, 1024);
                    umma_ss(s_col, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars->s_full[j & 1]);
                umma_commit(&bars->k_empty[s]);
                if (j >= 1 && !issue_pv(j - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok)
                ok = issue_pv(n_tiles - 1);
            if (!ok) {
                // Wait for the MMAs already issued before the CTA tears down.
                umma_commit(&bars->drain);
                mbar_drain(&bars->drain, 0);
            }
        }
    } else {
        // ----------------------------------------------------------- softmax
        const int row = threadIdx.x;  // 0..127
        const int i = p0 + row / p.gp;  // sequence index of this row
        const int h = h0 + row % p.gp;
        const bool row_valid = i < p.S;
        bool ok = mbar_wait(&bars->q_full, 0, abort_flag, p.err);

        // Partial RoPE of this row of Q, in place in swizzled shared memory.
        if (ok && row_valid && p.rope.half > 0) {
            const double pos = p.positions ? (double)__ldg(p.positions + i) : (double)i;
            for (int j = 0; j < p.rope.half; ++j) {
                const uint32_t oa = swz_offset(row, j, kBlockM * 128);
                const uint32_t ob = swz_offset(row, j + p.rope.half, kBlockM * 128);
                __nv_bfloat16 *pa = reinterpret_cast<__nv_bfloat16 *>(sQ + oa);
                __nv_bfloat16 *pb = reinterpret_cast<__nv_bfloat16 *>(sQ + ob);
                const float xa = __bfloat162float(*pa);
                const float xb = __bfloat162float(*pb);
                float c, s;
                rope_cos_sin(pos, p.rope.inv_freq[j], c, s);
                *pa = __float2bfloat16_rn(xa * c - xb * s);
                *pb = __float2bfloat16_rn(xb * c + xa * s);
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars->q_ready);

        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float m_ref = -INFINITY;  // reference max (base-2 units) of P and O
        float l_sum = 0.f;
        const int hi_rel = i;                               // last visible key
        const int lo_rel = p.is_swa ? i - p.window + 1 : -0x40000000;
        for (int j = 0; ok && j < n_tiles; ++j) {
            const int sb = j & 1;
            if (!mbar_wait(&bars->s_full[sb], (uint32_t)(j >> 1) & 1u, abort_flag, p.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t s_addr = lane_base + (sb ? kColS1 : kColS0);
            float x[kBlockN];
            {
                uint32_t r[kBlockN / 16][16];
#pragma unroll
                for (int c = 0; c < kBlockN / 16; ++c)
                    tmem_ld16(s_addr + 16 * c, r[c]);
                tmem_wait_ld_only();
#pragma unroll
                for (int c = 0; c < kBlockN / 16; ++c) {
                    tmem_tie(r[c]);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        x[16 * c + e] = __uint_as_float(r[c][e]) * p.scale_log2;
                }
            }
            const int k0 = k_lo + j * kBlockN;
            // Whole tile visible to every row of the CTA?
            const bool full = (k0 + kBlockN - 1 <= p0) &&
                              (!p.is_swa || k0 >= p0 + p.P - 1 - p.window + 1);
            float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (!full) {
                // branch-free mask: column c is visible iff lo <= c <= hi
                const int lo = lo_rel - k0;
                const unsigned span = (unsigned)(hi_rel - lo_rel);
#pragma unroll
                for (int c = 0; c < kBlockN; ++c)
                    x[c] = ((unsigned)(c - lo) <= span) ? x[c] : -INFINITY;
            }
#pragma unroll
            for (int c = 0; c < kBlockN; ++c)
                mxv[c & 3] = fmaxf(mxv[c & 3], x[c]);
            const float mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3]));
            // A row moves its reference max when the tile's max exceeds it by
            // more than the threshold; corr rescales the running sum, and O
            // once an earlier P*V has landed in it.
            const bool move = mx > m_ref + kRescaleThreshold || (m_ref == -INFINITY && mx > -INFINITY);
            const float corr = !move ? 1.f : (m_ref == -INFINITY ? 0.f : exp2f(m_ref - mx));
            // The TMEM load and store are warp-collective (.sync.aligned): the
            // whole warp rescales whenever one of its rows moved (the others by 1).
            if (j > 0 && __any_sync(0xffffffffu, move && m_ref != -INFINITY)) {
                if (!mbar_wait(&bars->o_done, (uint32_t)(j - 1) & 1u, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float f = (m_ref == -INFINITY) ? 1.f : corr;
#pragma unroll
                for (int c0 = 0; c0 < kDv; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(lane_base + kColO + c0, r);
                    tmem_wait_ld(r);
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        r[c] = __float_as_uint(__uint_as_float(r[c]) * f);
                    tmem_st32(lane_base + kColO + c0, r);
                }
            }
            if (move) {
                l_sum *= corr;
                m_ref = mx;
            }
            const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
            float rsv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c0 = 0; c0 < kBlockN; c0 += 16) {
                uint32_t r[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float e0 = fast_exp2(x[c0 + 2 * c] - m_use);
                    const float e1 = fast_exp2(x[c0 + 2 * c + 1] - m_use);
                    rsv[c & 3] += e0 + e1;
                    r[c] = pack_bf16x2(e0, e1);
                }
                tmem_st8(s_addr + c0 / 2, r);
            }
            l_sum += (rsv[0] + rsv[1]) + (rsv[2] + rsv[3]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[sb]);
        }

        // ----------------------------------------------------------- epilogue
        if (ok && mbar_wait(&bars->o_done, (uint32_t)(n_tiles - 1) & 1u, abort_flag, p.err)) {
            tc_fence_after();
            float o_scale;
            if (p.sinks != nullptr) {
                const float s2 = __ldg(p.sinks + h) * kLog2e;
                const float m_fin = fmaxf(m_ref, s2);
                const float a = exp2f(m_ref - m_fin);
                const float l_fin = l_sum * a + exp2f(s2 - m_fin);
                o_scale = a * p.v_scale / l_fin;
            } else {
                o_scale = p.v_scale / l_sum;
            }
            __nv_bfloat16 *dst = p.out + (((size_t)b * p.S + (row_valid ? i : 0)) * p.Hq + h) * kDv;
#pragma unroll
            for (int c0 = 0; c0 < kDv; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(lane_base + kColO + c0, r);
                tmem_wait_ld(r);
                if (row_valid) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(r[c + 0]) * o_scale, __uint_as_float(r[c + 1]) * o_scale);
                        w.y = pack_bf16x2(__uint_as_float(r[c + 2]) * o_scale, __uint_as_float(r[c + 3]) * o_scale);
                        w.z = pack_bf16x2(__uint_as_float(r[c + 4]) * o_scale, __uint_as_float(r[c + 5]) * o_scale);
                        w.w = pack_bf16x2(__uint_as_float(r[c + 6]) * o_scale, __uint_as_float(r[c + 7]) * o_scale);
                        d4[c / 8] = w;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

} // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 4-D bf16 tensor map over [d3][d2][d1][d0] (d0 innermost) with a row pitch
// of `pitch1` elements between consecutive d1 indices, d1*pitch1 between d2
// indices, and d2_alloc*d1*pitch1 between d3 indices.
bool make_bf16_map_4d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t d2_alloc, uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr)
        return false;
    cuuint64_t dims[4] = {d0, d1, d2, d3};
    cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2_alloc * 2};
    cuuint32_t box[4] = {b0, b1, b2, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}


bool prefill_tc_supported(const LayerArgs &L)
{
    if (L.Dqk != kDqk || L.Dv != kDv)
        return false;
    if (L.rope.rotary_dim > kDqk)
        return false;
    return true;
}

cudaError_t launch_prefill_tc(const LayerArgs &L, const PrefillArgs &a, cudaStream_t stream)
{
    TcParams p;
    memset(&p, 0, sizeof(p));
    // Pack the query heads of a KV group into the tile on sliding layers.
    int gp = 1;
    if (L.layer_type == 1) {
        for (int c = 16; c >= 2; c >>= 1)
            if (L.G % c == 0) {
                gp = c;
                break;
            }
    }
    const int P = kBlockM / gp;
    if (!make_bf16_map_4d(&p.tm_q, a.q, kDqk, L.Hq, a.S, a.S, a.B, 64, gp, P) ||
        !make_bf16_map_4d(&p.tm_k, a.krot, kDqk, L.Hkv, a.S, a.krot_rows, a.B, 64, 1, kBN) ||
        !make_bf16_map_4d(&p.tm_v, a.v, kDv, L.Hkv, a.S, a.S, a.B, 64, 1, kBN))
        return cudaErrorInvalidValue;
    p.out = reinterpret_cast<__nv_bfloat16 *>(a.out);
    p.positions = a.positions;
    p.sinks = L.sinks;
    p.err = a.err;
    p.S = a.S;
    p.Hq = L.Hq;
    p.G = L.G;
    p.gp = gp;
    p.P = P;
    p.window = L.window;
    p.is_swa = L.layer_type == 1;
    p.num_p_tiles = (a.S + P - 1) / P;
    p.num_g_tiles = L.G / gp;
    p.scale_log2 = L.scale_log2;
    p.v_scale = L.v_scale;
    p.rope = L.rope;

    static std::atomic<unsigned long long> prepared{0};
    cudaError_t e = prepare_kernel_once(prefill_tc_kernel<kBN, kStages>, TileCfg<kBN, kStages>::kSmemBytes, prepared);
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.num_p_tiles, L.Hkv * p.num_g_tiles, a.B);
    prefill_tc_kernel<kBN, kStages><<<grid, kThreads, TileCfg<kBN, kStages>::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

} // namespace mimo
