// Prefill attention of a global (causal) MiMo-V2-Flash layer on the sm_100a
// tensor cores: two query tiles per CTA share every K/V tile.
//
// A CTA owns query tiles A and B: the same 128 positions of two query heads
// of one KV group, so both tiles see the same causal key range and mask, and
// each K/V tile crosses L2 once for 256 query rows.
//
// Shared memory: Q_A and Q_B (2 x 48 KB, loaded once, rotated in place) and a
// ring of 8 entries of 16 KB. Each key tile j (128 keys) occupies 5
// consecutive entries: its K in 3 entries (64 dims each) and its V in 2
// entries (64 value dims each). Entries are released in load order, each after
// the last MMA that reads it, so the next tiles stream in while this one is
// used. Every entry is a 128-byte-swizzled block of 128 rows (the TMA
// SWIZZLE_128B layout): K-major for QK^T, MN-major for PV.
//
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// P (bf16) is written over the S columns it replaces.
//
// MMA order (one thread): QK_A(0), QK_B(0), then for j >= 1:
//   PV_A(j-1), QK_A(j), PV_B(j-1), QK_B(j)
// and finally PV_A(n-1), PV_B(n-1). While softmax A works on S_A(j), the
// tensor cores run PV_B(j-1) and QK_B(j), and the other way round. Because
// the tensor core completes one thread's MMAs in order, S_A(j) being ready
// also means PV_A(j-1) has landed in O_A, so a softmax thread may rescale its
// O row without a further wait.
//
// Warp roles (384 threads = 3 warpgroups; setmaxnreg moves registers from the
// control warpgroup to the two softmax warpgroups):
//   warps 0-3   tile A: RoPE of its Q rows, softmax (thread r owns row r),
//               conditional O rescale, epilogue.
//   warps 4-7   tile B: the same.
//   warp 8      TMA producer.
//   warp 9      MMA issuer (and TMEM owner).
//   warps 10-11 idle.
#include "kernels.cuh"

#include <math.h>

namespace mimo {
namespace {

constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kThreads = 384;
constexpr int kQBytes = kBlockM * kDqk * 2;   // 49152 per tile
constexpr int kEntryBytes = kBlockN * 128;    // 16384: 128 rows x 64 columns
constexpr int kRing = 8;
constexpr int kEntriesPerTile = 5;            // K: 3, V: 2
constexpr int kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;     // log2 units

// Register split: the block launches with kThreads x kLaunchRegs (ptxas must
// report exactly kLaunchRegs); the warpgroup shares add up to that pool.
constexpr int kLaunchRegs = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsControl = 88;
static_assert(128 * (2 * kRegsSoftmax + kRegsControl) == kThreads * kLaunchRegs,
              "warpgroup register shares must add up to the launch pool");

__device__ __forceinline__ uint32_t col_s(int t) { return t ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_o(int t) { return t ? 384u : 256u; }

struct GaParams {
    CUtensorMap tm_q;  // [B, S, Hq, Dqk]     box {64, 1, 128, 1}
    CUtensorMap tm_k;  // [B, rows, Hkv, Dqk] box {64, 1, 128, 1}
    CUtensorMap tm_v;  // [B, S, Hkv, Dv]     box {64, 1, 128, 1}
    __nv_bfloat16 *out;
    int out_v8;                // out is 32-byte aligned: 256-bit stores
    const float2 *rope_table;  // row (past + i): (cos, sin) of the pairs at query i's position
    const float *sinks;        // nullptr on global layers
    const int *past_lens;      // [B] cached tokens before the chunk, or nullptr
    unsigned *err;
    int S, Hq, G, num_p_tiles, num_pairs;
    int key_rows;              // key rows readable per batch (cache capacity when continuing a cache)
    int max_past;              // the RoPE table has max_past + S rows
    int rope_half;
    float scale_log2;
    float v_scale;
};

struct Bars {
    uint64_t q_full, q_ready[2];
    uint64_t k_full[2], v_full[2];    // per key tile (j & 1): all of its K / V entries landed
    uint64_t k_free[2], v_free[2];    // per key tile (j & 1): its K / V entries may be overwritten
    uint64_t s_full[2], p_full[2], pv_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr int kSmemBytes = 1024 + 2 * kQBytes + kRing * kEntryBytes + (int)sizeof(Bars) + 64;
static_assert(kSmemBytes <= 232448, "shared memory");

__global__ void __launch_bounds__(kThreads, 1) prefill_ga_kernel(const __grid_constant__ GaParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = smem;                  // Q_A, Q_B
    uint8_t *sRing = sQ + 2 * kQBytes;   // kRing entries
    Bars *bars = reinterpret_cast<Bars *>(sRing + kRing * kEntryBytes);
    volatile int *abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Launch order (x fastest): the query-head pairs of one KV head, then the
    // position tiles with the heaviest causal range first, then (KV head,
    // batch). The CTAs resident together read one K/V stream, and every
    // group's heaviest tiles start with the group, not at the end of the grid.
    const int pt = p.num_p_tiles - 1 - (int)blockIdx.y;
    const int hkv = p.num_pairs / (p.G / 2);
    const int kvh = (int)blockIdx.z % hkv;
    const int b = (int)blockIdx.z / hkv;
    const int hA = kvh * p.G + 2 * (int)blockIdx.x;
    const int p0 = pt * kBlockM;
    const int q_last = min(p0 + kBlockM, p.S) - 1;
    // Query i is the token at key index past + i (past = 0 for a plain prefill).
    const int past = p.past_lens != nullptr ? __ldg(p.past_lens + b) : 0;
    if (past < 0 || past > p.max_past || past + p.S > p.key_rows) {  // the whole CTA leaves before any setup
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
            atomicOr(p.err, kErrKvLen);
        return;
    }
    const int n_tiles = (q_last + past) / kBlockN + 1;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->q_ready[t], 128);
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_full[t], 128);
            mbar_init(&bars->pv_done[t], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->k_full[x], 1);
            mbar_init(&bars->v_full[x], 1);
            mbar_init(&bars->k_free[x], 1);
            mbar_init(&bars->v_free[x], 1);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 9) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp >= 8) {
        setmaxnreg_dec<kRegsControl>();
        if (warp == 8 && lane == 0) {
            // -------------------------------------------------- TMA producer
            tma_prefetch_desc(&p.tm_q);
            tma_prefetch_desc(&p.tm_k);
            tma_prefetch_desc(&p.tm_v);
            mbar_arrive_expect_tx(&bars->q_full, 2 * kQBytes);
            for (int t = 0; t < 2; ++t)
                for (int a = 0; a < 3; ++a)
                    tma_load_4d(sQ + t * kQBytes + a * kEntryBytes, &p.tm_q, &bars->q_full, a * 64, hA + t, p0, b);
            // Entry e of the ring (e = 5j + part) may be refilled once entry
            // e - kRing is free; entries are released per key tile (K and V
            // separately), so the wait is on the barrier of the tile that
            // owned it. A tile's K (or V) is issued only once all of its
            // entries are free, so an abort never leaves a tile half issued.
            auto wait_free = [&](int e) -> bool {
                if (e < kRing)
                    return true;
                const int jo = (e - kRing) / kEntriesPerTile;
                const int part = (e - kRing) - jo * kEntriesPerTile;
                uint64_t *bar = part < 3 ? &bars->k_free[jo & 1] : &bars->v_free[jo & 1];
                return mbar_wait(bar, (uint32_t)(jo >> 1) & 1u, abort_flag, p.err);
            };
            int k_armed[2] = {-1, -1}, v_armed[2] = {-1, -1};
            for (int j = 0; j < n_tiles; ++j) {
                const int e = j * kEntriesPerTile;
                if (!(wait_free(e) && wait_free(e + 1) && wait_free(e + 2)))
                    break;
                mbar_arrive_expect_tx(&bars->k_full[j & 1], 3 * kEntryBytes);
                k_armed[j & 1] = j;
                for (int part = 0; part < 3; ++part)
                    tma_load_4d(sRing + ((e + part) % kRing) * kEntryBytes, &p.tm_k, &bars->k_full[j & 1],
                                part * 64, kvh, j * kBlockN, b);
                if (!(wait_free(e + 3) && wait_free(e + 4)))
                    break;
                mbar_arrive_expect_tx(&bars->v_full[j & 1], 2 * kEntryBytes);
                v_armed[j & 1] = j;
                for (int part = 0; part < 2; ++part)
                    tma_load_4d(sRing + ((e + 3 + part) % kRing) * kEntryBytes, &p.tm_v, &bars->v_full[j & 1],
                                part * 64, kvh, j * kBlockN, b);
            }
            if (*abort_flag) {
                mbar_drain(&bars->q_full, 0);
                for (int x = 0; x < 2; ++x) {
                    if (k_armed[x] >= 0)
                        mbar_drain(&bars->k_full[x], (uint32_t)(k_armed[x] >> 1) & 1u);
                    if (v_armed[x] >= 0)
                        mbar_drain(&bars->v_full[x], (uint32_t)(v_armed[x] >> 1) & 1u);
                }
            }
        } else if (warp == 9 && lane == 0) {
            // ---------------------------------------------------- MMA issuer
            // Straight-line issue: one wait per dependency, no branch between
            // the MMAs of a group. On sm_100a a single issuing thread loses
            // tens of cycles per branch or per freshly built descriptor, which
            // is the whole budget of a 128x128x16 MMA (64 cycles), so the
            // descriptors are built once and stepped by adding byte offsets
            // >> 4 to the start-address field (addresses stay below 2^18).
            const uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false, false);
            const uint32_t idesc_pv64 = idesc_bf16_f32(kBlockM, 64, false, true);
            const uint32_t idesc_pv128 = idesc_bf16_f32(kBlockM, 128, false, true);
            const uint32_t q_lo = sdesc_lo(smem_u32(sQ), 16);
            const uint32_t k_lo = sdesc_lo(smem_u32(sRing), 16);
            const uint32_t v_lo = sdesc_lo(smem_u32(sRing), kEntryBytes);
            constexpr uint32_t kStep = kEntryBytes >> 4;
            bool ok = true;
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                if (!mbar_try_wait(bar, parity) && !mbar_wait(bar, parity, abort_flag, p.err))
                    ok = false;
            };
            // S_t = Q_t K_j^T: 3 entries x 4 k-steps of 16.
            auto qk = [&](int t, int j) {
                const int e = j * kEntriesPerTile;
                const uint32_t qa = q_lo + (uint32_t)t * (kQBytes >> 4);
                const uint32_t kb0 = k_lo + (uint32_t)(e % kRing) * kStep;
                const uint32_t kb1 = k_lo + (uint32_t)((e + 1) % kRing) * kStep;
                const uint32_t kb2 = k_lo + (uint32_t)((e + 2) % kRing) * kStep;
                const uint32_t d = tmem + col_s(t);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                    umma_ss_lo(d, qa + 2 * k4, kb0 + 2 * k4, idesc_qk, k4 ? 1u : 0u);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                    umma_ss_lo(d, qa + kStep + 2 * k4, kb1 + 2 * k4, idesc_qk, 1u);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                    umma_ss_lo(d, qa + 2 * kStep + 2 * k4, kb2 + 2 * k4, idesc_qk, 1u);
            };
            // O_t (+)= P_t V_j: P from the S_t columns of TMEM, V from its two entries.
            auto pv = [&](int t, int j) {
                const int s0 = (j * kEntriesPerTile + 3) % kRing;
                const uint32_t o = tmem + col_o(t), a = tmem + col_s(t);
                const uint32_t acc0 = j > 0 ? 1u : 0u;
                if (s0 + 1 < kRing) {
                    // both halves in adjacent entries: one N = 128 MMA per 16 keys
                    const uint32_t vb = v_lo + (uint32_t)s0 * kStep;
                    umma_ts_lo(o, a, vb, idesc_pv128, acc0);
#pragma unroll
                    for (int kk = 1; kk < kBlockN / 16; ++kk)
                        umma_ts_lo(o, a + kk * 8, vb + kk * (2048 >> 4), idesc_pv128, 1u);
                } else {
                    // the pair wraps around the ring: one N = 64 MMA per half
                    const uint32_t vb0 = v_lo + (uint32_t)s0 * kStep, vb1 = v_lo;
                    umma_ts_lo(o, a, vb0, idesc_pv64, acc0);
#pragma unroll
                    for (int kk = 1; kk < kBlockN / 16; ++kk)
                        umma_ts_lo(o, a + kk * 8, vb0 + kk * (2048 >> 4), idesc_pv64, 1u);
                    umma_ts_lo(o + 64, a, vb1, idesc_pv64, acc0);
#pragma unroll
                    for (int kk = 1; kk < kBlockN / 16; ++kk)
                        umma_ts_lo(o + 64, a + kk * 8, vb1 + kk * (2048 >> 4), idesc_pv64, 1u);
                }
            };
            wait(&bars->q_ready[0], 0);
            wait(&bars->q_ready[1], 0);
            wait(&bars->k_full[0], 0);
            tc_fence_after();
            qk(0, 0);
            umma_commit(&bars->s_full[0]);
            qk(1, 0);
            umma_commit(&bars->k_free[0]);
            umma_commit(&bars->s_full[1]);
            for (int j = 1; ok && j < n_tiles; ++j) {
                const int i = j - 1;
                // tile A: PV_A(j-1), QK_A(j)
                wait(&bars->p_full[0], (uint32_t)i & 1u);
                wait(&bars->v_full[i & 1], (uint32_t)(i >> 1) & 1u);
                tc_fence_after();
                pv(0, i);
                wait(&bars->k_full[j & 1], (uint32_t)(j >> 1) & 1u);
                qk(0, j);
                umma_commit(&bars->s_full[0]);
                // tile B: PV_B(j-1), QK_B(j); it is the last reader of both tiles
                wait(&bars->p_full[1], (uint32_t)i & 1u);
                tc_fence_after();
                pv(1, i);
                umma_commit(&bars->v_free[i & 1]);
                qk(1, j);
                umma_commit(&bars->k_free[j & 1]);
                umma_commit(&bars->s_full[1]);
            }
            if (ok) {
                const int i = n_tiles - 1;
                wait(&bars->p_full[0], (uint32_t)i & 1u);
                wait(&bars->v_full[i & 1], (uint32_t)(i >> 1) & 1u);
                tc_fence_after();
                pv(0, i);
                umma_commit(&bars->pv_done[0]);
                wait(&bars->p_full[1], (uint32_t)i & 1u);
                tc_fence_after();
                pv(1, i);
                umma_commit(&bars->v_free[i & 1]);
                umma_commit(&bars->pv_done[1]);
            }
            if (!ok) {
                umma_commit(&bars->drain);
                mbar_drain(&bars->drain, 0);
            }
        }
    } else {
        // ------------------------------------------ softmax of tile t (A or B)
        setmaxnreg_inc<kRegsSoftmax>();
        const int t = warp >> 2;
        const int row = threadIdx.x & 127;
        const int i = p0 + row;              // sequence index of this row
        const int h = hA + t;
        const bool row_valid = i < p.S;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        bool ok = mbar_wait(&bars->q_full, 0, abort_flag, p.err);

        // Partial RoPE of this row of Q_t, in place in swizzled shared memory.
        const int half = p.rope_half;
        if (ok && row_valid && half > 0) {
            uint8_t *qt = sQ + t * kQBytes;
            const float2 *cs = p.rope_table + (size_t)(past + i) * half;
            for (int j = 0; j < half; ++j) {
                const int ea = j, eb = j + half;
                __nv_bfloat16 *pa = reinterpret_cast<__nv_bfloat16 *>(
                    qt + (ea >> 6) * kEntryBytes + row * 128 + ((((ea & 63) >> 3) ^ (row & 7)) << 4) + ((ea & 7) << 1));
                __nv_bfloat16 *pb = reinterpret_cast<__nv_bfloat16 *>(
                    qt + (eb >> 6) * kEntryBytes + row * 128 + ((((eb & 63) >> 3) ^ (row & 7)) << 4) + ((eb & 7) << 1));
                const float xa = __bfloat162float(*pa);
                const float xb = __bfloat162float(*pb);
                const float2 c = __ldg(cs + j);
                *pa = __float2bfloat16_rn(xa * c.x - xb * c.y);
                *pb = __float2bfloat16_rn(xb * c.x + xa * c.y);
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars->q_ready[t]);

        float m_ref = -INFINITY;  // reference max (base-2 units) of P and O
        float l_sum = 0.f;
        const uint32_t s_addr = lane_base + col_s(t);
        const uint32_t o_addr = lane_base + col_o(t);
        for (int j = 0; ok && j < n_tiles; ++j) {
            if (!mbar_wait(&bars->s_full[t], (uint32_t)j & 1u, abort_flag, p.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float x[kBlockN];
            {
                uint32_t r[kBlockN / 32][32];
#pragma unroll
                for (int c = 0; c < kBlockN / 32; ++c)
                    tmem_ld32(s_addr + 32 * c, r[c]);
                tmem_wait_ld_only();
#pragma unroll
                for (int c = 0; c < kBlockN / 32; ++c) {
                    tmem_tie(r[c]);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        x[32 * c + e] = __uint_as_float(r[c][e]);  // raw scores; scale folded below
                }
            }
            const int k0 = j * kBlockN;
            if (k0 + kBlockN - 1 > p0 + past) {
                // diagonal tile: key c visible iff k0 + c <= past + i (branch-free)
                const int hi = past + i - k0;
#pragma unroll
                for (int c = 0; c < kBlockN; ++c)
                    x[c] = (c <= hi) ? x[c] : -INFINITY;
            }
            float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < kBlockN; ++c)
                mxv[c & 3] = fmaxf(mxv[c & 3], x[c]);
            const float mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])) * p.scale_log2;
            // A row moves its reference max when the tile's max exceeds it by
            // more than the threshold; corr rescales what was summed against
            // the old one. O already holds P*V of tiles < j (in-order MMAs).
            // The TMEM load and store are warp-collective (.sync.aligned), so
            // the whole warp rescales whenever one of its rows moved (the
            // others by 1), 16 columns at a time.
            const bool move = mx > m_ref + kRescaleThreshold || (m_ref == -INFINITY && mx > -INFINITY);
            if (__any_sync(0xffffffffu, move)) {
                const float corr = !move ? 1.f : (m_ref == -INFINITY ? 0.f : fast_exp2(m_ref - mx));
                if (j > 0 && __any_sync(0xffffffffu, move && m_ref != -INFINITY)) {
                    const float f = (m_ref == -INFINITY) ? 1.f : corr;
#pragma unroll 1
                    for (int c0 = 0; c0 < kDv; c0 += 16) {
                        uint32_t r[16];
                        tmem_ld16(o_addr + c0, r);
                        tmem_wait_ld_only();
                        tmem_tie(r);
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            r[c] = __float_as_uint(__uint_as_float(r[c]) * f);
                        tmem_st16(o_addr + c0, r);
                    }
                }
                if (move) {
                    l_sum *= corr;
                    m_ref = mx;
                }
            }
            const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
            const float sc = p.scale_log2;
            float rsv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c0 = 0; c0 < kBlockN; c0 += 64) {
                uint32_t r[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float e0 = fast_exp2(fmaf(x[c0 + 2 * c], sc, -m_use));
                    const float e1 = fast_exp2(fmaf(x[c0 + 2 * c + 1], sc, -m_use));
                    rsv[c & 3] += e0 + e1;
                    r[c] = pack_bf16x2(e0, e1);
                }
                tmem_st32(s_addr + c0 / 2, r);
            }
            l_sum += (rsv[0] + rsv[1]) + (rsv[2] + rsv[3]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[t]);
        }

        // ----------------------------------------------------------- epilogue
        if (ok && mbar_wait(&bars->pv_done[t], 0, abort_flag, p.err)) {
            tc_fence_after();
            float o_scale;
            if (p.sinks != nullptr) {
                const float s2 = __ldg(p.sinks + h) * kLog2e;
                const float m_fin = fmaxf(m_ref, s2);
                const float a = exp2f(m_ref - m_fin);
                o_scale = a * p.v_scale / (l_sum * a + exp2f(s2 - m_fin));
            } else {
                o_scale = p.v_scale / l_sum;
            }
            uint32_t o[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld32(o_addr + 32 * c, o[c]);
            tmem_wait_ld_only();
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_tie(o[c]);
            if (row_valid) {
                uint8_t *dst = reinterpret_cast<uint8_t *>(p.out + (((size_t)b * p.S + i) * p.Hq + h) * kDv);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            w[e] = pack_bf16x2(__uint_as_float(o[c][hh * 16 + 2 * e]) * o_scale,
                                               __uint_as_float(o[c][hh * 16 + 2 * e + 1]) * o_scale);
                        st_global_32B(dst + (c * 2 + hh) * 32, w, p.out_v8 != 0);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

} // namespace

bool prefill_ga_supported(const LayerArgs &L)
{
    return L.layer_type == 0 && L.Dqk == kDqk && L.Dv == kDv && L.G % 2 == 0 && L.rope.rotary_dim <= kDqk;
}

cudaError_t launch_prefill_ga(const LayerArgs &L, const PrefillArgs &a, cudaStream_t stream)
{
    GaParams p;
    memset(&p, 0, sizeof(p));
    if (!make_bf16_map_4d(&p.tm_q, a.q, kDqk, L.Hq, a.S, a.S, a.B, 64, 1, kBlockM) ||
        !make_bf16_map_4d(&p.tm_k, a.krot, kDqk, L.Hkv, a.key_rows_valid, a.krot_rows, a.B, 64, 1, kBlockN) ||
        !make_bf16_map_4d(&p.tm_v, a.v, kDv, L.Hkv, a.key_rows_valid, a.v_rows, a.B, 64, 1, kBlockN))
        return cudaErrorInvalidValue;
    p.out = reinterpret_cast<__nv_bfloat16 *>(a.out);
    p.out_v8 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
    p.rope_table = a.rope_table;
    p.sinks = L.sinks;
    p.past_lens = a.past_lens;
    p.err = a.err;
    p.S = a.S;
    p.key_rows = (int)a.key_rows_valid;
    p.max_past = a.past_lens != nullptr ? a.max_past : 0;
    p.Hq = L.Hq;
    p.G = L.G;
    p.num_p_tiles = (a.S + kBlockM - 1) / kBlockM;
    p.num_pairs = L.Hkv * (L.G / 2);
    p.rope_half = L.rope.half;
    p.scale_log2 = L.scale_log2;
    p.v_scale = L.v_scale;

    // The setmaxnreg split needs a launch with exactly kLaunchRegs registers.
    static std::atomic<unsigned long long> prepared{0};
    cudaError_t e = prepare_kernel_once(prefill_ga_kernel, kSmemBytes, prepared, kLaunchRegs);
    if (e != cudaSuccess)
        return e;
    if (p.num_p_tiles > 65535 || (long long)L.Hkv * a.B > 65535)
        return cudaErrorInvalidValue;
    dim3 grid(L.G / 2, p.num_p_tiles, L.Hkv * a.B);
    prefill_ga_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

} // namespace mimo
