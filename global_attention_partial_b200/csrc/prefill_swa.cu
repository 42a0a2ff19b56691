// Prefill attention of a sliding-window MiMo-V2-Flash layer on the sm_100a
// tensor cores: a persistent kernel that streams the keys through a ring.
//
// A tile is 128 query rows = P positions x gp query heads of one KV group
// (gp = 8, P = 16 for the MiMo layer). Keys are handled in blocks of 16. The
// tile's visible keys [p0 - W + 1, p0 + P - 1] lie in at most 9 consecutive
// blocks (144 keys), so one QK^T and one PV per tile suffice: no online
// rescaling, one softmax pass.
//
// Each CTA takes a contiguous range of tiles. Consecutive tiles of one KV
// group share all but P/16 of their key blocks, so K and V enter shared
// memory through a ring of 16-key blocks: each block is loaded once per CTA
// and freed after the PV of the last tile that uses it. Q tiles stream through
// two buffers.
//
// Two worker warpgroups take alternate tiles (tile n goes to warpgroup n % 2),
// so one softmax overlaps the other tile's MMAs and epilogue. A worker
// rotates its Q tile (partial RoPE, in place in swizzled shared memory, cos /
// sin from the table kprep wrote), runs the softmax (thread r owns row r: the
// row's 144 S values from TMEM, window mask, max, P as bf16 over the S
// columns), then the epilogue (O from TMEM, sink fold, normalise, V scale,
// store). Both workers run the same code, which keeps the instruction cache
// warm.
//
// Warp roles (384 threads = 3 warpgroups; setmaxnreg moves registers from the
// control warpgroup to the workers):
//   warps 0-3   worker for even tiles    warps 4-7   worker for odd tiles
//   warp 8      TMA producer: Q tiles and K/V ring blocks
//   warp 9      MMA issuer: QK^T and PV of the tiles in flight, in whichever
//               order their inputs become ready
//   warps 10-11 idle
//
// TMEM (512 columns), per worker t: S_t = [256t, 256t + 144) and
// O_t = [256t + 72, 256t + 200). O overlaps the upper S columns, which are
// dead once the softmax has read them; P (bf16) takes the first 72 columns.
// Shared memory: Q 2 x 48 KB; K ring 12 x 16 keys x 384 B; V ring 12 x 16
// keys x 256 B (128B-swizzled 64-column blocks, 1024-byte aligned).
#include "kernels.cuh"

#include <math.h>

namespace mimo {
namespace {

constexpr int kBlockM = 128;
constexpr int kKeyBlock = 16;
constexpr int kMaxSpanBlocks = 9;  // 144 keys
constexpr int kRing = 12;          // ring entries of 16 keys
constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kThreads = 384;
// Register split across the three warpgroups. The block launches with
// kThreads x kLaunchRegs registers (ptxas must report exactly kLaunchRegs);
// the shares below add up to that pool: 128 * (208 + 208 + 88) = 384 * 168.
constexpr int kLaunchRegs = 168;
constexpr int kRegsWorker = 208;
constexpr int kRegsControl = 88;
static_assert(128 * (2 * kRegsWorker + kRegsControl) == kThreads * kLaunchRegs,
              "warpgroup register shares must add up to the launch pool");
constexpr int kQBytes = kBlockM * kDqk * 2;             // 49152
constexpr int kKAtom = kRing * kKeyBlock * 128;         // 24576: one 64-column block of the K ring
constexpr int kVAtom = kRing * kKeyBlock * 128;         // 24576
constexpr int kKBytes = 3 * kKAtom;
constexpr int kVBytes = 2 * kVAtom;
constexpr int kEntryBytes = kKeyBlock * (kDqk + kDv) * 2;  // 10240
constexpr int kTmemCols = 512;

__device__ __forceinline__ uint32_t col_s(int t) { return t ? 256u : 0u; }
__device__ __forceinline__ uint32_t col_o(int t) { return col_s(t) + 72u; }

struct SwaParams {
    CUtensorMap tm_q;  // [B, S, Hq, Dqk]    box {64, gp, P, 1}
    CUtensorMap tm_k;  // [B, S, Hkv, Dqk]   box {64, 1, 16, 1}
    CUtensorMap tm_v;  // [B, S, Hkv, Dv]    box {64, 1, 16, 1}
    __nv_bfloat16 *out;
    const float2 *rope_table;  // [S][half] (cos, sin) of each token's position
    const float *sinks;
    unsigned *err;
    int S, Hq, Hkv, G, gp, P, window;
    int num_p_tiles, num_g_tiles, num_tiles, tiles_per_cta;
    int rope_half;
    float scale_log2;
    float v_scale;
};

struct Bars {
    uint64_t q_full[2], q_ready[2], q_empty[2];
    uint64_t kv_full[kRing], kv_empty[kRing];
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr int kSmemBytes = 1024 + 2 * kQBytes + kKBytes + kVBytes + (int)sizeof(Bars) + 64;

struct Tile {
    int b, kvh, h0, p0;
    int run;          // (b, kvh, g-tile): tiles of one run share key blocks
    int first_block;  // first 16-key block of the span
    int last_block;   // last block
};

__device__ __forceinline__ Tile tile_at(const SwaParams &p, int t)
{
    Tile c;
    const int pt = t % p.num_p_tiles;
    c.run = t / p.num_p_tiles;
    const int gt = c.run % p.num_g_tiles;
    const int bk = c.run / p.num_g_tiles;
    c.kvh = bk % p.Hkv;
    c.b = bk / p.Hkv;
    c.h0 = c.kvh * p.G + gt * p.gp;
    c.p0 = pt * p.P;
    const int k_lo = c.p0 - p.window + 1;
    c.first_block = k_lo > 0 ? k_lo / kKeyBlock : 0;
    c.last_block = (c.p0 + p.P - 1) / kKeyBlock;
    return c;
}

// Ring bookkeeping shared (and replayed identically) by the producer and
// the MMA issuer: entries are numbered in load order; a run's blocks get
// consecutive entries.
struct RingCursor {
    int run = -1;
    int last_block = -1;
    int base = 0;        // entry of block 0 of the current run
    int next_entry = 0;  // entries pushed so far
    // Advances to tile c; returns the first new block to load (blocks up to
    // c.last_block are new).
    __device__ __forceinline__ int advance(const Tile &c)
    {
        int first_new;
        if (c.run != run) {
            run = c.run;
            base = next_entry - c.first_block;
            first_new = c.first_block;
        } else {
            first_new = last_block + 1;
        }
        next_entry += c.last_block - first_new + 1;
        last_block = c.last_block;
        return first_new;
    }
    __device__ __forceinline__ int entry(int block) const { return base + block; }
};

__global__ void __launch_bounds__(kThreads, 1) prefill_swa_kernel(const __grid_constant__ SwaParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = smem;                  // 2 buffers
    uint8_t *sK = sQ + 2 * kQBytes;      // 3 atoms of the ring
    uint8_t *sV = sK + kKBytes;          // 2 atoms of the ring
    Bars *bars = reinterpret_cast<Bars *>(sV + kVBytes);
    volatile int *abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t_begin = (int)blockIdx.x * p.tiles_per_cta;
    const int t_end = min(p.num_tiles, t_begin + p.tiles_per_cta);
    const int n_local = max(0, t_end - t_begin);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->q_full[i], 1);
            mbar_init(&bars->q_ready[i], 128);
            mbar_init(&bars->q_empty[i], 1);
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 128);
            mbar_init(&bars->o_full[i], 1);
            mbar_init(&bars->o_free[i], 128);
        }
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&bars->kv_full[i], 1);
            mbar_init(&bars->kv_empty[i], 1);
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
    }
    if (warp == 8) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0 && n_local > 0) {
            tma_prefetch_desc(&p.tm_q);
            tma_prefetch_desc(&p.tm_k);
            tma_prefetch_desc(&p.tm_v);
            int last_q[2] = {-1, -1};
            int loaded = 0;  // ring entries issued
            RingCursor cur;
            bool ok = true;
            auto load_q = [&](int n) -> bool {
                const int qb = n & 1;
                if (!mbar_wait(&bars->q_empty[qb], ((uint32_t)(n >> 1) & 1u) ^ 1u, abort_flag, p.err))
                    return false;
                const Tile c = tile_at(p, t_begin + n);
                mbar_arrive_expect_tx(&bars->q_full[qb], kQBytes);
                for (int a = 0; a < 3; ++a)
                    tma_load_4d(sQ + qb * kQBytes + a * (kBlockM * 128), &p.tm_q, &bars->q_full[qb], a * 64,
                                c.h0, c.p0, c.b);
                last_q[qb] = n;
                return true;
            };
            auto load_blocks = [&](int n) -> bool {
                const Tile c = tile_at(p, t_begin + n);
                const int first_new = cur.advance(c);
                for (int blk = first_new; blk <= c.last_block; ++blk) {
                    const int e = loaded;
                    const int slot = e % kRing;
                    if (!mbar_wait(&bars->kv_empty[slot], ((uint32_t)(e / kRing) & 1u) ^ 1u, abort_flag, p.err))
                        return false;
                    mbar_arrive_expect_tx(&bars->kv_full[slot], kEntryBytes);
                    const int key0 = blk * kKeyBlock;
                    for (int a = 0; a < 3; ++a)
                        tma_load_4d(sK + a * kKAtom + slot * (kKeyBlock * 128), &p.tm_k, &bars->kv_full[slot],
                                    a * 64, c.kvh, key0, c.b);
                    for (int a = 0; a < 2; ++a)
                        tma_load_4d(sV + a * kVAtom + slot * (kKeyBlock * 128), &p.tm_v, &bars->kv_full[slot],
                                    a * 64, c.kvh, key0, c.b);
                    ++loaded;
                }
                return true;
            };
            ok = load_q(0) && load_blocks(0);
            if (ok && n_local > 1)
                ok = load_q(1);
            for (int n = 1; ok && n < n_local; ++n) {
                ok = load_blocks(n);
                if (ok && n + 1 < n_local)
                    ok = load_q(n + 1);
            }
            if (*abort_flag) {
                for (int qb = 0; qb < 2; ++qb)
                    if (last_q[qb] >= 0)
                        mbar_drain(&bars->q_full[qb], (uint32_t)(last_q[qb] >> 1) & 1u);
                for (int e = max(0, loaded - kRing); e < loaded; ++e)
                    mbar_drain(&bars->kv_full[e % kRing], (uint32_t)(e / kRing) & 1u);
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0 && n_local > 0) {
            const uint32_t idesc_pv = idesc_bf16_f32(kBlockM, kDv, false, true);
            const uint32_t q_base = smem_u32(sQ);
            const uint32_t k_base = smem_u32(sK);
            const uint32_t v_base = smem_u32(sV);
            // Ring ranges of the tiles in flight (registers only, by parity).
            int first0 = 0, nb0 = 0, first1 = 0, nb1 = 0;
            // Tile walk without divisions: run and first block of tile next_qk.
            const Tile t0 = tile_at(p, t_begin);
            int qk_pt = t0.p0 / p.P;  // position tile of next_qk within its run
            int qk_run = t0.run;
            int qk_base = -t0.first_block;  // entry of block 0 of qk_run
            int qk_last_block = -1;
            int pushed = 0;                 // entries the producer pushes for tiles < next_qk
            int known_full = 0;             // entries [0, known_full) have landed
            int freed = 0;
            int next_qk = 0, next_pv = 0;
            long long t_last = cycles_now();
            uint32_t idle = 0;
            bool ok = true;
            while (ok && next_pv < n_local) {
                bool progressed = false;
                // QK_n needs its worker's S/O columns back (epilogue of tile n-2
                // done, which also implies PV_{n-2} landed), its rotated Q and its keys.
                if (next_qk < n_local && mbar_test_wait(&bars->o_free[next_qk & 1], ((uint32_t)(next_qk >> 1) & 1u) ^ 1u)) {
                    const int n = next_qk;
                    const int qb = n & 1;
                    // Span of tile n in ring entries.
                    const int p0 = qk_pt * p.P;
                    const int k_lo = p0 - p.window + 1;
                    const int fb = k_lo > 0 ? k_lo / kKeyBlock : 0;
                    const int lb = (p0 + p.P - 1) / kKeyBlock;
                    int base = qk_base;
                    int push = pushed;
                    if (qk_last_block < 0) {  // first tile of a run in this CTA
                        base = pushed - fb;
                        push += lb - fb + 1;
                    } else {
                        push += lb - qk_last_block;
                    }
                    const int e0 = base + fb;
                    const int nb = lb - fb + 1;
                    while (known_full < push &&
                           mbar_test_wait(&bars->kv_full[known_full % kRing], (uint32_t)(known_full / kRing) & 1u))
                        ++known_full;
                    if (known_full >= e0 + nb && mbar_test_wait(&bars->q_ready[qb], (uint32_t)(n >> 1) & 1u)) {
                        tc_fence_after();
                        const uint32_t q_addr = q_base + qb * kQBytes;
                        const int s0 = e0 % kRing;
                        const int run1 = min(nb, kRing - s0);
                        for (int part = 0; part < 2; ++part) {
                            const int blocks = part == 0 ? run1 : nb - run1;
                            if (blocks <= 0)
                                continue;
                            const int slot = part == 0 ? s0 : 0;
                            const uint32_t d = tmem + col_s(qb) + (part == 0 ? 0u : (uint32_t)(run1 * kKeyBlock));
                            const uint32_t idesc = idesc_bf16_f32(kBlockM, blocks * kKeyBlock, false, false);
#pragma unroll
                            for (int kk = 0; kk < kDqk / 16; ++kk) {
                                const int atom = kk >> 2;
                                const uint32_t off = (uint32_t)(kk & 3) * 32u;
                                umma_ss(d, sdesc_sw128(q_addr + atom * (kBlockM * 128) + off, 16, 1024),
                                        sdesc_sw128(k_base + atom * kKAtom + slot * (kKeyBlock * 128) + off, 16, 1024),
                                        idesc, kk > 0 ? 1u : 0u);
                            }
                        }
                        umma_commit(&bars->s_full[qb]);
                        umma_commit(&bars->q_empty[qb]);
                        if (qb) {
                            first1 = e0;
                            nb1 = nb;
                        } else {
                            first0 = e0;
                            nb0 = nb;
                        }
                        // advance the walk to the next tile
                        pushed = push;
                        qk_base = base;
                        qk_last_block = lb;
                        if (++qk_pt == p.num_p_tiles) {
                            qk_pt = 0;
                            ++qk_run;
                            qk_last_block = -1;
                        }
                        ++next_qk;
                        progressed = true;
                    }
                }
                if (next_pv < next_qk) {
                    const int n = next_pv;
                    const int sb = n & 1;
                    if (mbar_test_wait(&bars->p_full[sb], (uint32_t)(n >> 1) & 1u)) {
                        tc_fence_after();
                        const int e0 = sb ? first1 : first0;
                        const int nb = sb ? nb1 : nb0;
                        for (int j = 0; j < nb; ++j) {
                            const int slot = (e0 + j) % kRing;
                            umma_ts(tmem + col_o(sb), tmem + col_s(sb) + j * 8,
                                    sdesc_sw128(v_base + slot * (kKeyBlock * 128), kVAtom, 1024), idesc_pv,
                                    j > 0 ? 1u : 0u);
                        }
                        umma_commit(&bars->o_full[sb]);
                        // Release the ring entries no later tile uses: all of them
                        // unless tile n+1 (already walked by the QK side when it is
                        // in flight, else computed here) continues the same run.
                        int keep_from = e0 + nb;
                        if (n + 1 < n_local) {
                            int nfirst;
                            if (n + 1 < next_qk) {
                                nfirst = sb ? first0 : first1;
                            } else {
                                // tile n+1 not walked yet: same run iff its walk state continues
                                const int p0 = qk_pt * p.P;
                                const int k_lo = p0 - p.window + 1;
                                const int fb = k_lo > 0 ? k_lo / kKeyBlock : 0;
                                nfirst = qk_last_block < 0 ? e0 + nb : qk_base + fb;
                            }
                            keep_from = min(keep_from, nfirst);
                        }
                        for (; freed < keep_from; ++freed)
                            umma_commit(&bars->kv_empty[freed % kRing]);
                        ++next_pv;
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = 0;
                } else {
                    // Nothing ready: yield the issue slots to the softmax warp
                    // sharing this SM sub-partition, and bound the wait.
                    __nanosleep(32);
                    if (idle++ == 0)
                        t_last = cycles_now();
                    if (*abort_flag) {
                        ok = false;
                    } else if ((idle & 63u) == 0 && cycles_now() - t_last > kWaitLimitCycles) {
                        *abort_flag = 1;
                        atomicOr(p.err, kErrTimeout);
                        ok = false;
                    }
                }
            }
            if (!ok) {
                umma_commit(&bars->drain);
                mbar_drain(&bars->drain, 0);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ workers
        setmaxnreg_inc<kRegsWorker>();
        const int t = warp >> 2;             // this worker takes tiles n with n % 2 == t
        const int row = threadIdx.x & 127;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t s_addr = lane_base + col_s(t);
        const uint32_t o_addr = lane_base + col_o(t);
        const int half = p.rope_half;
        const float sc = p.scale_log2;
        bool ok = true;
        for (int n = t; ok && n < n_local; n += 2) {
            const uint32_t ph = (uint32_t)(n >> 1) & 1u;
            const Tile c = tile_at(p, t_begin + n);
            const int i = c.p0 + row / p.gp;
            const int h = c.h0 + row % p.gp;
            // ---- partial RoPE of this row of Q_n (buffer t)
            // cos/sin of the row's 32 pairs are fetched before waiting for Q,
            // so their latency overlaps the Q load.
            const bool fast_rope = half == 32 && i < p.S;
            float4 tb[16];
            if (fast_rope) {
                const float4 *cs4 = reinterpret_cast<const float4 *>(p.rope_table + (size_t)i * half);
#pragma unroll
                for (int w = 0; w < 16; ++w)
                    tb[w] = __ldg(cs4 + w);
            }
            if (!mbar_wait(&bars->q_full[t], ph, abort_flag, p.err)) {
                ok = false;
                break;
            }
            if (i < p.S && half > 0) {
                uint8_t *q_row = sQ + t * kQBytes + row * 128;
                const float2 *cs = p.rope_table + (size_t)i * half;
                if (fast_rope) {
                    // One 128-byte swizzled row: chunks 0-3 hold dims 0-31, 4-7 dims 32-63.
                    uint4 v[8];
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        v[ch] = *reinterpret_cast<const uint4 *>(q_row + ((ch ^ (row & 7)) << 4));
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t *a = reinterpret_cast<uint32_t *>(&v[ch]);
                        uint32_t *bb = reinterpret_cast<uint32_t *>(&v[ch + 4]);
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const float2 xa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&a[w]));
                            const float2 xb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&bb[w]));
                            const float4 cc = tb[ch * 4 + w];  // (cos, sin) of pairs 8ch+2w, 8ch+2w+1
                            a[w] = pack_bf16x2(xa.x * cc.x - xb.x * cc.y, xa.y * cc.z - xb.y * cc.w);
                            bb[w] = pack_bf16x2(xb.x * cc.x + xa.x * cc.y, xb.y * cc.z + xa.y * cc.w);
                        }
                    }
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<uint4 *>(q_row + ((ch ^ (row & 7)) << 4)) = v[ch];
                } else {
                    for (int j = 0; j < half; ++j) {
                        const int ea = j, eb = j + half;
                        __nv_bfloat16 *pa = reinterpret_cast<__nv_bfloat16 *>(
                            sQ + t * kQBytes + (ea >> 6) * (kBlockM * 128) + row * 128 +
                            ((((ea & 63) >> 3) ^ (row & 7)) << 4) + ((ea & 7) << 1));
                        __nv_bfloat16 *pb = reinterpret_cast<__nv_bfloat16 *>(
                            sQ + t * kQBytes + (eb >> 6) * (kBlockM * 128) + row * 128 +
                            ((((eb & 63) >> 3) ^ (row & 7)) << 4) + ((eb & 7) << 1));
                        const float xa = __bfloat162float(*pa);
                        const float xb = __bfloat162float(*pb);
                        const float2 cj = __ldg(cs + j);
                        *pa = __float2bfloat16_rn(xa * cj.x - xb * cj.y);
                        *pb = __float2bfloat16_rn(xb * cj.x + xa * cj.y);
                    }
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->q_ready[t]);

            // ---- softmax over the tile's key span
            const int k0 = c.first_block * kKeyBlock;
            const int lo = i - p.window + 1 - k0;      // first visible column
            const unsigned span = (unsigned)(p.window - 1);  // column c visible iff c - lo <= span
            if (!mbar_wait(&bars->s_full[t], ph, abort_flag, p.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float x[kMaxSpanBlocks * kKeyBlock];
            {
                uint32_t r[kMaxSpanBlocks][16];
#pragma unroll
                for (int q = 0; q < kMaxSpanBlocks; ++q)
                    tmem_ld16(s_addr + 16 * q, r[q]);
                tmem_wait_ld_only();
#pragma unroll
                for (int q = 0; q < kMaxSpanBlocks; ++q) {
                    tmem_tie(r[q]);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        x[16 * q + e] = __uint_as_float(r[q][e]);
                }
            }
            float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int col = 0; col < kMaxSpanBlocks * kKeyBlock; ++col) {
                x[col] = ((unsigned)(col - lo) <= span) ? x[col] : -INFINITY;
                mxv[col & 3] = fmaxf(mxv[col & 3], x[col]);
            }
            const float mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3]));
            const float m2 = mx * sc;   // base-2 units
            const float mu = (mx == -INFINITY) ? 0.f : m2;
            float rsv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < kMaxSpanBlocks; ++q) {
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float e0 = fast_exp2(fmaf(x[16 * q + 2 * e], sc, -mu));
                    const float e1 = fast_exp2(fmaf(x[16 * q + 2 * e + 1], sc, -mu));
                    rsv[e & 3] += e0 + e1;
                    pk[e] = pack_bf16x2(e0, e1);
                }
                tmem_st8(s_addr + 8 * q, pk);
            }
            const float rs = (rsv[0] + rsv[1]) + (rsv[2] + rsv[3]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[t]);

            // ---- epilogue
            float o_scale;
            if (p.sinks != nullptr) {
                const float s2 = __ldg(p.sinks + h) * kLog2e;
                const float mf = fmaxf(m2, s2);
                const float a = exp2f(m2 - mf);
                o_scale = a * p.v_scale / (rs * a + exp2f(s2 - mf));
            } else {
                o_scale = p.v_scale / rs;
            }
            if (!mbar_wait(&bars->o_full[t], ph, abort_flag, p.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t o[4][32];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tmem_ld32(o_addr + 32 * q, o[q]);
            tmem_wait_ld_only();
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tmem_tie(o[q]);
            tc_fence_before();
            mbar_arrive(&bars->o_free[t]);
            if (i < p.S) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (((size_t)c.b * p.S + i) * p.Hq + h) * kDv);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(o[q][c8 * 8 + 0]) * o_scale, __uint_as_float(o[q][c8 * 8 + 1]) * o_scale);
                        w.y = pack_bf16x2(__uint_as_float(o[q][c8 * 8 + 2]) * o_scale, __uint_as_float(o[q][c8 * 8 + 3]) * o_scale);
                        w.z = pack_bf16x2(__uint_as_float(o[q][c8 * 8 + 4]) * o_scale, __uint_as_float(o[q][c8 * 8 + 5]) * o_scale);
                        w.w = pack_bf16x2(__uint_as_float(o[q][c8 * 8 + 6]) * o_scale, __uint_as_float(o[q][c8 * 8 + 7]) * o_scale);
                        dst[q * 4 + c8] = w;
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

// Query heads of one KV group packed into a 128-row tile.
int swa_heads_per_tile(const LayerArgs &L)
{
    int gp = 1;
    for (int c = 16; c >= 2; c >>= 1)
        if (L.G % c == 0) {
            gp = c;
            break;
        }
    return gp;
}

bool prefill_swa_supported(const LayerArgs &L)
{
    if (L.layer_type != 1 || L.Dqk != kDqk || L.Dv != kDv || L.rope.rotary_dim > kDqk)
        return false;
    const int P = kBlockM / swa_heads_per_tile(L);
    if (P % kKeyBlock != 0)
        return false;
    // Worst-case block-aligned span of a tile: the window rounded up to whole
    // blocks plus the tile's own positions.
    const int span = ((L.window - 1 + kKeyBlock - 1) / kKeyBlock) * kKeyBlock + P;
    return span <= kMaxSpanBlocks * kKeyBlock;
}

cudaError_t launch_prefill_swa(const LayerArgs &L, const PrefillArgs &a, const float2 *rope_table,
                               int num_sms, cudaStream_t stream)
{
    SwaParams p;
    memset(&p, 0, sizeof(p));
    const int gp = swa_heads_per_tile(L);
    const int P = kBlockM / gp;
    if (!make_bf16_map_4d(&p.tm_q, a.q, kDqk, L.Hq, a.S, a.S, a.B, 64, gp, P) ||
        !make_bf16_map_4d(&p.tm_k, a.krot, kDqk, L.Hkv, a.S, a.krot_rows, a.B, 64, 1, kKeyBlock) ||
        !make_bf16_map_4d(&p.tm_v, a.v, kDv, L.Hkv, a.S, a.S, a.B, 64, 1, kKeyBlock))
        return cudaErrorInvalidValue;
    p.out = reinterpret_cast<__nv_bfloat16 *>(a.out);
    p.rope_table = rope_table;
    p.sinks = L.sinks;
    p.err = a.err;
    p.S = a.S;
    p.Hq = L.Hq;
    p.Hkv = L.Hkv;
    p.G = L.G;
    p.gp = gp;
    p.P = P;
    p.window = L.window;
    p.num_p_tiles = (a.S + P - 1) / P;
    p.num_g_tiles = L.G / gp;
    p.num_tiles = p.num_p_tiles * p.num_g_tiles * L.Hkv * a.B;
    p.tiles_per_cta = (p.num_tiles + num_sms - 1) / num_sms;
    p.rope_half = L.rope.half;
    p.scale_log2 = L.scale_log2;
    p.v_scale = L.v_scale;

    static bool attr_set = false;
    if (!attr_set) {
        // The setmaxnreg split assumes the block launches with exactly
        // kLaunchRegs registers per thread; refuse to launch otherwise (a
        // smaller pool would leave setmaxnreg.inc waiting forever).
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, prefill_swa_kernel);
        if (e != cudaSuccess)
            return e;
        if (fa.numRegs != kLaunchRegs)
            return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(prefill_swa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess)
            return e;
        attr_set = true;
    }
    const int grid = (p.num_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta;
    prefill_swa_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

} // namespace mimo
