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
// Two workers take alternate tiles (tile n goes to worker n % 2), so one
// worker's softmax overlaps the other tile's MMAs and epilogue. A worker is
// two warpgroups, one per column half: the thread pair (row r, half 0) and
// (row r, half 1) shares query row r. The pair runs the softmax (each half 72
// of the 144 S columns from TMEM: window mask, max exchanged through shared
// memory, P as bf16 written back over the S columns) and the epilogue (64 of
// the 128 O columns: sink fold, normalise, V scale, store). Between the two,
// while PV runs, it moves the first 64 dims of the row's next Q tile from
// shared memory into TMEM, applying the partial RoPE on the way (cos / sin
// from the per-call table; each half 16 of the 32 pairs): QK^T takes those
// four k-steps' A operand from TMEM and the other eight straight from the Q
// buffer, which its commit then frees. So a tile's QK^T can start as soon as
// the epilogue of the worker's previous tile has read O, and it runs while
// that epilogue's stores drain.
//
// The keys arrive unrotated in a plain prefill: the Q-producer warp rotates
// each 16-key block in the ring once it lands, before any QK^T reads it. (A
// prefill continuing a cache reads a window of rotated keys.)
//
// Warp roles (640 threads = 5 warpgroups; setmaxnreg moves registers from the
// control warpgroup to the workers):
//   warps 0-3 / 4-7     worker 0 (even tiles), column half 0 / half 1
//   warps 8-11 / 12-15  worker 1 (odd tiles), column half 0 / half 1
//   warp 16             TMA producer of the Q tiles; rotates the new key blocks
//   warp 17             MMA issuer of worker 0 (QK^T and PV of the even tiles)
//   warp 18             MMA issuer of worker 1 (the odd tiles)
//   warp 19             TMA producer of the K/V ring blocks
//
// TMEM (512 columns), per worker t: S_t = [256t, 256t + 144),
// O_t = [256t + 72, 256t + 200) and Q_t = [256t + 200, 256t + 232) (dims
// 0 .. 63 as bf16 pairs), X_t = [256t + 232, 256t + 234) (the halves' row
// sums). O overlaps the upper S columns, which are dead once the
// softmax has read them; P (bf16) takes the first 72 columns.
// Shared memory: Q 2 x 48 KB; K ring 11 x 16 keys x 384 B; V ring 11 x 16
// keys x 256 B (128B-swizzled 64-column blocks, 1024-byte aligned); 16 KB of
// O staging.
//
// Epilogue: each warp writes its 32 rows x 64 output columns (scaled, bf16)
// into a 4 KB staging slot and one lane issues a TMA store of them, so the
// warp goes on at once; the slot is released a tile later, once the store
// has read it. Half 0 stages in the first 64-column block of its worker's Q
// buffer (dead once copied into TMEM, refilled only after the release); half
// 1 in a 16 KB region the two workers take in turn. The two halves of a row
// exchange their row maxima through shared memory and their row sums through
// two TMEM columns.
#include "kernels.cuh"

#include <math.h>

namespace mimo {
namespace {

constexpr int kBlockM = 128;
constexpr int kKeyBlock = 16;
constexpr int kMaxSpanBlocks = 9;  // 144 keys
constexpr int kHalfCols = kMaxSpanBlocks * kKeyBlock / 2;  // 72 S columns per thread
constexpr int kRing = 11;          // ring entries of 16 keys
constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kThreads = 640;
constexpr int kWorkerThreads = 256;  // one worker: two warpgroups
// Register split across the five warpgroups. The block launches with
// kThreads x kLaunchRegs registers (ptxas must report exactly kLaunchRegs);
// the shares below add up to that pool: 128 * (4 * 104 + 64) = 640 * 96.
constexpr int kLaunchRegs = 96;
constexpr int kRegsWorker = 104;
constexpr int kRegsControl = 64;
static_assert(128 * (4 * kRegsWorker + kRegsControl) == kThreads * kLaunchRegs,
              "warpgroup register shares must add up to the launch pool");
constexpr int kQBytes = kBlockM * kDqk * 2;             // 49152
constexpr int kKAtom = kRing * kKeyBlock * 128;         // one 64-column block of the K ring
constexpr int kVAtom = kRing * kKeyBlock * 128;
constexpr int kKBytes = 3 * kKAtom;
constexpr int kVBytes = 2 * kVAtom;
constexpr int kEntryBytes = kKeyBlock * (kDqk + kDv) * 2;  // 10240
constexpr int kTmemCols = 512;
constexpr int kWarpQ = 16, kWarpMma0 = 17, kWarpKV = 19;

__device__ __forceinline__ uint32_t col_s(int t) { return t ? 256u : 0u; }
__device__ __forceinline__ uint32_t col_o(int t) { return col_s(t) + 72u; }
__device__ __forceinline__ uint32_t col_q(int t) { return col_s(t) + 200u; }
// Two columns per worker through which the two halves of a row exchange
// their row sums (read together with O).
__device__ __forceinline__ uint32_t col_x(int t) { return col_s(t) + 232u; }

struct SwaParams {
    CUtensorMap tm_q;  // [B, S, Hq, Dqk]    box {64, gp, P, 1}
    CUtensorMap tm_k;  // [B, S, Hkv, Dqk]   box {64, 1, 16, 1}
    CUtensorMap tm_v;  // [B, S, Hkv, Dv]    box {64, 1, 16, 1}
    CUtensorMap tm_o;  // [B, S, Hq, Dv]     box {64, gp, 32 / gp, 1}: one warp's 32 rows, one half
    __nv_bfloat16 *out;
    int o_tma;                 // O through the staging slots and TMA stores, else direct stores
    int out_v8;                // (direct stores) out is 32-byte aligned: 256-bit stores
    const float2 *rope_table;  // row (past + i): (cos, sin) of the pairs at query i's position
    const float *sinks;
    const int *past_lens;      // [B] cached tokens before the chunk, or nullptr
    unsigned *err;
    int S, Hq, Hkv, G, gp, P, window;
    int key_off;               // key index of query 0 (a multiple of 16; 0 for a plain prefill)
    int max_past;
    int num_p_tiles, num_g_tiles, num_tiles, tiles_per_cta;
    int rope_half;
    int rotate_k;              // K arrives unrotated: rotate each ring block in shared memory
    float scale_log2;
    float v_scale;
};

struct Bars {
    uint64_t q_full[2], q_ready[2], q_empty[2];
    uint64_t kv_full[kRing], kv_empty[kRing];
    uint64_t kv_ready[kRing];  // the block's keys are rotated in place (or need no rotation)
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint64_t ost_free[4];  // half 1's staging slot of warp quarter q: the previous tile's store has read it
    uint64_t xchg[2];      // both halves of worker t published their row maxima
    uint64_t qrot[2];      // (generic RoPE only) both halves rotated Q in shared memory
    uint64_t drain[2];
    uint32_t tmem_base;
    int abort;
};

// O staging: a warp's 32 rows x 64 columns (4 KB, 128-byte swizzled rows).
// Half 0 of worker t stages in the first 64-column block of its own Q
// buffer (dead once copied into TMEM); half 1 of both workers shares one
// region, a slot per warp quarter, handed from one tile to the next.
constexpr int kOSlotBytes = 32 * 128;
constexpr int kOStageBytes = 4 * kOSlotBytes;
// Per worker: each half's row maximum per query row.
constexpr int kRedBytes = 2 * 2 * kBlockM * 4;
constexpr int kSmemBytes = 1024 + 2 * kQBytes + kKBytes + kVBytes + kOStageBytes + kRedBytes + (int)sizeof(Bars) + 64;
static_assert(kSmemBytes <= 232448, "shared memory");

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
    const int k_lo = c.p0 + p.key_off - p.window + 1;
    c.first_block = k_lo > 0 ? k_lo / kKeyBlock : 0;
    c.last_block = (c.p0 + p.key_off + p.P - 1) / kKeyBlock;
    return c;
}

// Ring bookkeeping shared (and replayed identically) by the producers and
// the MMA issuers: entries are numbered in load order; a run's blocks get
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

// Partial RoPE of the 16-byte chunk pair (a, b) = dims (8c .. 8c+7,
// 8c+half .. 8c+half+7) of one row: pair 8c + 2w turns by the angle whose
// (cos, sin) cs[w] holds in (x, y), pair 8c + 2w + 1 by (z, w).
__device__ __forceinline__ void rope_chunk_pair(uint4 &va, uint4 &vb, const float4 (&cs)[4])
{
    uint32_t *a = reinterpret_cast<uint32_t *>(&va);
    uint32_t *b = reinterpret_cast<uint32_t *>(&vb);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const float2 xa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&a[w]));
        const float2 xb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&b[w]));
        const float4 cc = cs[w];
        a[w] = pack_bf16x2(xa.x * cc.x - xb.x * cc.y, xa.y * cc.z - xb.y * cc.w);
        b[w] = pack_bf16x2(xb.x * cc.x + xa.x * cc.y, xb.y * cc.z + xa.y * cc.w);
    }
}

__global__ void __launch_bounds__(kThreads, 1) prefill_swa_kernel(const __grid_constant__ SwaParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = smem;                  // 2 buffers
    uint8_t *sK = sQ + 2 * kQBytes;      // 3 atoms of the ring
    uint8_t *sV = sK + kKBytes;          // 2 atoms of the ring
    uint8_t *sOst = sV + kVBytes;        // half 1's O staging (1024-byte aligned)
    float *sRedMax = reinterpret_cast<float *>(sOst + kOStageBytes);  // [worker][half][row]
    Bars *bars = reinterpret_cast<Bars *>(sOst + kOStageBytes + kRedBytes);
    volatile int *abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t_begin = (int)blockIdx.x * p.tiles_per_cta;
    const int t_end = min(p.num_tiles, t_begin + p.tiles_per_cta);
    const int n_local = max(0, t_end - t_begin);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->q_full[i], 1);
            mbar_init(&bars->q_ready[i], kWorkerThreads);
            // QK^T of the tile has read the buffer, and the four half-0 warps
            // have released their O staging in its first block
            mbar_init(&bars->q_empty[i], 1 + 4);
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], kWorkerThreads);
            mbar_init(&bars->o_full[i], 1);
            mbar_init(&bars->o_free[i], kWorkerThreads);
            mbar_init(&bars->xchg[i], kWorkerThreads);
            mbar_init(&bars->qrot[i], kWorkerThreads);
        }
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&bars->kv_full[i], 1);
            mbar_init(&bars->kv_empty[i], 2);  // one commit from each issuer
            mbar_init(&bars->kv_ready[i], 1);
        }
        for (int i = 0; i < 4; ++i)
            mbar_init(&bars->ost_free[i], 1);
        mbar_init(&bars->drain[0], 1);
        mbar_init(&bars->drain[1], 1);
        bars->abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kWarpMma0) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp >= kWarpQ)
        setmaxnreg_dec<kRegsControl>();
    if (warp == kWarpQ) {
        // --------------------------------- TMA producer of Q; key rotation
        // An event loop that never blocks on one stream while the other can
        // move (non-blocking barrier tests, a short sleep when idle): lane 0
        // issues each Q tile into its buffer once the QK^T of the tile two
        // before has read it, and the whole warp rotates (partial RoPE, in
        // place in the ring) each key block as soon as it lands, in ring
        // order, then marks it ready. Each lane takes key rows x 16-byte chunk
        // pairs (c, c + half / 8), i.e. 8 rotary pairs, with cos / sin from
        // the per-call table; the rotary dims all lie in the first 64-column
        // block of the ring entry. Keys that arrive rotated are only marked
        // ready.
        int last_q[2] = {-1, -1};
        RingCursor cur;
        const int nch = p.rope_half >> 3;
        int nq = 0;                     // next Q tile to issue
        int nr = 0;                     // tile whose new key blocks are being processed
        int blk = 0, blk_end = -1;      // its blocks still to process: [blk, blk_end]
        if (n_local > 0) {
            const Tile c0 = tile_at(p, t_begin);
            blk = cur.advance(c0);
            blk_end = c0.last_block;
        }
        long long idle_since = cycles_now();
        const long long limit = wait_limit_of(p.err);
        bool ok = true;
        if (lane == 0 && n_local > 0)
            tma_prefetch_desc(&p.tm_q);
        while (nq < n_local || nr < n_local) {
            bool moved = false;
            if (nq < n_local) {
                int go = 0;
                const int qb = nq & 1;
                if (lane == 0 && mbar_test_wait(&bars->q_empty[qb], ((uint32_t)(nq >> 1) & 1u) ^ 1u)) {
                    const Tile c = tile_at(p, t_begin + nq);
                    mbar_arrive_expect_tx(&bars->q_full[qb], kQBytes);
                    for (int a = 0; a < 3; ++a)
                        tma_load_4d(sQ + qb * kQBytes + a * (kBlockM * 128), &p.tm_q, &bars->q_full[qb], a * 64,
                                    c.h0, c.p0, c.b);
                    last_q[qb] = nq;
                    go = 1;
                }
                if (__shfl_sync(0xffffffffu, go, 0)) {
                    ++nq;
                    moved = true;
                }
            }
            if (nr < n_local) {
                const int e = cur.entry(blk);
                const int slot = e % kRing;
                int go = 0;
                if (lane == 0)
                    go = mbar_test_wait(&bars->kv_full[slot], (uint32_t)(e / kRing) & 1u) ? 1 : 0;
                if (__shfl_sync(0xffffffffu, go, 0)) {
                    for (int item = lane; p.rotate_k && item < kKeyBlock * nch; item += 32) {
                        const int kr = item / nch;
                        const int cp = item - kr * nch;
                        const int u = blk * kKeyBlock + kr;  // key index = sequence index
                        if (u >= p.S)
                            continue;
                        uint8_t *k_row = sK + slot * (kKeyBlock * 128) + kr * 128;
                        uint4 *pa = reinterpret_cast<uint4 *>(k_row + ((cp ^ (kr & 7)) << 4));
                        uint4 *pb = reinterpret_cast<uint4 *>(k_row + (((cp + nch) ^ (kr & 7)) << 4));
                        const float4 *g =
                            reinterpret_cast<const float4 *>(p.rope_table + (size_t)u * p.rope_half + cp * 8);
                        float4 cs[4];
#pragma unroll
                        for (int w = 0; w < 4; ++w)
                            cs[w] = __ldg(g + w);
                        uint4 va = *pa, vb = *pb;
                        rope_chunk_pair(va, vb, cs);
                        *pa = va;
                        *pb = vb;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars->kv_ready[slot]);
                    moved = true;
                    if (++blk > blk_end && ++nr < n_local) {
                        const Tile c = tile_at(p, t_begin + nr);
                        blk = cur.advance(c);
                        blk_end = c.last_block;
                    }
                }
            }
            if (moved) {
                idle_since = cycles_now();
                continue;
            }
            // nothing ready: stop on another thread's abort or after the wait limit
            int stop = 0;
            if (lane == 0) {
                if (*abort_flag) {
                    stop = 1;
                } else if (cycles_now() - idle_since > limit) {
                    *abort_flag = 1;
                    atomicOr(p.err, kErrTimeout);
                    stop = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) {
                ok = false;
                break;
            }
            __nanosleep(64);
        }
        if (lane == 0 && !ok)
            for (int qb = 0; qb < 2; ++qb)
                if (last_q[qb] >= 0)
                    mbar_drain(&bars->q_full[qb], (uint32_t)(last_q[qb] >> 1) & 1u);
    } else if (warp == kWarpKV) {
        // ---------------------------------------------- TMA producer: K/V ring
        // Independent of the Q stream, so key blocks run ahead of the tiles
        // as far as the ring's free entries allow.
        if (lane == 0 && n_local > 0) {
            tma_prefetch_desc(&p.tm_k);
            tma_prefetch_desc(&p.tm_v);
            int loaded = 0;  // ring entries issued
            RingCursor cur;
            bool ok = true;
            for (int n = 0; ok && n < n_local; ++n) {
                const Tile c = tile_at(p, t_begin + n);
                const int first_new = cur.advance(c);
                for (int blk = first_new; blk <= c.last_block; ++blk) {
                    const int e = loaded;
                    const int slot = e % kRing;
                    if (!mbar_wait(&bars->kv_empty[slot], ((uint32_t)(e / kRing) & 1u) ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
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
            }
            if (*abort_flag)
                for (int e = max(0, loaded - kRing); e < loaded; ++e)
                    mbar_drain(&bars->kv_full[e % kRing], (uint32_t)(e / kRing) & 1u);
        }
    } else if (warp >= kWarpQ) {
        // ------------------------------------------------------ MMA issuers
        // Issuer t (warp 17 + t) serves worker t: the tiles n with n % 2 == t,
        // in order, each with blocking waits, so it reacts as soon as an input
        // is ready. Both walk every tile with the producer's ring cursor to
        // number the entries. An entry is free (its kv_empty barrier counts
        // two arrivals) once each issuer has committed it: issuer t commits the
        // entries below the span of a tile before waiting for it and below the
        // span of its next tile after the PV of its current one, and every
        // remaining entry after its last tile. As a tile spans at most 9 of
        // the 11 entries, every entry the producer waits on is then committed
        // by an issuer that is not waiting on that producer.
        const int t = warp - kWarpMma0;
        if (lane == 0 && t < n_local) {
            const uint32_t idesc_pv = idesc_bf16_f32(kBlockM, kDv, false, true);
            const uint32_t k_lo = sdesc_lo(smem_u32(sK), 16);
            const uint32_t v_lo = sdesc_lo(smem_u32(sV), kVAtom);
            const uint32_t q_lo = sdesc_lo(smem_u32(sQ + t * kQBytes), 16);  // this worker's Q buffer
            constexpr uint32_t kQBoxStep = (kBlockM * 128) >> 4;
            constexpr uint32_t kKAtomStep = kKAtom >> 4;
            constexpr uint32_t kSlotStep = (kKeyBlock * 128) >> 4;
            const uint32_t s_col = tmem + col_s(t), o_col = tmem + col_o(t), q_col = tmem + col_q(t);
            bool ok = true;
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                if (!mbar_try_wait(bar, parity) && !mbar_wait(bar, parity, abort_flag, p.err))
                    ok = false;
            };
            RingCursor cur;
            int walked = -1;  // tiles [0, walked] have been walked
            int e0 = 0, nb = 0;
            auto walk_to = [&](int n) {
                while (walked < n) {
                    ++walked;
                    const Tile c = tile_at(p, t_begin + walked);
                    cur.advance(c);
                    e0 = cur.entry(c.first_block);
                    nb = c.last_block - c.first_block + 1;
                }
            };
            // S_t = Q_t K^T over the entries [e0, e0 + nb): groups of 12
            // MMAs (K = 16 dims each) over at most 8 entries (N <= 128 keys:
            // with A in shared memory, N = 144 ran at about half the rate of
            // 128 + 16), split again where the span wraps the ring. The first
            // four k-steps take A from TMEM (dims 0 .. 63, rotated by the
            // workers: 8 columns per k-step), the other eight from the Q
            // buffer's 64-column blocks 1 and 2.
            auto qk_part = [&](uint32_t d0, int slot0, int blocks0) {
                for (int b0 = 0; b0 < blocks0; b0 += 8) {
                    const int blocks = min(8, blocks0 - b0);
                    const uint32_t d = d0 + (uint32_t)(b0 * kKeyBlock);
                    const uint32_t idesc = idesc_bf16_f32(kBlockM, blocks * kKeyBlock, false, false);
                    const uint32_t kb = k_lo + (uint32_t)(slot0 + b0) * kSlotStep;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        umma_ts_lo(d, q_col + (uint32_t)(8 * k4), kb + 2 * k4, idesc, k4 ? 1u : 0u);
#pragma unroll
                    for (int atom = 1; atom < 3; ++atom)
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4)
                            umma_ss_lo(d, q_lo + atom * kQBoxStep + 2 * k4, kb + atom * kKAtomStep + 2 * k4, idesc,
                                       1u);
                }
            };
            int known_full = 0;  // entries [0, known_full) have landed (and are rotated)
            int freed = 0;       // entries [0, freed) committed by this issuer
            walk_to(t);
            for (int n = t; ok && n < n_local; n += 2) {
                const uint32_t ph = (uint32_t)(n >> 1) & 1u;
                // Entries below this tile's span are never read by this issuer
                // again: commit them before waiting, so that the ring can refill
                // while this tile's blocks are still missing (otherwise two
                // tiles of 9 blocks from different runs, one per issuer, could
                // wait on each other's ring).
                for (; freed < e0; ++freed)
                    umma_commit(&bars->kv_empty[freed % kRing]);
                wait(&bars->o_free[t], ph ^ 1u);  // epilogue of tile n - 2 has read O
                wait(&bars->q_ready[t], ph);
                // Only this tile's entries: those below e0 may already be
                // released (and refilled) on behalf of the other worker.
                for (known_full = max(known_full, e0); known_full < e0 + nb; ++known_full) {
                    wait(&bars->kv_full[known_full % kRing], (uint32_t)(known_full / kRing) & 1u);
                    wait(&bars->kv_ready[known_full % kRing], (uint32_t)(known_full / kRing) & 1u);
                }
                tc_fence_after();
                const int s0 = e0 % kRing;
                const int run1 = min(nb, kRing - s0);
                qk_part(s_col, s0, run1);
                if (nb > run1)
                    qk_part(s_col + (uint32_t)(run1 * kKeyBlock), 0, nb - run1);
                umma_commit(&bars->s_full[t]);
                umma_commit(&bars->q_empty[t]);  // the Q buffer may take the worker's next tile
                // O_t = P_t V over the same entries, one N = 128 MMA per entry.
                wait(&bars->p_full[t], ph);
                tc_fence_after();
                int slot = s0;
                for (int j = 0; j < nb; ++j) {
                    umma_ts_lo(o_col, s_col + (uint32_t)(j * 8), v_lo + (uint32_t)slot * kSlotStep, idesc_pv,
                               j > 0 ? 1u : 0u);
                    slot = slot + 1 == kRing ? 0 : slot + 1;
                }
                umma_commit(&bars->o_full[t]);
                // Release what no later tile of this worker reads.
                int keep_from;
                if (n + 2 < n_local) {
                    walk_to(n + 2);
                    keep_from = e0;
                } else {
                    walk_to(n_local - 1);
                    keep_from = cur.next_entry;
                }
                for (; freed < keep_from; ++freed)
                    umma_commit(&bars->kv_empty[freed % kRing]);
            }
            if (!ok) {
                umma_commit(&bars->drain[t]);
                mbar_drain(&bars->drain[t], 0);
            }
        }
    } else {
        // ------------------------------------------------------------ workers
        setmaxnreg_inc<kRegsWorker>();
        const int t = warp >> 3;             // this worker takes tiles n with n % 2 == t
        const int hf = (warp >> 2) & 1;      // column half
        const int row = threadIdx.x & 127;   // = the TMEM lane this warp may access
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t s_addr = lane_base + col_s(t) + (uint32_t)(kHalfCols * hf);
        const uint32_t p_addr = lane_base + col_s(t) + (uint32_t)(kHalfCols / 2 * hf);
        const uint32_t o_addr = lane_base + col_o(t) + (uint32_t)(64 * hf);
        const uint32_t q_addr = lane_base + col_q(t);
        const uint32_t x_addr = lane_base + col_x(t);  // row sum exchange with the other half
        float *red_max = sRedMax + t * (2 * kBlockM);   // [half][row]
        const int wq = warp & 3;                        // this warp's 32 rows of the tile
        uint8_t *const o_stage = hf == 0 ? sQ + t * kQBytes + wq * kOSlotBytes : sOst + wq * kOSlotBytes;
        bool o_used = false;     // (lane 0) this warp wrote o_stage in its last epilogue
        bool o_pending = false;  // (lane 0) ... and a store from it may still be reading it
        // Lane 0 lets the staging slot go once its store has read it: half 0's
        // slot back to the Q buffer's next fill (one of the five arrivals of
        // q_empty, made every tile), half 1's to the other worker's next tile
        // (one arrival per use, a store issued or not).
        auto release_stage = [&](bool every_tile) {
            if (lane == 0) {
                if (o_pending)
                    bulk_wait_read_all();
                if (hf == 0 ? every_tile : o_used)
                    mbar_arrive(hf == 0 ? &bars->q_empty[t] : &bars->ost_free[wq]);
                o_pending = false;
                o_used = false;
            }
        };
        const int half = p.rope_half;
        const float sc = p.scale_log2;
        const bool fast_rope = half == 32 && p.P == 16;
        // Q tile nn's first 64 dims into TMEM (the A operand of the first four
        // k-steps of QK^T; the other eight read the Q buffer), partial RoPE on
        // the way. Half hf takes rotary pairs 16hf .. 16hf + 15: 16-byte
        // chunks 2hf, 2hf + 1 and their partners 4 chunks up. Dims (2c, 2c + 1)
        // form TMEM column c of Q_t. Other rotary widths rotate every rotary
        // dim in place in the buffer first (both halves, then a barrier).
        auto load_q = [&](int nn) -> bool {
            const uint32_t ph = (uint32_t)(nn >> 1) & 1u;
            const Tile c = tile_at(p, t_begin + nn);
            const int i = c.p0 + row / p.gp;
            const int past = p.past_lens != nullptr ? min(max(__ldg(p.past_lens + c.b), 0), p.max_past) : 0;
            const bool rot = i < p.S && half > 0;
            if (!mbar_wait(&bars->q_full[t], ph, abort_flag, p.err))
                return false;
            uint8_t *q_row = sQ + t * kQBytes + row * 128;
            if (half > 0 && !fast_rope) {
                // every thread arrives, rows past the sequence end included
                const float2 *cs = p.rope_table + (size_t)(past + i) * half;
                for (int j = hf; rot && j < half; j += 2) {
                    const int ea = j, eb = j + half;
                    __nv_bfloat16 *pa = reinterpret_cast<__nv_bfloat16 *>(
                        q_row + (ea >> 6) * (kBlockM * 128) + ((((ea & 63) >> 3) ^ (row & 7)) << 4) + ((ea & 7) << 1));
                    __nv_bfloat16 *pb = reinterpret_cast<__nv_bfloat16 *>(
                        q_row + (eb >> 6) * (kBlockM * 128) + ((((eb & 63) >> 3) ^ (row & 7)) << 4) + ((eb & 7) << 1));
                    const float xa = __bfloat162float(*pa);
                    const float xb = __bfloat162float(*pb);
                    const float2 cj = __ldg(cs + j);
                    *pa = __float2bfloat16_rn(xa * cj.x - xb * cj.y);
                    *pb = __float2bfloat16_rn(xb * cj.x + xa * cj.y);
                }
                mbar_arrive(&bars->qrot[t]);
                if (!mbar_wait(&bars->qrot[t], ph, abort_flag, p.err))
                    return false;
            }
            uint4 ca[2], cb[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int ch = 2 * hf + k;
                ca[k] = *reinterpret_cast<const uint4 *>(q_row + ((ch ^ (row & 7)) << 4));
                cb[k] = *reinterpret_cast<const uint4 *>(q_row + (((ch + 4) ^ (row & 7)) << 4));
            }
            if (rot && fast_rope) {
                // this half's 16 (cos, sin) pairs from the table (the
                // producer warp read the same rows for the keys: L1 hits)
                const float4 *g = reinterpret_cast<const float4 *>(p.rope_table + (size_t)(past + i) * 32) + 8 * hf;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float4 cs[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        cs[w] = __ldg(g + 4 * k + w);  // pairs 8 (2hf + k) + 2w, + 1
                    rope_chunk_pair(ca[k], cb[k], cs);
                }
            }
            const uint32_t lo8[8] = {ca[0].x, ca[0].y, ca[0].z, ca[0].w, ca[1].x, ca[1].y, ca[1].z, ca[1].w};
            const uint32_t hi8[8] = {cb[0].x, cb[0].y, cb[0].z, cb[0].w, cb[1].x, cb[1].y, cb[1].z, cb[1].w};
            tmem_st8(q_addr + 8 * hf, lo8);       // dims 16hf .. 16hf + 15
            tmem_st8(q_addr + 16 + 8 * hf, hi8);  // dims 32 + 16hf .. 32 + 16hf + 15
            if (half > 0 && !fast_rope)
                fence_proxy_async_smem();  // the in-place rotation, before QK^T reads the buffer
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->q_ready[t]);
            return true;
        };
        bool ok = t >= n_local || load_q(t);
        for (int n = t; ok && n < n_local; n += 2) {
            const uint32_t ph = (uint32_t)(n >> 1) & 1u;
            const Tile c = tile_at(p, t_begin + n);
            const int i = c.p0 + row / p.gp;
            const int h = c.h0 + row % p.gp;
            // cached tokens before this chunk (0 for a plain prefill): query i
            // has position past + i; key rows below key_off - past precede
            // position 0 and are never visible
            const int past = p.past_lens != nullptr ? min(max(__ldg(p.past_lens + c.b), 0), p.max_past) : 0;
            const float sink = p.sinks != nullptr ? __ldg(p.sinks + h) : 0.f;  // read now, used in the epilogue

            // ---- softmax over the tile's key span, this half's 72 columns
            const int k0 = c.first_block * kKeyBlock;
            const int hi = i + p.key_off - k0;  // the row's own key column
            const int lo = max(hi - p.window + 1, max(p.key_off - past, 0) - k0);  // first visible column
            const unsigned span = (unsigned)(hi - lo);  // column c visible iff c - lo <= span
            if (!mbar_wait(&bars->s_full[t], ph, abort_flag, p.err)) {
                ok = false;
                break;
            }
            // The O staging of this worker's previous tile (its store was
            // issued a tile ago), released before this tile's epilogue reuses
            // it; half 0 arrives every tile (QK^T of this tile has read the
            // Q buffer's other blocks by now).
            release_stage(true);
            tc_fence_after();
            float x[kHalfCols];
            {
                uint32_t r[4][16], r8[8];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_ld16(s_addr + 16 * q, r[q]);
                tmem_ld8(s_addr + 64, r8);
                tmem_wait_ld_only();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    tmem_tie(r[q]);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        x[16 * q + e] = __uint_as_float(r[q][e]);
                }
                tmem_tie(r8);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    x[64 + e] = __uint_as_float(r8[e]);
            }
            // Window mask. On interior tiles every row sees columns 16 .. 127
            // (its window starts at most 16 columns in, ends at least at 127),
            // so only the 16 edge columns of each half need the test.
            const int c0 = kHalfCols * hf;  // global column of x[0]
            if (__all_sync(0xffffffffu, lo <= 16 && hi >= 127)) {
                if (hf == 0) {  // (static indices keep x in registers)
#pragma unroll
                    for (int col = 0; col < 16; ++col)
                        x[col] = ((unsigned)(col - lo) <= span) ? x[col] : -INFINITY;
                } else {
#pragma unroll
                    for (int col = kHalfCols - 16; col < kHalfCols; ++col)
                        x[col] = ((unsigned)(kHalfCols + col - lo) <= span) ? x[col] : -INFINITY;
                }
            } else {
#pragma unroll
                for (int col = 0; col < kHalfCols; ++col)
                    x[col] = ((unsigned)(c0 + col - lo) <= span) ? x[col] : -INFINITY;
            }
            float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int col = 0; col < kHalfCols; col += 8)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mxv[k] = fmax3(mxv[k], x[col + 2 * k], x[col + 2 * k + 1]);
            float mx = fmax3(mxv[0], mxv[1], fmaxf(mxv[2], mxv[3]));
            // the row's maximum over both halves
            red_max[hf * kBlockM + row] = mx;
            mbar_arrive(&bars->xchg[t]);
            if (!mbar_wait(&bars->xchg[t], ph, abort_flag, p.err)) {
                ok = false;
                break;
            }
            mx = fmaxf(mx, red_max[(hf ^ 1) * kBlockM + row]);
            const float m2 = mx * sc;   // base-2 units
            const float mu = (mx == -INFINITY) ? 0.f : m2;
            const f32x2 sc2 = {sc, sc}, nmu2 = {-mu, -mu};
            f32x2 rsv[2] = {{0.f, 0.f}, {0.f, 0.f}};
            // P over this half's columns: bf16 pairs into TMEM columns
            // [36 hf, 36 hf + 36) of S. Both halves have read their S columns
            // (the exchange above), so no write lands on unread scores.
#pragma unroll
            for (int q = 0; q < kHalfCols / 8; ++q) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const f32x2 z = fma2(f32x2{x[8 * q + 2 * e], x[8 * q + 2 * e + 1]}, sc2, nmu2);
                    const f32x2 ez = {fast_exp2(z.x), fast_exp2(z.y)};
                    rsv[e & 1] = add2(rsv[e & 1], ez);
                    pk[e] = pack_bf16x2(ez.x, ez.y);
                }
                tmem_st4(p_addr + 4 * q, pk);
            }
            const float rs_half = (rsv[0].x + rsv[0].y) + (rsv[1].x + rsv[1].y);
            {
                const uint32_t v[1] = {__float_as_uint(rs_half)};
                tmem_st1(x_addr + hf, v);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[t]);

            // ---- while PV runs: the rotary block of this worker's next Q
            // tile into TMEM (QK^T of this tile, complete at s_full, has read
            // Q_t), so that tile's QK^T can start as soon as O is read below.
            if (n + 2 < n_local && !load_q(n + 2)) {
                ok = false;
                break;
            }

            // ---- epilogue: this half's 64 output columns. The p_full wait
            // returns at once (the PV behind o_full needed it) and orders the
            // partner's row sum, read before o_free lets the next tile reuse it.
            if (!mbar_wait(&bars->o_full[t], ph, abort_flag, p.err) ||
                !mbar_wait(&bars->p_full[t], ph, abort_flag, p.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t o[2][32], rsp[1];
            tmem_ld1(x_addr + (hf ^ 1), rsp);
            tmem_ld32(o_addr, o[0]);
            tmem_ld32(o_addr + 32, o[1]);
            tmem_wait_ld_only();
            tmem_tie(rsp);
            tmem_tie(o[0]);
            tmem_tie(o[1]);
            tc_fence_before();
            mbar_arrive(&bars->o_free[t]);
            const float rs = rs_half + __uint_as_float(rsp[0]);
            // (rs >= 1: the row maximum's own term; approximate exp2 and
            // division, well inside bf16 output rounding)
            float o_scale;
            if (p.sinks != nullptr) {
                const float s2 = sink * kLog2e;
                const float mf = fmaxf(m2, s2);
                const float a = fast_exp2(m2 - mf);
                o_scale = __fdividef(a * p.v_scale, rs * a + fast_exp2(s2 - mf));
            } else {
                o_scale = __fdividef(p.v_scale, rs);
            }
            if (!p.o_tma) {
                // direct stores: this row's 64 columns as four 32-byte pieces
                if (i < p.S) {
                    uint8_t *dst =
                        reinterpret_cast<uint8_t *>(p.out + (((size_t)c.b * p.S + i) * p.Hq + h) * kDv + 64 * hf);
                    const f32x2 os2 = {o_scale, o_scale};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int col = 16 * q + 2 * e;
                            const f32x2 v = mul2(f32x2{__uint_as_float(o[col >> 5][col & 31]),
                                                       __uint_as_float(o[col >> 5][(col & 31) + 1])},
                                                 os2);
                            w[e] = pack_bf16x2(v.x, v.y);
                        }
                        st_global_32B(dst + q * 32, w, p.out_v8 != 0);
                    }
                }
                continue;
            }
            // The slot must be free: half 0's block of the Q buffer holds the
            // next tile's rotary dims until both halves have copied them
            // (q_ready); half 1's slot until the other worker's previous
            // store has read it. (The parity wait is exact: this worker
            // released its own use of two tiles ago before this point.)
            {
                const bool waited = hf == 0 ? (n + 2 >= n_local ||
                                               mbar_wait(&bars->q_ready[t], (uint32_t)((n + 2) >> 1) & 1u, abort_flag,
                                                         p.err))
                                            : mbar_wait(&bars->ost_free[wq], ((uint32_t)n & 1u) ^ 1u, abort_flag, p.err);
                if (!waited) {
                    ok = false;
                    break;
                }
            }
            // Row = lane, 128 bytes; 16-byte chunk j at j ^ (lane & 7), the
            // 128-byte swizzle of the store's tensor map.
            {
                const f32x2 os2 = {o_scale, o_scale};
                uint8_t *srow = o_stage + lane * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = 8 * j + 2 * e;
                        const f32x2 v = mul2(f32x2{__uint_as_float(o[col >> 5][col & 31]),
                                                   __uint_as_float(o[col >> 5][(col & 31) + 1])},
                                             os2);
                        w[e] = pack_bf16x2(v.x, v.y);
                    }
                    *reinterpret_cast<uint4 *>(srow + ((j ^ (lane & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            // (a warp whose rows all lie past the sequence end stores nothing;
            // a partly past box is clipped by the tensor map)
            const int w_pos = c.p0 + wq * (32 / p.gp);
            if (lane == 0) {
                o_used = true;
                if (w_pos < p.S) {
                    tma_store_4d(&p.tm_o, o_stage, 64 * hf, c.h0, w_pos, c.b);
                    bulk_commit_group();
                    o_pending = true;
                }
            }
        }
        // the last tile's staging: released for the other worker, and every
        // store complete before the CTA ends
        release_stage(false);
        if (lane == 0)
            bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma0) {
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

bool swa_rotates_keys(const LayerArgs &L)
{
    // every rotary dim in the first 64-column block, pairs in whole 16-byte chunks
    return L.rope.half > 0 && L.rope.rotary_dim <= 64 && L.rope.half % 8 == 0;
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
        !make_bf16_map_4d(&p.tm_k, a.krot, kDqk, L.Hkv, a.key_rows_valid, a.krot_rows, a.B, 64, 1, kKeyBlock) ||
        !make_bf16_map_4d(&p.tm_v, a.v, kDv, L.Hkv, a.key_rows_valid, a.v_rows, a.B, 64, 1, kKeyBlock) ||
        !make_bf16_map_4d(&p.tm_o, a.out, kDv, L.Hq, a.S, a.S, a.B, 64, gp, 32 / gp))
        return cudaErrorInvalidValue;
    p.out = reinterpret_cast<__nv_bfloat16 *>(a.out);
    p.out_v8 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
    p.rope_table = rope_table;
    p.sinks = L.sinks;
    p.past_lens = a.past_lens;
    p.err = a.err;
    p.S = a.S;
    p.key_off = a.past_lens != nullptr ? a.swa_key_off : 0;
    p.max_past = a.max_past;
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
    // The staged TMA-store epilogue pays off once a CTA runs many tiles
    // (B4 S32768: ~440 per CTA, 1.85 -> 1.74 ms per layer); for short runs
    // (B1 S4096: 14 per CTA) direct stores measured faster (0.087 against
    // 0.089 ms).
    p.o_tma = p.tiles_per_cta >= 16 ? 1 : 0;
    p.rope_half = L.rope.half;
    p.rotate_k = a.k_unrotated ? 1 : 0;
    p.scale_log2 = L.scale_log2;
    p.v_scale = L.v_scale;

    // The setmaxnreg split assumes the block launches with exactly
    // kLaunchRegs registers per thread; refuse to launch otherwise (a smaller
    // pool would leave setmaxnreg.inc waiting forever).
    static std::atomic<unsigned long long> prepared{0};
    cudaError_t e = prepare_kernel_once(prefill_swa_kernel, kSmemBytes, prepared, kLaunchRegs);
    if (e != cudaSuccess)
        return e;
    const int grid = (p.num_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta;
    prefill_swa_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

} // namespace mimo
