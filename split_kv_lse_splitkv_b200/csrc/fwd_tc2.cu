// Chunk-partial forward on pairs of SMs (sm_100a): TMA -> tcgen05.mma.cta_group::2 -> TMEM.
//
// Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, Abstract: exact
// attention over context chunks, each producing a query-sized partial output and a per-row
// log-sum-exp; the chunks are placed by the cost-aware LPT plan. Here each LPT worker is a pair of
// SMs: a two-CTA cluster that walks one queue. A work item (s, c, g, t) is a 256-row query tile (the
// P consecutive blocks of tile t at kv head g, block * G rows each) against the key tiles of chunk c
// that its rows see; CTA r of the pair owns tile rows 128 r .. 128 r + 127 (its P / 2 blocks). One
// thread of the leader CTA (rank 0) issues every MMA for both SMs as M = 256 instructions:
//   S = Q K^T:  A = each CTA's 128 Q rows, B = the key tile, 64 keys held by each CTA;
//   O += P V:   A = each CTA's P in its own TMEM, B = the key tile's V, 64 head-dim columns per CTA;
// and each SM's TMEM receives its own 128 rows of S and O. One M = 256 instruction does the work of
// two M = 128 instructions, and a single issuing thread is limited by instruction count (one
// 128x128x16 MMA per ~120 cycles on one SM, one 256x128x16 pair MMA per ~98 cycles), so the pair
// halves the issue time per FLOP; each SM also loads and reads only half of every K/V tile.
// Self items (tile t, kv head g) take the tile's rows against the tile's own keys: one key tile of
// Kb/Vb from row block * (first block), where the rows of block x see columns block*x .. +block-1.
//
// Roles in each CTA (512 threads, four warpgroups; registers moved with setmaxnreg):
//   warps 0-7   softmax of this CTA's 128 rows (two warps per TMEM lane quadrant, key columns
//               0-63 / 64-127, agreeing on the row maximum through shared memory)
//   warps 8-11  epilogue: normalises O of a finished item and stores O_c (bf16), LSE_c
//   warp 12     lane 0: TMA producer of this CTA's halves (Q rows, K keys, V columns);
//               lane 1 (leader only): the claimer, which writes the pair's item sequence into the
//               item rings of both CTAs
//   warp 13     TMEM owner of this CTA (pair-wide allocation); in the leader: the QK issuer
//   warp 14     in the leader: the PV issuer
//
// Synchronisation across the pair: the producers' copies complete on the leader's full barriers
// (cta_group::2 copies, no multicast); MMA completions are committed to the barrier at the same offset
// in both CTAs (commit multicast); both CTAs' softmax warps arrive on the leader's P barrier and both
// epilogues on the leader's O-free barrier through cluster addresses. TMEM per SM (512 columns):
// S[2] = Q K^T of tiles n % 2 (P written over its first 64 columns as bf16 pairs), O[2] for items
// k % 2. The pipeline is that of the one-SM kernel: QK(n) needs K(n) and PV(n-2) complete, PV(n)
// needs P(n) of both CTAs, V(n) and, on an item's first tile, both epilogues done with O[k % 2].
//
// Every wait is bounded (2 s); on expiry the CTA raises SPLITKV_DEV_TIMEOUT, tells its peer, gives its
// own copies in flight time to land, and the pair meets at a cluster barrier (after the leader's MMAs
// are drained) before TMEM is freed.
#include <climits>
#include <cstdio>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_map.cuh"

namespace splitkv {

namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int kEpiWarp0 = 8;
constexpr int kLoadWarp = 12;  // lane 0: TMA producer; lane 1: claimer (leader)
constexpr int kMmaWarp = 13;   // TMEM owner; QK issuer (leader)
constexpr int kPvWarp = 14;    // PV issuer (leader)
constexpr int kSoftmaxRegs = 160;  // per SM sub-partition: 160 + 160 + 88 + 104 = 512 = 4 x 128 launched
constexpr int kEpilogueRegs = 88;
constexpr int kControlRegs = 104;
constexpr int kQBytes = 32768;  // 128 query rows x 128 d, as two 128-byte-wide halves
constexpr int kQHalf = 16384;
constexpr int kKBytes = 16384;  // this CTA's 64 keys of a key tile x 128 d, two halves
constexpr int kKHalf = 8192;
constexpr int kVBytes = 16384;  // the key tile's 128 keys x this CTA's 64 head-dim columns
constexpr int kKeysPerTile = 128;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint64_t kTestLimitNs = 20000ull;  // the starved pair's limit in test mode (20 us)
constexpr uint64_t kDrainNs = 50000ull;      // after an abort: time given to this CTA's copies in flight
constexpr float kRescaleLog2 = 8.0f;

constexpr uint32_t kColS = 0, kColO = 256;  // S[b] at 128 b, O[b] at 256 + 128 b

constexpr int kRing = 128;     // entries of the item ring
constexpr int kReaders = 15;   // producer, QK and PV issuers, softmax warps 8, epilogue warps 4
constexpr int32_t kRingEnd = -1;

constexpr int kOffQ = 0;                          // Q[item parity]
constexpr int kOffK = 2 * kQBytes;                // K[tile parity]
constexpr int kOffV = kOffK + 2 * kKBytes;        // V[tile parity]
constexpr int kOffStat = kOffV + 2 * kVBytes;     // float [item parity][m, l0, l1][128]
constexpr int kOffXchg = kOffStat + 2 * 3 * 128 * 4;  // float [tile parity][quad][half][32]
constexpr int kOffBar = kOffXchg + 2 * 4 * 2 * 32 * 4;

struct Bars {
    // Leader's barriers that both CTAs' copies complete on (the leader arms them with both halves' bytes).
    uint64_t q_full[2], k_full[2], v_full[2];
    // Completions of the leader's MMAs, committed to both CTAs.
    uint64_t q_empty[2];   // every QK^T of item k complete: Q slot k % 2 free
    uint64_t s_full[2];    // QK^T(n) complete: S(n) ready, K slot n % 2 free
    uint64_t pv_done[2];   // PV(n) complete: V slot n % 2 free, S(n) free
    uint64_t o_ready[2];   // last PV of item k complete: O[k % 2] final
    // Leader's barriers that both CTAs arrive on.
    uint64_t p_full[2];    // P(n) written: 8 softmax warps per CTA
    uint64_t o_free[2];    // O[k % 2] of item k read: 4 epilogue warps per CTA
    // This CTA's own.
    uint64_t epi_done[2];  // its epilogue has read (m, l) and O of item k (4 warps)
    uint64_t stat_full[2]; // its softmax wrote (m, l) of item k (8 warps)
    uint64_t drain[2];     // leader: every MMA of the QK / PV issuer complete
    // The pair's item sequence, written into both CTAs by the leader's claimer.
    int32_t ring_id[kRing];   // item id (n_items + p: self tile p / Hkv at kv head p % Hkv; kRingEnd: no more)
    int32_t ring_nvis[kRing]; // keys of the chunk its last block sees (self: the tile's own keys)
    int32_t ring_j[kRing];    // first block of its query tile
    int32_t ring_c[kRing];    // chunk
    int32_t ring_sgn[kRing];  // sample | blocks in the tile << 8 | kv head << 16
    int32_t ring_w;           // entries written
    int32_t ring_r[kReaders];       // entries read, per reader of this CTA
    int32_t ring_r_peer[kReaders];  // leader: entries read by the peer's readers
    int32_t xflag[4][2];            // [quad][half]: tiles whose half row max is in xchg
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

constexpr int kSmemBytes = kOffBar + (int)sizeof(Bars) + 1024;  // + alignment slack

struct TileRef {
    int64_t id;                // item id, or n_items + p for a self tile
    int32_t s, c, g, j;
    int32_t nvis, ntiles;      // keys its last block sees (self: block * blocks), key tiles
    int32_t nbt;               // blocks in the query tile
    int32_t self_item;
};

// S columns 64h .. 64h+63 of this thread's row; keys outside [lo, hi) (tile-local) read as -inf.
__device__ __forceinline__ void load_half(uint32_t ts, int h, int lo, int hi, uint32_t (&ra)[32],
                                          uint32_t (&rb)[32]) {
    tmem_ld32(ts + h * 64, ra);
    tmem_ld32(ts + h * 64 + 32, rb);
    tmem_wait_ld();
    if (lo > h * 64 || hi < h * 64 + 64) {
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int c0 = h * 64 + u, c1 = h * 64 + 32 + u;
            if (c0 < lo || c0 >= hi) ra[u] = __float_as_uint(-INFINITY);
            if (c1 < lo || c1 >= hi) rb[u] = __float_as_uint(-INFINITY);
        }
    }
}

__device__ __forceinline__ float max_half(const uint32_t (&ra)[32], const uint32_t (&rb)[32]) {
    float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
    for (int u = 0; u < 32; u += 4) {
        m0 = max3f(m0, __uint_as_float(ra[u]), __uint_as_float(ra[u + 1]));
        m1 = max3f(m1, __uint_as_float(ra[u + 2]), __uint_as_float(ra[u + 3]));
        m2 = max3f(m2, __uint_as_float(rb[u]), __uint_as_float(rb[u + 1]));
        m3 = max3f(m3, __uint_as_float(rb[u + 2]), __uint_as_float(rb[u + 3]));
    }
    return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// P = 2^(s*c - m) for 64 keys as 32 bf16 pairs (low half = even key), summed into acc.
__device__ __forceinline__ void exp_half(const uint32_t (&ra)[32], const uint32_t (&rb)[32], uint64_t c2,
                                         uint64_t negm2, uint64_t (&acc)[4], uint32_t (&pk)[32]) {
#pragma unroll
    for (int u = 0; u < 32; ++u) {
        const uint32_t* src = u < 16 ? ra : rb;
        const int v = (u & 15) * 2;
        float t0, t1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(src[v]), __uint_as_float(src[v + 1])), c2, negm2), t0, t1);
        const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
        acc[u & 3] = f2_add(acc[u & 3], f2_pack(p0, p1));
        __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
        pk[u] = *reinterpret_cast<uint32_t*>(&hp);
    }
}

// ---------------------------------------------------------------- item ring
// The pair's work is its LPT queue, in queue order, then self tiles (one key tile each, outside the
// plan) claimed one at a time through a global counter once its own work runs low. The leader's
// claimer writes each decoded item into the rings of both CTAs; every role of both CTAs reads its
// ring in order and publishes its progress to the leader (the claimer reuses a slot once every
// reader of both CTAs has passed it).

// Next ring entry (blocking). Returns 1 (entry in t), or -1 at the end of the sequence or on
// abort/timeout. `prog` is this reader's progress word in the leader (cluster address); a warp-wide
// reader (all 32 lanes in step) publishes after __syncwarp.
__device__ __forceinline__ int ring_next(const Meta& m, Bars* bars, int32_t& idx, uint32_t prog, bool warp_wide,
                                         TileRef& t, volatile int* abort_flag, uint64_t lim) {
    uint64_t t0 = 0;
    for (uint32_t spin = 0;; ++spin) {
        if (idx < ld_acquire_cluster_s32(&bars->ring_w)) {
            const int e = idx % kRing;
            const int32_t id = ((volatile int32_t*)bars->ring_id)[e];
            const int32_t nvis = ((volatile int32_t*)bars->ring_nvis)[e];
            const int32_t jj = ((volatile int32_t*)bars->ring_j)[e];
            const int32_t cc = ((volatile int32_t*)bars->ring_c)[e];
            const int32_t sgn = ((volatile int32_t*)bars->ring_sgn)[e];
            if (id == kRingEnd) return -1;  // the end entry stays: every later call sees it again
            ++idx;
            if (warp_wide) __syncwarp();
            if (!warp_wide || (threadIdx.x & 31) == 0) st_release_cluster_u32(prog, (uint32_t)idx);
            t.id = id;
            t.self_item = id >= m.n_items ? 1 : 0;
            t.nvis = nvis;
            t.ntiles = (nvis + kKeysPerTile - 1) / kKeysPerTile;
            t.j = jj;
            t.c = cc;
            t.s = sgn & 0xff;
            t.nbt = (sgn >> 8) & 0xff;
            t.g = sgn >> 16;
            return 1;
        }
        if ((spin & 63u) == 63u) {
            if (*abort_flag) return -1;
            if (t0 == 0) t0 = globaltimer();
            else if (globaltimer() - t0 > lim) {
                *abort_flag = 1;
                return -1;
            }
        }
        __nanosleep(32);
    }
}

// Number of query tiles (P blocks each) of all samples before sample s, and the sample of tile T.
__device__ __forceinline__ void self_tile(const Meta& m, int64_t T, int32_t& s, int32_t& j0, int32_t& nbt) {
    int64_t base = 0;
    for (s = 0; s < m.batch; ++s) {
        const int32_t nb = m.anchor_off[s + 1] - m.anchor_off[s];
        const int64_t nt = (nb + m.pack - 1) / m.pack;
        if (T < base + nt) break;
        base += nt;
    }
    const int32_t nb = m.anchor_off[s + 1] - m.anchor_off[s];
    const int32_t b = (int32_t)(T - base) * m.pack;
    j0 = m.anchor_off[s] + b;
    nbt = nb - b < m.pack ? nb - b : m.pack;
}

// The leader's claimer: the pair's queue, then self tiles while the producer runs low, then the end
// entry. One thread.
__device__ void claim_items(const Meta& m, Bars* bars, const int32_t* __restrict__ anchors,
                            const int32_t* __restrict__ item_id, const int32_t* __restrict__ queue_off,
                            const int32_t* __restrict__ queue_items, int32_t* pool, int64_t n_self,
                            int32_t* status, volatile int* abort_flag, uint64_t lim) {
    const int32_t wq = (int32_t)(blockIdx.x >> 1);
    const int32_t q0 = queue_off[wq], q1 = queue_off[wq + 1];
    const int32_t* rr = bars->ring_r;
    const int32_t* rp = bars->ring_r_peer;
    int32_t w = 0;
    bool ok = true;
    // Wait until slot w is free (every reader of both CTAs is past entry w - kRing) and, if ahead > 0,
    // until the leader's producer (reader 0) has fewer than `ahead` entries left to read.
    auto wait_room = [&](int ahead) -> bool {
        const uint64_t t0 = globaltimer();
        for (uint32_t spin = 0;; ++spin) {
            // Acquire: a reader's loads of an entry happen before its progress store that frees it.
            const int32_t r0 = ld_acquire_cluster_s32(rr);
            int32_t lo = r0;
            for (int x = 1; x < kReaders; ++x) lo = min(lo, ld_acquire_cluster_s32(rr + x));
            for (int x = 0; x < kReaders; ++x) lo = min(lo, ld_acquire_cluster_s32(rp + x));
            if (lo > w - kRing && (ahead <= 0 || r0 > w - ahead)) return true;
            if ((spin & 63u) == 63u && (*abort_flag || globaltimer() - t0 > lim)) {
                *abort_flag = 1;
                return false;
            }
            __nanosleep(64);
        }
    };
    auto put = [&](int32_t id, int32_t nvis, int32_t j, int32_t c, int32_t sgn) {
        const int e = w % kRing;
        for (uint32_t r = 0; r < 2; ++r) {
            st_cluster_u32(mapa_rank(&bars->ring_id[e], r), (uint32_t)id);
            st_cluster_u32(mapa_rank(&bars->ring_nvis[e], r), (uint32_t)nvis);
            st_cluster_u32(mapa_rank(&bars->ring_j[e], r), (uint32_t)j);
            st_cluster_u32(mapa_rank(&bars->ring_c[e], r), (uint32_t)c);
            st_cluster_u32(mapa_rank(&bars->ring_sgn[e], r), (uint32_t)sgn);
        }
        ++w;
        for (uint32_t r = 0; r < 2; ++r) st_release_cluster_u32(mapa_rank(&bars->ring_w, r), (uint32_t)w);
    };
    for (int32_t pos = q0; ok && pos < q1; ++pos) {
        const int32_t id = __ldg(item_id + __ldg(queue_items + pos));
        if (id < 0 || id >= m.n_items) {
            raise_status(status, SPLITKV_DEV_BAD_PLAN);
            continue;
        }
        const Item it = decode_item(m, id);
        const int32_t nvis = visible_in_chunk(m, it.s, it.c, __ldg(anchors + it.j + it.nbt - 1));
        if (nvis <= 0) continue;
        ok = wait_room(0);
        if (ok) put(id, nvis, it.j, it.c, it.s | (it.nbt << 8) | (it.g << 16));
    }
    while (ok) {
        // Claim when the producer has fewer than 2 entries left to read.
        if (!wait_room(2)) {
            ok = false;
            break;
        }
        const int64_t p = atomicAdd(pool, 1);
        if (p >= n_self) break;
        int32_t s, j0, nbt;
        self_tile(m, p / m.hkv, s, j0, nbt);
        put((int32_t)(m.n_items + p), m.block * nbt, j0, 0, s | (nbt << 8) | ((int32_t)(p % m.hkv) << 16));
    }
    if (ok && wait_room(0)) put(kRingEnd, 0, 0, 0, 0);
}

// Keys [lo, hi) of the item (chunk-local; self: tile-local) that tile row tr sees; a row of no block
// of the tile sees none.
__device__ __forceinline__ void row_window(const Meta& m, const int32_t* __restrict__ anchors, const TileRef& t,
                                           int tr, int& lo, int& hi) {
    const int32_t x = tr / m.rows;
    lo = 0;
    hi = 0;
    if (x >= t.nbt) return;
    if (t.self_item) {
        lo = m.block * x;
        hi = lo + m.block;
    } else {
        hi = visible_in_chunk(m, t.s, t.c, __ldg(anchors + t.j + x));
    }
}

// O *= alpha over this warp's 64 columns of its rows.
__device__ __forceinline__ void rescale_o64(uint32_t to, float alpha) {
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
        uint32_t ov[16];
        tmem_ld16(to + cc * 16, ov);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * alpha);
        tmem_st16(to + cc * 16, ov);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc2_kernel(const __grid_constant__ Meta m, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
                   const int32_t* __restrict__ anchors, const int32_t* __restrict__ item_id,
                   const int32_t* __restrict__ queue_off, const int32_t* __restrict__ queue_items,
                   __nv_bfloat16* __restrict__ o_part, float* __restrict__ lse_part, int32_t* __restrict__ pool,
                   int64_t n_self, int32_t* __restrict__ status, int32_t test_starve) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* stat = reinterpret_cast<float*>(smem + kOffStat);
    float* xchg = reinterpret_cast<float*>(smem + kOffXchg);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    // Limit of every wait that can run out while work is expected (drains keep the full limit).
    const uint64_t lim = (test_starve && (blockIdx.x >> 1) == 0) ? kTestLimitNs : kTimeoutNs;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->k_full[b], 1);
            mbar_init(&bars->v_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->pv_done[b], 1);
            mbar_init(&bars->o_ready[b], 1);
            mbar_init(&bars->p_full[b], 16);
            mbar_init(&bars->o_free[b], 8);
            mbar_init(&bars->epi_done[b], 4);
            mbar_init(&bars->stat_full[b], 8);
            mbar_init(&bars->drain[b], 1);
        }
        bars->ring_w = 0;
        for (int x = 0; x < kReaders; ++x) {
            bars->ring_r[x] = 0;
            // The peer has no QK / PV issuer: its slots never hold the claimer back.
            bars->ring_r_peer[x] = (x == 1 || x == 2) ? INT_MAX / 2 : 0;
        }
        for (int x = 0; x < 8; ++x) (&bars->xflag[0][0])[x] = 0;
        bars->abort_flag = 0;
        bars->status0 = leader && status_bad(status) ? 1 : 0;
        fence_barrier_init();
    }
    __syncthreads();
    cluster_sync_all();  // both CTAs running, their barriers and rings initialised, before any remote access
    // One decision for the pair: the peer takes the leader's reading of the status word.
    if (!leader && threadIdx.x == 0) bars->status0 = ld_cluster_s32(mapa_rank(&bars->status0, 0));
    if (warp == kMmaWarp) {  // the same warp in both CTAs: one pair-wide allocation
        tmem_alloc_pair(&bars->tmem_base, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const bool skip = bars->status0 != 0;
    const int G = m.group;
    const int qrows = m.block * (m.pack / 2);  // query rows (of G heads each) per CTA
    // Where this CTA's readers publish their progress (leader: own words; peer: the leader's copy).
    auto prog_addr = [&](int slot) -> uint32_t {
        return mapa_rank(leader ? &bars->ring_r[slot] : &bars->ring_r_peer[slot], 0);
    };

    if (warp >= kLoadWarp) {
        // ------------------------------------------------------------ control warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kControlRegs));
        if (!skip && warp == kLoadWarp && lane == 0) {
            // TMA producer of this CTA's halves: Q rows of its blocks (slot k % 2), then per key tile
            // its 64 keys of K(n) and its 64 head-dim columns of V(n) (slot n % 2); all complete on the
            // leader's barriers, which the leader arms with both CTAs' bytes.
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            const uint32_t q_bytes = 2u * 64u * (uint32_t)G * (uint32_t)qrows * 2u;
            // The leader's barriers (cluster addresses; [1] is 8 bytes after [0]).
            const uint32_t qf = mapa_rank(&bars->q_full[0], 0), kf = mapa_rank(&bars->k_full[0], 0),
                           vf = mapa_rank(&bars->v_full[0], 0);
            int32_t ridx = 0;
            TileRef t;
            uint32_t k = 0, nk = 0;
            bool ok = true, issued = false;
            const uint32_t prog = prog_addr(0);
            while (ok && ring_next(m, bars, ridx, prog, false, t, abort_flag, lim) == 1) {
                const int qb = k & 1;
                if (k >= 2 && !mbar_wait(&bars->q_empty[qb], ((k >> 1) - 1) & 1u, abort_flag, lim)) {
                    ok = false;
                    break;
                }
                if (leader) mbar_arrive_expect_tx(&bars->q_full[qb], 2u * q_bytes);
                uint8_t* qdst = smem + kOffQ + qb * kQBytes;
                const int32_t qrow = m.block * (t.j + (int32_t)rank * (m.pack / 2));
                tma_load_3d_pair(qdst, &tmQ, qf + 8u * qb, 0, t.g * G, qrow);
                tma_load_3d_pair(qdst + kQHalf, &tmQ, qf + 8u * qb, 64, t.g * G, qrow);
                issued = true;
                ++k;
                const CUtensorMap* mk = t.self_item ? &tmKb : &tmK;
                const CUtensorMap* mv = t.self_item ? &tmVb : &tmV;
                for (int32_t tt = 0; tt < t.ntiles; ++tt) {
                    const uint32_t n = nk;
                    const int b = n & 1;
                    const uint32_t ph = ((n >> 1) & 1u) ^ 1u;
                    const int32_t row = t.self_item ? m.block * t.j
                                                    : (int32_t)(m.key_off[t.s] + (int64_t)t.c * m.chunk +
                                                                (int64_t)tt * kKeysPerTile);
                    if (!mbar_wait(&bars->s_full[b], ph, abort_flag, lim)) {  // QK(n-2) done: K slot free
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(&bars->k_full[b], 2u * kKBytes);
                    uint8_t* kdst = smem + kOffK + b * kKBytes;
                    tma_load_3d_pair(kdst, mk, kf + 8u * b, 0, t.g, row + 64 * (int32_t)rank);
                    tma_load_3d_pair(kdst + kKHalf, mk, kf + 8u * b, 64, t.g, row + 64 * (int32_t)rank);
                    ++nk;
                    if (!mbar_wait(&bars->pv_done[b], ph, abort_flag, lim)) {  // PV(n-2) done: V slot free
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(&bars->v_full[b], 2u * kVBytes);
                    tma_load_3d_pair(smem + kOffV + b * kVBytes, mv, vf + 8u * b, 64 * (int32_t)rank, t.g, row);
                }
            }
            if (!ok) *abort_flag = 1;
            if (*abort_flag && issued) {
                // Copies of this CTA may still be in flight with nothing left to consume them (their
                // completions go to the leader's barriers): give them time to land before the exit.
                const uint64_t t0 = globaltimer();
                while (globaltimer() - t0 < kDrainNs) __nanosleep(1000);
            }
        } else if (!skip && leader && warp == kLoadWarp && lane == 1) {
            // Test mode (SPLITKV_FWD_TEST_STARVE): the first pair's claimer publishes nothing, so every
            // role of both CTAs waits for its first item with no copy or MMA issued, and gives up.
            if (!(test_starve && blockIdx.x == 0))
                claim_items(m, bars, anchors, item_id, queue_off, queue_items, pool, n_self, status, abort_flag,
                            lim);
        } else if (!skip && leader && (warp == kMmaWarp || warp == kPvWarp) && lane == 0) {
            // Two issuers of pair MMAs. QK issuer: S[n % 2] = Q K(n)^T once K(n) has landed (both halves)
            // and PV(n-2) has read P(n-2) out of S[n % 2]. PV issuer: O[k % 2] += P(n) V(n) once P(n) is
            // written in both CTAs; the first PV of item k also waits until both epilogues have read
            // O[k % 2] of item k-2.
            const bool is_qk = warp == kMmaWarp;
            constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(256, 128, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(256, 128, false, true);
            uint64_t dq[2], dk[2], dv[2];
            for (int b = 0; b < 2; ++b) {
                dq[b] = umma_desc_sw128(smem_u32(smem + kOffQ + b * kQBytes), 16, 1024);
                dk[b] = umma_desc_sw128(smem_u32(smem + kOffK + b * kKBytes), 16, 1024);
                dv[b] = umma_desc_sw128(smem_u32(smem + kOffV + b * kVBytes), kVBytes, 1024);
            }
            int32_t ridx = 0;
            TileRef t;
            uint32_t k = 0, n = 0;
            bool ok = true;
            const uint32_t prog = prog_addr(is_qk ? 1 : 2);
            while (ok && ring_next(m, bars, ridx, prog, false, t, abort_flag, lim) == 1) {
                const int ib = k & 1;
                if (is_qk) {
                    if (!mbar_wait(&bars->q_full[ib], (k >> 1) & 1u, abort_flag, lim)) {
                        ok = false;
                        break;
                    }
                    for (int32_t tt = 0; tt < t.ntiles; ++tt, ++n) {
                        const int b = n & 1;
                        if (!mbar_wait(&bars->k_full[b], (n >> 1) & 1u, abort_flag, lim) ||
                            !mbar_wait(&bars->pv_done[b], ((n >> 1) & 1u) ^ 1u, abort_flag, lim)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t ts = tmem + kColS + 128u * b;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t offa = (uint64_t)(((kk >> 2) * kQHalf + (kk & 3) * 32) / 16);
                            const uint64_t offb = (uint64_t)(((kk >> 2) * kKHalf + (kk & 3) * 32) / 16);
                            mma_ss_pair(ts, dq[ib] + offa, dk[b] + offb, idesc_qk, kk > 0 ? 1u : 0u);
                        }
                        mma_commit_pair_mc(&bars->s_full[b], 3);
                        if (tt == t.ntiles - 1) mma_commit_pair_mc(&bars->q_empty[ib], 3);
                    }
                } else {
                    const uint32_t tO = tmem + kColO + 128u * ib;
                    for (int32_t tt = 0; tt < t.ntiles; ++tt, ++n) {
                        const int b = n & 1;
                        if (!mbar_wait(&bars->p_full[b], (n >> 1) & 1u, abort_flag, lim) ||
                            (tt == 0 && k >= 2 &&
                             !mbar_wait(&bars->o_free[ib], ((k >> 1) & 1u) ^ 1u, abort_flag, lim)) ||
                            !mbar_wait(&bars->v_full[b], (n >> 1) & 1u, abort_flag, lim)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t tp = tmem + kColS + 128u * b;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ts_pair(tO, tp + (uint32_t)(kk * 8), dv[b] + (uint64_t)(kk * 2048 / 16), idesc_pv,
                                        (tt > 0 || kk > 0) ? 1u : 0u);
                        mma_commit_pair_mc(&bars->pv_done[b], 3);
                        if (tt == t.ntiles - 1) mma_commit_pair_mc(&bars->o_ready[ib], 3);
                    }
                }
                ++k;
            }
            if (!ok) *abort_flag = 1;
            // Drain: all MMAs issued by this thread complete before the pair meets for the exit.
            uint64_t* dr = &bars->drain[is_qk ? 0 : 1];
            mma_commit_pair_mc(dr, 1);
            volatile int never = 0;
            mbar_wait(dr, 0, &never, kTimeoutNs);
        }
        __syncwarp();
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------------ epilogue warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kEpilogueRegs));
        if (!skip) {
            const int quad = warp & 3;
            const int lr = quad * 32 + lane;                    // this CTA's row
            const int tr = (int)rank * 128 + lr;                // the item tile's row
            const int RT = m.rows_item;                         // rows of a partial slot (256)
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            int32_t ridx = 0;
            TileRef t;
            uint32_t k = 0;
            bool ok = true;
            const uint32_t prog = prog_addr(11 + quad);
            const uint32_t of = mapa_rank(&bars->o_free[0], 0);  // the leader's; [1] is 8 bytes after
            while (ok && ring_next(m, bars, ridx, prog, true, t, abort_flag, lim) == 1) {
                const int ob = k & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&bars->stat_full[ob], (k >> 1) & 1u, abort_flag, lim) &&
                                                 mbar_wait(&bars->o_ready[ob], (k >> 1) & 1u, abort_flag, lim));
                if (!ok) break;
                tc_fence_after();
                const float* sp = stat + ob * 384;
                const float m_l = sp[lr], l = sp[128 + lr] + sp[256 + lr];  // the two column halves' sums
                const uint32_t to = tmem + kColO + 128u * ob + lane_off;
                const float inv = l > 0.f ? 1.f / l : 0.f;  // a row that sees no key: O = 0, LSE = -inf
                // Slot and row of this tile row's partial: the item's own slot, or for a self tile the
                // self slot of the row's block (rows 0 .. block*G - 1).
                const int32_t x = tr / m.rows;
                const bool write = x < t.nbt;
                int64_t slot = t.id;
                int row = tr;
                if (t.self_item) {
                    slot = m.n_items + (int64_t)(t.j + x) * m.hkv + t.g;
                    row = tr - x * m.rows;
                }
                __nv_bfloat16* op = o_part + slot * (int64_t)RT * 128;  // [d/8][RT][8] bf16
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    uint32_t ov[16];
                    tmem_ld16(to + cc * 16, ov);
                    tmem_wait_ld();
                    if (cc == 7) {  // O[k % 2] fully read: the PV issuer may start item k+2 in it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive_cluster(of + 8u * ob);
                            mbar_arrive(&bars->epi_done[ob]);
                        }
                    }
                    if (write) {  // 16 columns: two groups of 8 bf16, 16 bytes each
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(ov[8 * u + 2 * e]) * inv,
                                                                         __uint_as_float(ov[8 * u + 2 * e + 1]) * inv);
                                pk[e] = *reinterpret_cast<uint32_t*>(&h);
                            }
                            *reinterpret_cast<uint4*>(op + ((int64_t)(cc * 2 + u) * RT + row) * 8) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
                if (write)
                    lse_part[slot * RT + row] = l > 0.f ? (m_l + lg2_approx(l)) * 0.6931471805599453f : -INFINITY;
                ++k;
            }
            if (!ok) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
        if (!skip) {
            const int quad = warp & 3;              // TMEM lane quadrant: rows 32 quad .. +31
            const int half = warp >> 2;             // key columns 64 half .. +63 of each tile
            const int lr = quad * 32 + lane;        // this CTA's row
            const int tr = (int)rank * 128 + lr;    // the item tile's row
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const uint32_t to0 = tmem + kColO + lane_off + 64u * half;  // this warp's 64 columns of O[0]
            const float c = m.scale * 1.4426950408889634f;  // log2(e)
            const uint64_t c2 = f2_pack(c, c);
            volatile int32_t* my_flag = &bars->xflag[quad][half];
            volatile int32_t* other_flag = &bars->xflag[quad][half ^ 1];
            uint32_t k = 0, n = 0;
            bool ok = true;
            int32_t ridx = 0;
            TileRef t;
            const uint32_t prog = prog_addr(3 + warp);
            while (ok && ring_next(m, bars, ridx, prog, true, t, abort_flag, lim) == 1) {
                int row_lo, row_hi;
                row_window(m, anchors, t, tr, row_lo, row_hi);
                float m_l = -INFINITY, l = 0.f;  // reference max and this half's row sum (relative to m_l)
                for (int32_t tt = 0; tt < t.ntiles; ++tt, ++n) {
                    // The whole warp leaves together on a timeout: the TMEM accesses below are collective.
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[n & 1], (n >> 1) & 1u, abort_flag, lim))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ts = tmem + kColS + 128u * (n & 1) + lane_off;  // S(n), this row
                    uint32_t ra[32], rb[32];
                    load_half(ts, half, row_lo - tt * kKeysPerTile, row_hi - tt * kKeysPerTile, ra, rb);
                    const float hmax = max_half(ra, rb) * c;
                    // Row max over both halves: publish mine, wait for my partner's (bounded).
                    float* slot = xchg + (n & 1) * 256;
                    slot[(quad * 2 + half) * 32 + lane] = hmax;
                    tc_fence_before();  // my S loads are ordered before the flag (my partner writes P next)
                    __threadfence_block();
                    __syncwarp();
                    if (lane == 0) *my_flag = (int32_t)(n + 1);
                    bool got = true;
                    {
                        const uint64_t t0 = globaltimer();
                        for (uint32_t spin = 0; *other_flag < (int32_t)(n + 1); ++spin) {
                            if ((spin & 63u) == 63u && (*abort_flag || globaltimer() - t0 > lim)) {
                                got = false;
                                break;
                            }
                        }
                    }
                    if (!__all_sync(0xffffffffu, got)) {
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float mx = fmaxf(hmax, ((volatile float*)slot)[(quad * 2 + (half ^ 1)) * 32 + lane]);
                    if (tt == 0) {
                        m_l = mx;
                    } else {
                        const bool move = mx > m_l + kRescaleLog2;  // the same decision in both halves
                        if (__any_sync(0xffffffffu, move)) {
                            // The max moved: rescale my columns of O once PV(n-1) is complete, and my sum.
                            if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1u,
                                                                   abort_flag, lim))) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const float alpha = move ? ex2_approx(m_l - mx) : 1.f;
                            rescale_o64(to0 + 128u * (k & 1u), alpha);
                            l *= alpha;
                            if (move) m_l = mx;
                        }
                    }
                    // P = 2^(s*c - m) as bf16 pairs (keys 2u, 2u+1 -> column u) into columns 32 half.. of
                    // S(n): my partner has read its S columns (it published its max after the reads).
                    const float m_use = m_l == -INFINITY ? 0.f : m_l;  // fully masked row: P = 2^-inf = 0
                    const uint64_t negm2 = f2_pack(-m_use, -m_use);
                    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
                    uint32_t pk[32];
                    exp_half(ra, rb, c2, negm2, acc, pk);
                    tmem_st32(ts + 32 * half, pk);
                    {
                        float a0, a1, b0, b1, c0, c1, d0, d1;
                        f2_unpack(acc[0], a0, a1);
                        f2_unpack(acc[1], b0, b1);
                        f2_unpack(acc[2], c0, c1);
                        f2_unpack(acc[3], d0, d1);
                        l += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)  // the leader's P barrier: its PV issuer waits for 16 warps
                        mbar_arrive_cluster(mapa_rank(&bars->p_full[n & 1], 0));
                }
                if (!ok) break;
                // Hand (m, l) of item k to the epilogue; stat[k % 2] was last read for item k-2.
                const int ob = k & 1;
                if (k >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->epi_done[ob], ((k >> 1) - 1) & 1u,
                                                                 abort_flag, lim))) {
                    ok = false;
                    break;
                }
                float* sp = stat + ob * 384;
                if (half == 0) sp[lr] = m_l;
                sp[128 + 128 * half + lr] = l;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->stat_full[ob]);
                ++k;
            }
            if (!ok) *abort_flag = 1;
        }
    }

    // A CTA that gave up tells its peer, whose waits then end too.
    if (*abort_flag) st_cluster_u32(mapa_rank(&bars->abort_flag, cluster_ctarank() ^ 1u), 1u);
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the leader's MMAs are drained and no CTA accesses the other's memory after this
    tc_fence_after();
    if (threadIdx.x == 0 && bars->abort_flag) raise_status(status, SPLITKV_DEV_TIMEOUT);
    if (warp == kMmaWarp) tmem_dealloc_pair(tmem, 512);
}

}  // namespace

bool fwd_tc2_supported(const Meta& m) {
    // 256-row items whose halves are whole blocks and whose own keys fit one key tile.
    return m.dtype == SPLITKV_BF16 && m.d == 128 && m.rows_item == 256 && m.pack % 2 == 0 &&
           m.block * m.pack <= kKeysPerTile && m.block * (m.pack / 2) <= 256 && m.group <= 256 &&
           m.total_keys < INT32_MAX && m.n_queries < INT32_MAX;
}

cudaError_t fwd_tc2_max_workers(int32_t* out) {
    // Two-CTA clusters of this kernel that the current device holds at once (GPCs with an odd number
    // of usable SMs leave one SM without a partner).
    cudaError_t e = cudaFuncSetAttribute(fwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(fwd_tc2_kernel, smem)");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 1024, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, fwd_tc2_kernel, &cfg);
    if (e != cudaSuccess) return note_error(e, "cudaOccupancyMaxActiveClusters(fwd_tc2_kernel)");
    *out = n;
    return cudaSuccess;
}

cudaError_t launch_fwd_tc2(const Meta& m, const void* q, const void* k, const void* v, const void* kb,
                           const void* vb, const int32_t* anchors, const int32_t* item_id, const int32_t* queue_off,
                           const int32_t* queue_items, int32_t n_workers, void* o_part, float* lse_part,
                           int32_t* status, void* ws, int32_t flags, cudaStream_t st) {
    CUtensorMap tq, tk, tv, tkb, tvb;
    if (m.n_queries == 0 || m.total_keys == 0) return cudaSuccess;
    if (!make_bf16_map(&tq, q, m.n_queries, m.hq, m.d, m.group, m.block * (m.pack / 2)) ||
        !make_bf16_map(&tk, k, m.total_keys, m.hkv, m.d, 1, kKeysPerTile / 2) ||
        !make_bf16_map(&tv, v, m.total_keys, m.hkv, m.d, 1, kKeysPerTile) ||
        !make_bf16_map(&tkb, kb, m.n_queries, m.hkv, m.d, 1, kKeysPerTile / 2) ||
        !make_bf16_map(&tvb, vb, m.n_queries, m.hkv, m.d, 1, kKeysPerTile))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(fwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(fwd_tc2_kernel, smem)");
    int32_t* pool = reinterpret_cast<int32_t*>(ws);  // the shared pool's claim counter
    e = cudaMemsetAsync(pool, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return note_error(e, "cudaMemsetAsync(pool counter)");
    // Self tiles: every query tile of P blocks, at every kv head.
    int64_t tiles = 0;
    for (int s = 0; s < m.batch; ++s) tiles += (m.anchor_off[s + 1] - m.anchor_off[s] + m.pack - 1) / m.pack;
    const int64_t n_self = tiles * m.hkv;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2u * (unsigned)n_workers, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, fwd_tc2_kernel, m, tq, tk, tv, tkb, tvb, anchors, item_id, queue_off, queue_items,
                           (__nv_bfloat16*)o_part, lse_part, pool, n_self, status,
                           (int32_t)((flags & SPLITKV_FWD_TEST_STARVE) ? 1 : 0));
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        cudaFuncAttributes fa;
        char what[160] = "launch fwd_tc2_kernel";
        if (cudaFuncGetAttributes(&fa, fwd_tc2_kernel) == cudaSuccess)
            std::snprintf(what, sizeof(what),
                          "launch fwd_tc2_kernel (regs %d, local %zu B, static smem %zu B, dyn smem %d B)", fa.numRegs,
                          fa.localSizeBytes, fa.sharedSizeBytes, kSmemBytes);
        return note_error(e, what);
    }
    return cudaSuccess;
}

}  // namespace splitkv
