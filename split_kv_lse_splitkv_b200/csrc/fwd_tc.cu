// Chunk-partial forward on the 5th-generation tensor cores (sm_100a): TMA -> tcgen05.mma -> TMEM.
//
// Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, Abstract: exact
// attention over context chunks, each producing a query-sized partial output and a per-row
// log-sum-exp; the chunks are placed by the cost-aware LPT plan. Here one persistent CTA per SM
// walks the SM's LPT queue. A work item (s, c, g, t) is one 128-row query tile (the block*G rows
// (query i, head g*G+hl) of the tile's blocks at kv head g, shared by the G query heads of the GQA
// group) against the key tiles of chunk c that its rows see. Then self items (block j, kv head g):
// the block's query rows against its own 16 keys (Kb, Vb), one key tile, partial at slot
// n_items + j*Hkv + g. The CTA's key tiles form one sequence n = 0, 1, ... across its items.
//
// Roles (512 threads, four warpgroups; registers moved with setmaxnreg):
//   warps 0-7   softmax: warp w owns rows 32*(w%4) .. +31 (its TMEM lane quadrant) and key columns
//               64*(w/4) .. +63 of every tile; warps w and w+4 (same rows, same SM sub-partition)
//               agree on the row maximum through shared memory. Two warps per sub-partition share
//               each tile's exponentials: one warp alone keeps the MUFU unit only about 60% busy.
//   warps 8-11  epilogue: normalises O of a finished item and stores O_c (bf16), LSE_c
//   warp 12     lane 0: TMA producer (Q per item, K(n), V(n)); lane 1: the claimer (item ring)
//   warp 13     QK issuer (tcgen05.mma S = Q K^T) and TMEM owner
//   warp 14     PV issuer (tcgen05.mma O += P V)
//
// TMEM (512 columns): S[2] = Q K^T of tiles n with n % 2 = 0 / 1 (128 fp32 columns each), with
// P = softmax numerators written over the first 64 columns of S[n % 2] as bf16 pairs, and O[2]
// (128 fp32 columns each) for items k with k % 2 = 0 / 1. The two issuers run on their own: QK(n)
// needs K(n) and PV(n-2) complete (PV(n-2) has read P(n-2) out of S[n % 2]); PV(n) needs P(n), V(n)
// and, for the first tile of item k, the epilogue done with O[k % 2] of item k-2. So QK(n+1)
// computes while the softmax works on tile n, and an item's epilogue overlaps the next item.
// (One thread issuing PV(n) then QK(n+2) in turn measured about 8% slower: a thread that issues
// tcgen05.mma waits while the tensor core works through its previous instruction.)
//
// Online softmax in log2 units (x = s * scale * log2 e). The reference max m of a row only moves
// when a tile's max exceeds it by more than 8 (so P <= 256); a move rescales O (each warp its 64
// columns) and the row sums. Each warp sums P over its columns; the epilogue adds the two sums.
// LSE = (m + log2 l) * ln 2.
//
// Every wait is bounded (2 s); on expiry the CTA raises SPLITKV_DEV_TIMEOUT, drains its copies and
// MMAs in flight, frees TMEM and returns.
#include <cstdio>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_map.cuh"

namespace splitkv {

namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int kEpiWarp0 = 8;
constexpr int kLoadWarp = 12;  // lane 0: TMA producer; lane 1: claimer
constexpr int kMmaWarp = 13;   // QK issuer, TMEM owner
constexpr int kPvWarp = 14;    // PV issuer
constexpr int kSoftmaxRegs = 160;  // per SM sub-partition: 160 + 160 + 88 + 104 = 512 = 4 x 128 launched
constexpr int kEpilogueRegs = 88;
constexpr int kControlRegs = 104;
constexpr int kTileBytes = 32768;  // 128 x 128 bf16, as two 128-byte-wide halves
constexpr int kHalfBytes = 16384;
constexpr int kKeysPerTile = 128;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint64_t kTestLimitNs = 20000ull;  // the starved CTA's limit in test mode (20 us)
constexpr float kRescaleLog2 = 8.0f;
constexpr int kSoftmaxThreads = 256;

constexpr uint32_t kColS = 0, kColO = 256;  // S[b] at 128 b, O[b] at 256 + 128 b

constexpr int kRing = 128;     // entries of the item ring
constexpr int kReaders = 15;   // producer, QK and PV issuers, softmax warps 8, epilogue warps 4
constexpr int32_t kRingEnd = -1;

constexpr int kOffQ = 0;                   // Q[item parity]
constexpr int kOffK = 2 * kTileBytes;      // K[tile parity]
constexpr int kOffV = 4 * kTileBytes;      // V[tile parity]
constexpr int kOffStat = 6 * kTileBytes;   // float [item parity][m, l0, l1][128]
constexpr int kOffXchg = kOffStat + 2 * 3 * 128 * 4;  // float [tile parity][quad][half][32]
constexpr int kOffBar = kOffXchg + 2 * 4 * 2 * 32 * 4;

struct Bars {
    uint64_t q_full[2], q_empty[2];  // Q of item k landed / every QK^T of item k complete (by k % 2)
    uint64_t k_full[2], v_full[2];   // K(n) / V(n) landed (by n % 2)
    uint64_t s_full[2];              // QK^T(n) complete: S(n) ready, and slot K(n % 2) free again
    uint64_t p_full[2];              // P(n) written by all 256 softmax threads
    uint64_t pv_done[2];             // PV(n) complete: slot V(n % 2) free again
    uint64_t o_ready[2];             // last PV of item k complete: O[k % 2] final
    uint64_t o_free[2];              // epilogue has read O[k % 2] of item k
    uint64_t stat_full[2];           // (m, l0, l1) of item k written (by k % 2)
    uint64_t drain[2];               // every MMA of the QK / PV issuer complete
    // The CTA's item sequence, written by one claiming thread, read by every role (see ring_next).
    int32_t ring_id[kRing];          // item id (n_items + j*Hkv + g: self item; kRingEnd: no more)
    int32_t ring_nvis[kRing];        // keys of the chunk its last block sees
    int32_t ring_j[kRing];           // first block of its query tile
    int32_t ring_c[kRing];           // chunk
    int32_t ring_sgn[kRing];         // sample | blocks in the tile << 8 | kv head << 16
    int32_t ring_w;                  // entries written
    int32_t ring_r[kReaders];        // entries read, per reader
    int32_t xflag[4][2];             // [quad][half]: tiles whose half row max is in xchg
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

constexpr int kSortCap = 512;  // longest queue executed in item-id order (see sort_queue)
constexpr int kOffSort = (kOffBar + (int)sizeof(Bars) + 15) / 16 * 16;
constexpr int kSmemBytes = kOffSort + kSortCap * 4 + 1024;  // + alignment slack

struct TileRef {
    int64_t id;                // partial slot: item id, or n_items + j*Hkv + g for a self item
    int32_t s, c, g, j;
    int32_t nvis, ntiles;      // keys its last block sees (the most), key tiles
    int32_t nbt;               // blocks in the query tile (rows of block x: x*block*G ..)
    int32_t self_item;         // 1: keys are the block's own (Kb/Vb rows block*j ..)
};

// S columns 64h .. 64h+63 of this thread's row; keys at or beyond `valid` read as -inf.
__device__ __forceinline__ void load_half(uint32_t ts, int h, int valid, uint32_t (&ra)[32], uint32_t (&rb)[32]) {
    tmem_ld32(ts + h * 64, ra);
    tmem_ld32(ts + h * 64 + 32, rb);
    tmem_wait_ld();
    if (valid < h * 64 + 64) {
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            if (h * 64 + u >= valid) ra[u] = __float_as_uint(-INFINITY);
            if (h * 64 + 32 + u >= valid) rb[u] = __float_as_uint(-INFINITY);
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
// The CTA's work is its LPT queue, in queue order, then self items (one key tile each, outside the
// plan) claimed one at a time through a global counter once its own work runs low, so that SMs that
// finish their queue early take more of them. (Also putting the smallest quarter of every queue into
// that pool was measured slower.) One thread, the claimer, turns this into the CTA's item sequence,
// written decoded into a ring in shared memory that every role reads in order.

// Next ring entry. blocking: wait for it; otherwise return 0 at once if none has been written.
// Returns 1 (entry in t), or -1 at the end of the sequence or on abort/timeout. `slot` is this
// reader's progress word; a warp-wide reader (all 32 lanes in step) publishes after __syncwarp.
__device__ __forceinline__ int ring_next(const Meta& m, Bars* bars, int32_t& idx, int slot, bool blocking,
                                         bool warp_wide, TileRef& t, volatile int* abort_flag, uint64_t lim) {
    volatile int32_t* rw = &bars->ring_w;
    uint64_t t0 = 0;
    for (uint32_t spin = 0;; ++spin) {
        if (idx < *rw) {
            const int e = idx % kRing;
            const int32_t id = ((volatile int32_t*)bars->ring_id)[e];
            const int32_t nvis = ((volatile int32_t*)bars->ring_nvis)[e];
            const int32_t jj = ((volatile int32_t*)bars->ring_j)[e];
            const int32_t cc = ((volatile int32_t*)bars->ring_c)[e];
            const int32_t sgn = ((volatile int32_t*)bars->ring_sgn)[e];
            if (id == kRingEnd) return -1;  // the end entry stays: every later call sees it again
            ++idx;
            if (warp_wide) __syncwarp();
            if (!warp_wide || (threadIdx.x & 31) == 0) ((volatile int32_t*)bars->ring_r)[slot] = idx;
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
        if (!blocking) return 0;
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

// Execution order of the CTA's queue: ascending item id. The plan fixes which items an SM runs (its load
// does not depend on their order); ids are chunk-major (sample, run of chunks, kv head, query tile), so in
// id order every SM walks the context from its start and the items that read one run's K/V, full or
// partial, run at about the same time on all SMs, while that K/V is in L2 (in plan order, cost
// descending, the partial runs come last and read their K/V from DRAM again). Used when the problem's
// K and V exceed the L2 cache (otherwise plan order: measured 1.6 % faster on a 67 MB context). One warp
// sorts the queue (bitonic, in shared memory) before its lanes take their roles; queues longer than
// kSortCap keep plan order. Returns the number of sorted entries, or -1. Invalid ids raise
// SPLITKV_DEV_BAD_PLAN and sort last as INT32_MAX.
__device__ int32_t sort_queue(const Meta& m, const int32_t* __restrict__ item_id,
                              const int32_t* __restrict__ queue_off, const int32_t* __restrict__ queue_items,
                              int32_t* s, int32_t* status) {
    const int lane = threadIdx.x & 31;
    const int32_t q0 = queue_off[blockIdx.x], n = queue_off[blockIdx.x + 1] - q0;
    if (n <= 0 || n > kSortCap) return -1;
    int P = 32;
    while (P < n) P <<= 1;
    for (int i = lane; i < P; i += 32) {
        int32_t id = INT32_MAX;
        if (i < n) {
            id = __ldg(item_id + __ldg(queue_items + q0 + i));
            if (id < 0 || id >= m.n_items) {
                raise_status(status, SPLITKV_DEV_BAD_PLAN);
                id = INT32_MAX;
            }
        }
        s[i] = id;
    }
    __syncwarp();
    for (int k = 2; k <= P; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = lane; i < P; i += 32) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const int32_t a = s[i], b = s[ixj];
                    if ((a > b) == ((i & k) == 0)) {
                        s[i] = b;
                        s[ixj] = a;
                    }
                }
            }
            __syncwarp();
        }
    return n;
}

// The claimer: the CTA's queue (in id order when sorted), then self items while the producer runs low,
// then the end entry. One thread.
__device__ void claim_items(const Meta& m, Bars* bars, const int32_t* __restrict__ anchors,
                            const int32_t* __restrict__ item_id, const int32_t* __restrict__ queue_off,
                            const int32_t* __restrict__ queue_items, const int32_t* sorted, int32_t n_sorted,
                            int32_t* pool, int32_t* status, volatile int* abort_flag, uint64_t lim) {
    const int32_t q0 = queue_off[blockIdx.x], q1 = queue_off[blockIdx.x + 1];
    volatile int32_t* rr = bars->ring_r;
    int32_t w = 0;
    bool ok = true;
    // Wait until slot w is free (every reader is past entry w - kRing) and, if ahead > 0, until the
    // producer (reader 0) has fewer than `ahead` entries left to read.
    auto wait_room = [&](int ahead) -> bool {
        const uint64_t t0 = globaltimer();
        for (uint32_t spin = 0;; ++spin) {
            int32_t lo = rr[0];
            for (int x = 1; x < kReaders; ++x) lo = min(lo, rr[x]);
            if (lo > w - kRing && (ahead <= 0 || rr[0] > w - ahead)) return true;
            if ((spin & 63u) == 63u && (*abort_flag || globaltimer() - t0 > lim)) {
                *abort_flag = 1;
                return false;
            }
            __nanosleep(64);
        }
    };
    auto put = [&](int32_t id, int32_t nvis) {
        const int e = w % kRing;
        int32_t j = 0, c = 0, sgn = 0;
        if (id >= m.n_items) {  // self item n_items + j*Hkv + g
            const int32_t sid = id - (int32_t)m.n_items;
            j = sid / m.hkv;
            sgn = sample_of_block(m, j) | (1 << 8) | ((sid % m.hkv) << 16);
        } else if (id >= 0) {
            const Item it = decode_item(m, id);
            j = it.j;
            c = it.c;
            sgn = it.s | (it.nbt << 8) | (it.g << 16);
        }
        ((volatile int32_t*)bars->ring_id)[e] = id;
        ((volatile int32_t*)bars->ring_nvis)[e] = nvis;
        ((volatile int32_t*)bars->ring_j)[e] = j;
        ((volatile int32_t*)bars->ring_c)[e] = c;
        ((volatile int32_t*)bars->ring_sgn)[e] = sgn;
        __threadfence_block();
        ++w;
        ((volatile int32_t*)&bars->ring_w)[0] = w;
    };
    const int32_t n_q = n_sorted >= 0 ? n_sorted : q1 - q0;
    for (int32_t x = 0; ok && x < n_q; ++x) {
        const int32_t id = n_sorted >= 0 ? sorted[x] : __ldg(item_id + __ldg(queue_items + q0 + x));
        if (id < 0 || id >= m.n_items) {
            if (n_sorted < 0) raise_status(status, SPLITKV_DEV_BAD_PLAN);  // (sort_queue raised it)
            continue;
        }
        const Item it = decode_item(m, id);
        const int32_t nvis = visible_in_chunk(m, it.s, it.c, __ldg(anchors + it.j + it.nbt - 1));
        if (nvis <= 0) continue;
        ok = wait_room(0);
        if (ok) put(id, nvis);
    }
    const int64_t n_self = m.n_blocks * m.hkv;
    while (ok) {
        // Claim when the producer has fewer than 2 entries left to read.
        if (!wait_room(2)) {
            ok = false;
            break;
        }
        const int64_t p = atomicAdd(pool, 1);
        if (p >= n_self) break;
        put((int32_t)(m.n_items + p), m.block);
    }
    if (ok && wait_room(0)) put(kRingEnd, 0);
}

// Keys of the chunk that row r of query tile t sees: its own block's prefix (a row of no block of
// the tile, or of a self item beyond the block's own rows, sees none). A row's keys lie in the
// item's first key tiles.
__device__ __forceinline__ int32_t row_keys(const Meta& m, const int32_t* __restrict__ anchors, const TileRef& t,
                                            int r) {
    const int32_t x = r / m.rows;
    if (t.self_item) return x == 0 ? m.block : 0;
    return x < t.nbt ? visible_in_chunk(m, t.s, t.c, __ldg(anchors + t.j + x)) : 0;
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
    fwd_tc_kernel(const __grid_constant__ Meta m, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
                  const int32_t* __restrict__ anchors, const int32_t* __restrict__ item_id,
                  const int32_t* __restrict__ queue_off, const int32_t* __restrict__ queue_items,
                  __nv_bfloat16* __restrict__ o_part, float* __restrict__ lse_part, int32_t* __restrict__ pool,
                  int32_t* __restrict__ status, int32_t mode) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* stat = reinterpret_cast<float*>(smem + kOffStat);
    float* xchg = reinterpret_cast<float*>(smem + kOffXchg);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Limit of every wait that can run out while work is expected (drains keep the full limit).
    // mode bit 0: test of the wait limit (SPLITKV_FWD_TEST_STARVE); bit 1: run the queue in item-id order.
    const bool test_starve = (mode & 1) != 0;
    const uint64_t lim = (test_starve && blockIdx.x == 0) ? kTestLimitNs : kTimeoutNs;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
            mbar_init(&bars->k_full[b], 1);
            mbar_init(&bars->v_full[b], 1);
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->p_full[b], kSoftmaxThreads);
            mbar_init(&bars->pv_done[b], 1);
            mbar_init(&bars->o_free[b], 128);
            mbar_init(&bars->stat_full[b], kSoftmaxThreads);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->o_ready[b], 1);
            mbar_init(&bars->drain[b], 1);
        }
        bars->ring_w = 0;
        for (int x = 0; x < kReaders; ++x) bars->ring_r[x] = 0;
        for (int x = 0; x < 8; ++x) (&bars->xflag[0][0])[x] = 0;
        bars->abort_flag = 0;
        bars->status0 = status_bad(status) ? 1 : 0;
        fence_barrier_init();
    }
    // Rows of the Q buffers beyond the tile's rows are never loaded: keep them finite (zero).
    for (int i = threadIdx.x; i < 2 * kTileBytes / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem + kOffQ)[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == kMmaWarp) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const bool skip = bars->status0 != 0;  // every CTA may take self items
    const int G = m.group, R = m.rows_item;

    if (warp >= kLoadWarp) {
        // ------------------------------------------------------------ control warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kControlRegs));
        int32_t* qsort = reinterpret_cast<int32_t*>(smem + kOffSort);
        int32_t n_sorted = -1;
        if (!skip && warp == kLoadWarp && (mode & 2))
            n_sorted = sort_queue(m, item_id, queue_off, queue_items, qsort, status);
        if (!skip && warp == kLoadWarp && lane == 0) {
            // TMA producer: Q of item k (slot k % 2), then K(n) and V(n) of its key tiles (slot n % 2).
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            const uint32_t q_bytes = 2u * 64u * (uint32_t)G * (uint32_t)(m.block * m.pack) * 2u;
            int32_t ridx = 0;
            TileRef t;
            uint32_t k = 0, nk = 0, nv = 0;  // copies issued: Q, K, V
            bool ok = true;
            while (ok && ring_next(m, bars, ridx, 0, true, false, t, abort_flag, lim) == 1) {
                const int qb = k & 1;
                if (k >= 2 && !mbar_wait(&bars->q_empty[qb], ((k >> 1) - 1) & 1u, abort_flag, lim)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars->q_full[qb], q_bytes);
                uint8_t* qdst = smem + kOffQ + qb * kTileBytes;
                tma_load_3d(qdst, &tmQ, &bars->q_full[qb], 0, t.g * G, m.block * t.j);
                tma_load_3d(qdst + kHalfBytes, &tmQ, &bars->q_full[qb], 64, t.g * G, m.block * t.j);
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
                    if (!mbar_wait(&bars->s_full[b], ph, abort_flag, lim)) {  // QK(n-2) done
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->k_full[b], kTileBytes);
                    uint8_t* kdst = smem + kOffK + b * kTileBytes;
                    tma_load_3d(kdst, mk, &bars->k_full[b], 0, t.g, row);
                    tma_load_3d(kdst + kHalfBytes, mk, &bars->k_full[b], 64, t.g, row);
                    ++nk;
                    if (!mbar_wait(&bars->pv_done[b], ph, abort_flag, lim)) {  // PV(n-2) done
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->v_full[b], kTileBytes);
                    uint8_t* vdst = smem + kOffV + b * kTileBytes;
                    tma_load_3d(vdst, mv, &bars->v_full[b], 0, t.g, row);
                    tma_load_3d(vdst + kHalfBytes, mv, &bars->v_full[b], 64, t.g, row);
                    ++nv;
                }
            }
            if (!ok) *abort_flag = 1;
            // Drain: the most recent copies into every buffer have landed before the CTA exits.
            volatile int never = 0;
            for (uint32_t x = (k > 2 ? k - 2 : 0); x < k; ++x)
                mbar_wait(&bars->q_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
            for (uint32_t x = (nk > 2 ? nk - 2 : 0); x < nk; ++x)
                mbar_wait(&bars->k_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
            for (uint32_t x = (nv > 2 ? nv - 2 : 0); x < nv; ++x)
                mbar_wait(&bars->v_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
        } else if (!skip && warp == kLoadWarp && lane == 1) {
            // Test mode (SPLITKV_FWD_TEST_STARVE): the first CTA's claimer publishes nothing, so every
            // role of that CTA waits for its first item with no copy or MMA issued, and gives up.
            if (!(test_starve && blockIdx.x == 0))
                claim_items(m, bars, anchors, item_id, queue_off, queue_items, qsort, n_sorted, pool, status,
                            abort_flag, lim);
        } else if (!skip && (warp == kMmaWarp || warp == kPvWarp) && lane == 0) {
            // Two issuers on one tensor core. QK issuer: S[n % 2] = Q K(n)^T once K(n) has landed and
            // PV(n-2) has read P(n-2) out of S[n % 2]. PV issuer: O[k % 2] += P(n) V(n) once P(n) is
            // written; the first PV of item k also waits until the epilogue has read O[k % 2] of item k-2.
            const bool is_qk = warp == kMmaWarp;
            constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, 128, false, true);
            // Descriptor bases; a K step only adds a constant to the (16-byte unit) start address.
            uint64_t dq[2], dk[2], dv[2];
            for (int b = 0; b < 2; ++b) {
                dq[b] = umma_desc_sw128(smem_u32(smem + kOffQ + b * kTileBytes), 16, 1024);
                dk[b] = umma_desc_sw128(smem_u32(smem + kOffK + b * kTileBytes), 16, 1024);
                dv[b] = umma_desc_sw128(smem_u32(smem + kOffV + b * kTileBytes), kHalfBytes, 1024);
            }
            int32_t ridx = 0;
            TileRef t;
            uint32_t k = 0, n = 0;
            bool ok = true;
            while (ok && ring_next(m, bars, ridx, is_qk ? 1 : 2, true, false, t, abort_flag, lim) == 1) {
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
                            const uint64_t off = (uint64_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) / 16);
                            mma_ss(ts, dq[ib] + off, dk[b] + off, idesc_qk, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&bars->s_full[b]);
                        if (tt == t.ntiles - 1) mma_commit(&bars->q_empty[ib]);
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
                            mma_ts(tO, tp + (uint32_t)(kk * 8), dv[b] + (uint64_t)(kk * 2048 / 16), idesc_pv,
                                   (tt > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&bars->pv_done[b]);
                        if (tt == t.ntiles - 1) mma_commit(&bars->o_ready[ib]);
                    }
                }
                ++k;
            }
            if (!ok) *abort_flag = 1;
            // Drain: all MMAs issued by this thread complete before TMEM is released.
            uint64_t* dr = &bars->drain[is_qk ? 0 : 1];
            mma_commit(dr);
            volatile int never = 0;
            mbar_wait(dr, 0, &never, kTimeoutNs);
        }
        __syncwarp();
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------------ epilogue warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kEpilogueRegs));
        if (!skip) {
            const int quad = warp & 3;
            const int r = quad * 32 + lane;
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            int32_t ridx = 0;
            TileRef t;
            uint32_t k = 0;
            bool ok = true;
            while (ok && ring_next(m, bars, ridx, 11 + quad, true, true, t, abort_flag, lim) == 1) {
                const int ob = k & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(&bars->stat_full[ob], (k >> 1) & 1u, abort_flag, lim) &&
                                                 mbar_wait(&bars->o_ready[ob], (k >> 1) & 1u, abort_flag, lim));
                if (!ok) break;
                tc_fence_after();
                const float* sp = stat + ob * 384;
                const float m_l = sp[r], l = sp[128 + r] + sp[256 + r];  // the two column halves' sums
                const uint32_t to = tmem + kColO + 128u * ob + lane_off;
                const float inv = l > 0.f ? 1.f / l : 0.f;  // a row that sees no key: O = 0, LSE = -inf
                __nv_bfloat16* op = o_part + t.id * (int64_t)R * 128;  // [d/8][R][8] bf16
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    uint32_t ov[16];
                    tmem_ld16(to + cc * 16, ov);
                    tmem_wait_ld();
                    if (cc == 7) {  // O[k % 2] fully read: the PV issuer may start item k+2 in it
                        tc_fence_before();
                        mbar_arrive(&bars->o_free[ob]);
                    }
                    if (r < R) {  // 16 columns: two groups of 8 bf16, 16 bytes each
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(ov[8 * u + 2 * e]) * inv,
                                                                         __uint_as_float(ov[8 * u + 2 * e + 1]) * inv);
                                pk[e] = *reinterpret_cast<uint32_t*>(&h);
                            }
                            *reinterpret_cast<uint4*>(op + ((int64_t)(cc * 2 + u) * R + r) * 8) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
                if (r < R)
                    lse_part[t.id * R + r] = l > 0.f ? (m_l + lg2_approx(l)) * 0.6931471805599453f : -INFINITY;
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
            const int r = quad * 32 + lane;         // query-tile row
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
            while (ok && ring_next(m, bars, ridx, 3 + warp, true, true, t, abort_flag, lim) == 1) {
                const int32_t row_nvis = row_keys(m, anchors, t, r);
                float m_l = -INFINITY, l = 0.f;  // reference max and this half's row sum (relative to m_l)
                for (int32_t tt = 0; tt < t.ntiles; ++tt, ++n) {
                    // The whole warp leaves together on a timeout: the TMEM accesses below are collective.
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[n & 1], (n >> 1) & 1u, abort_flag, lim))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ts = tmem + kColS + 128u * (n & 1) + lane_off;  // S(n), this row
                    const int valid = row_nvis - tt * kKeysPerTile - 64 * half;  // keys of my columns it sees
                    uint32_t ra[32], rb[32];
                    load_half(ts, half, valid + 64 * half, ra, rb);
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
                    mbar_arrive(&bars->p_full[n & 1]);
                }
                if (!ok) break;
                // Hand (m, l) of item k to the epilogue; stat[k % 2] was last read for item k-2.
                const int ob = k & 1;
                if (k >= 2 && !mbar_wait(&bars->o_free[ob], ((k >> 1) - 1) & 1u, abort_flag, lim)) {
                    ok = false;
                    break;
                }
                float* sp = stat + ob * 384;
                if (half == 0) sp[r] = m_l;
                sp[128 + 128 * half + r] = l;
                mbar_arrive(&bars->stat_full[ob]);
                ++k;
            }
            if (!ok) *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && bars->abort_flag) raise_status(status, SPLITKV_DEV_TIMEOUT);
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D bf16 map (declared in tma_map.cuh) over [rows][heads][d] with a 128-byte swizzled box {64, box_heads, box_rows}.
bool make_bf16_map(CUtensorMap* map, const void* base, int64_t rows, int heads, int d, int box_heads, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        note_error(cudaErrorNotSupported, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
        return false;
    }
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char what[96];
        std::snprintf(what, sizeof(what), "cuTensorMapEncodeTiled -> CUresult %d", (int)r);
        note_error(cudaErrorInvalidValue, what);
        return false;
    }
    return true;
}


bool fwd_tc_supported(const Meta& m) {
    return m.dtype == SPLITKV_BF16 && m.d == 128 && m.rows_item <= 128 && m.block <= 256 && m.group <= 256 &&
           m.total_keys < INT32_MAX && m.n_queries < INT32_MAX;
}

cudaError_t launch_fwd_tc(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                          const int32_t* anchors, const int32_t* item_id, const int32_t* queue_off,
                          const int32_t* queue_items, int32_t n_workers, void* o_part, float* lse_part,
                          int32_t* status, void* ws, int32_t flags, cudaStream_t st) {
    CUtensorMap tq, tk, tv, tkb, tvb;
    if (m.n_queries == 0 || m.total_keys == 0) return cudaSuccess;
    if (!make_bf16_map(&tq, q, m.n_queries, m.hq, m.d, m.group, m.block * m.pack) ||
        !make_bf16_map(&tk, k, m.total_keys, m.hkv, m.d, 1, kKeysPerTile) ||
        !make_bf16_map(&tv, v, m.total_keys, m.hkv, m.d, 1, kKeysPerTile) ||
        !make_bf16_map(&tkb, kb, m.n_queries, m.hkv, m.d, 1, kKeysPerTile) ||
        !make_bf16_map(&tvb, vb, m.n_queries, m.hkv, m.d, 1, kKeysPerTile))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(fwd_tc_kernel, smem)");
    int32_t* pool = reinterpret_cast<int32_t*>(ws);  // the shared pool's claim counter
    e = cudaMemsetAsync(pool, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return note_error(e, "cudaMemsetAsync(pool counter)");
    // Item-id order when K and V do not fit in L2 (see sort_queue).
    int dev = 0, l2 = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
    if (e != cudaSuccess) return note_error(e, "cudaDeviceGetAttribute(L2 size)");
    const double kv_bytes = 2.0 * (double)m.total_keys * m.hkv * m.d * 2.0;
    const int32_t mode = ((flags & SPLITKV_FWD_TEST_STARVE) ? 1 : 0) | (kv_bytes > (double)l2 ? 2 : 0);
    fwd_tc_kernel<<<n_workers, kThreads, kSmemBytes, st>>>(m, tq, tk, tv, tkb, tvb, anchors, item_id, queue_off,
                                                           queue_items, (__nv_bfloat16*)o_part, lse_part, pool, status,
                                                           mode);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        cudaFuncAttributes fa;
        char what[160] = "launch fwd_tc_kernel";
        if (cudaFuncGetAttributes(&fa, fwd_tc_kernel) == cudaSuccess)
            std::snprintf(what, sizeof(what), "launch fwd_tc_kernel (regs %d, local %zu B, static smem %zu B, dyn smem %d B)",
                          fa.numRegs, fa.localSizeBytes, fa.sharedSizeBytes, kSmemBytes);
        return note_error(e, what);
    }
    return cudaSuccess;
}

}  // namespace splitkv
