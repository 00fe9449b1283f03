// Chunk-partial forward on the 5th-generation tensor cores (sm_100a): TMA -> tcgen05.mma -> TMEM.
//
// Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, Abstract: exact
// attention over context chunks, each producing a query-sized partial output and a per-row
// log-sum-exp; the chunks are placed by the cost-aware LPT plan. Here one persistent CTA per SM
// walks the SM's LPT queue. A work item (s, c, g, b) is one 128-row query tile — the block*G rows
// (query i, head g*G+hl) of block b at kv head g, shared by the G query heads of the GQA group —
// against the ceil(nvis/128) key tiles of chunk c that the block sees. After its queue, every CTA
// also takes a share of the self items (block j, kv head g): the same query tile against the
// block's own 16 keys (Kb, Vb), one tile with 16 visible keys, whose partial goes to slot
// n_items + j*Hkv + g. The CTA's key tiles form one sequence n = 0, 1, ... across its items
// i = 0, 1, ...
//
// Two lanes. The CTA's items are dealt to two independent pipelines (lanes), each item to the
// lane with fewer key tiles so far (ties to lane 0); every role derives the same split from the
// item list. A lane owns its Q, K and V buffers, its S and O in TMEM, a softmax warpgroup, an MMA
// issuer and a TMA producer; the lanes share only the tensor core and the epilogue, so one lane's
// exponentials overlap the other's matrix products.
//
// Roles (512 threads, four warpgroups; registers moved with setmaxnreg):
//   WG0 / WG1 (warps 0-7)  softmax of lane 0 / 1: row r = 32*(warp%4) + lane
//   WG2 (warps 8-11)       epilogue: stores O_c, LSE_c of whichever lane finished an item
//   warp 12 / 15           TMA producer of lane 0 / 1: Q per item, K(n) and V(n) per key tile
//   warp 13 / 14           tcgen05.mma issuer of lane 0 / 1 (warp 13 owns TMEM)
//
// TMEM (512 columns): S_L = Q K^T of lane L's current key tile (128 fp32 columns at 128 L), with
// P_L = softmax numerators written over its first 64 columns as bf16 pairs, and O_L (128 fp32
// columns at 256 + 128 L). Issuer L runs QK(n) -> [P(n) ready] -> PV(n) -> QK(n+1) -> ...: the
// tensor core executes one thread's MMAs in issue order, so QK(n+1) overwrites S_L only after
// PV(n) has read P_L from it, and S_L(n+1) ready implies PV(n) complete (so O_L is current when
// the softmax rescales it). A thread issuing tcgen05.mma waits while the tensor core works through
// its previous instruction; two issuers with independent chains keep it busy.
//
// Online softmax in log2 units (x = s * scale * log2 e). The reference max m of a row only moves
// when a tile's max exceeds it by more than 8 (so P <= 256); a move rescales O_L and the row sum l.
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
constexpr int kLoadWarp0 = 12;  // TMA producer of lane 0 (lane 1: warp 15)
constexpr int kLoadWarp1 = 15;
constexpr int kMmaWarp0 = 13;  // issuer of lane 0, TMEM owner (lane 1: warp 14)
constexpr int kMmaWarp1 = 14;
constexpr int kSoftmaxRegs = 160;  // per SM sub-partition: 160 + 160 + 88 + 104 = 512 = 4 x 128 launched
constexpr int kEpilogueRegs = 88;
constexpr int kControlRegs = 104;
constexpr int kTileBytes = 32768;  // 128 x 128 bf16, as two 128-byte-wide halves
constexpr int kHalfBytes = 16384;
constexpr int kKeysPerTile = 128;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kWgThreads = 128;

constexpr uint32_t kColS = 0, kColO = 256;  // S_L at 128 L, O_L at 256 + 128 L

constexpr int kRing = 128;           // entries of the item ring
constexpr int kReaders = 20;         // producers 2, issuers 2, softmax warps 8, epilogue warps 4 x 2 lanes
constexpr int32_t kRingEnd = -1;

constexpr int kOffQ = 0;                  // Q[lane]
constexpr int kOffK = 2 * kTileBytes;     // K[lane]
constexpr int kOffV = 4 * kTileBytes;     // V[lane]
constexpr int kOffStat = 6 * kTileBytes;  // float [lane][item parity][m, l][128]
constexpr int kOffBar = kOffStat + 2 * 2 * 2 * 128 * 4;

// Per lane L (one buffer each; phases count the lane's items k or key tiles n).
struct Bars {
    uint64_t q_full[2], q_empty[2];  // Q of item k landed / every QK^T of item k complete
    uint64_t k_full[2], k_empty[2];  // K(n) landed / QK^T(n) complete
    uint64_t v_full[2], v_empty[2];  // V(n) landed / PV(n) complete
    uint64_t s_full[2];              // QK^T(n) complete
    uint64_t p_full[2];              // P(n) written
    uint64_t o_ready[2];             // last PV of item k complete
    uint64_t o_free[2][2];           // [lane][k % 2]: epilogue has read O_L of item k
    uint64_t stat_full[2][2];        // [lane][k % 2]: (m, l) of item k written
    uint64_t drain[2];               // all MMAs of issuer L complete
    int32_t exp_slot[4];             // per SM sub-partition: 1 while a softmax warp is in its exponential pass
    // The CTA's item sequence, written by one claiming thread, read by every role (see ring_next).
    int32_t ring_id[kRing];          // item id (n_items + j*Hkv + g: self item; kRingEnd: no more)
    int32_t ring_lane[kRing];        // lane the item is dealt to
    int32_t ring_nvis[kRing];        // keys of the chunk its last block sees
    int32_t ring_j[kRing];           // first block of its query tile
    int32_t ring_c[kRing];           // chunk
    int32_t ring_sgn[kRing];         // sample | blocks in the tile << 8 | kv head << 16
    int32_t ring_w;                  // entries written
    int32_t ring_r[kReaders];        // entries read, per reader
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

constexpr int kSmemBytes = kOffBar + (int)sizeof(Bars) + 1024;  // + alignment slack

struct TileRef {
    int64_t id;                // partial slot: item id, or n_items + j*Hkv + g for a self item
    int32_t s, c, g, j;
    int32_t nvis, ntiles;      // keys its last block sees (the most), key tiles
    int32_t nbt;               // blocks in the query tile (rows of block x: x*block*G ..)
    int32_t self_item;         // 1: keys are the block's own (Kb/Vb rows block*j ..)
};

// The CTA's items (queue positions first, first+1, ...), fetched ahead: each call hands out the
// next (item id, anchor) and issues the loads one link further for the three items after it
// (anchor of n+1, id of n+2, queue entry of n+3), so no role waits on a dependent global load
// chain when it moves to a new item. The self items follow the queue.
struct ItemStream {
    int32_t pos, end, left;
    int64_t id1;  // item n+1 (loaded)
    int32_t a1;   // anchor of item n+1 (in flight)
    int64_t id2;  // item n+2 (in flight)
    int32_t k3;   // queue entry of item n+3 (in flight)
    int32_t self_pos, self_n;  // self items blockIdx.x, blockIdx.x + gridDim.x, ... < self_n
};

__device__ __forceinline__ int64_t load_id(const int32_t* __restrict__ item_id, int32_t k) {
    return k >= 0 ? (int64_t)__ldg(item_id + k) : -1;
}
__device__ __forceinline__ int32_t load_anchor(const Meta& m, const int32_t* __restrict__ anchors, int64_t id) {
    if (id < 0 || id >= m.n_items) return 0;
    const Item it = decode_item(m, id);
    return __ldg(anchors + it.j + it.nbt - 1);  // the tile's largest anchor
}

__device__ __forceinline__ void stream_init(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                            const int32_t* queue_items, int32_t first, int32_t end, ItemStream& st) {
    st.end = end;
    st.left = first < end ? end - first : 0;
    const int32_t k0 = st.left > 0 ? __ldg(queue_items + first) : -1;
    const int32_t k1 = st.left > 1 ? __ldg(queue_items + first + 1) : -1;
    st.k3 = st.left > 2 ? __ldg(queue_items + first + 2) : -1;
    st.id1 = load_id(item_id, k0);
    st.id2 = load_id(item_id, k1);
    st.a1 = load_anchor(m, anchors, st.id1);
    st.pos = first + 3;
    st.self_pos = blockIdx.x;
    st.self_n = (int32_t)(m.n_blocks * m.hkv);
}

__device__ __forceinline__ bool stream_more(const ItemStream& st) { return st.left > 0 || st.self_pos < st.self_n; }

// Next item as a tile reference (ntiles == 0 for an invalid entry, which raises BAD_PLAN).
__device__ __forceinline__ void stream_next(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                            const int32_t* queue_items, ItemStream& st, TileRef& tr, int32_t* status) {
    if (st.left <= 0) {  // self item
        const int32_t sid = st.self_pos;
        st.self_pos += gridDim.x;
        tr.self_item = 1;
        tr.id = m.n_items + sid;
        tr.j = sid / m.hkv;
        tr.g = sid % m.hkv;
        tr.s = sample_of_block(m, tr.j);
        tr.c = 0;
        tr.nvis = m.block;
        tr.ntiles = 1;
        tr.nbt = 1;
        return;
    }
    tr.self_item = 0;
    const int64_t id = st.id1;
    const int32_t a = st.a1;
    --st.left;
    st.a1 = load_anchor(m, anchors, st.id2);
    st.id1 = st.id2;
    st.id2 = load_id(item_id, st.k3);
    st.k3 = st.pos < st.end ? __ldg(queue_items + st.pos) : -1;
    st.pos += 1;
    if (id < 0 || id >= m.n_items) {
        raise_status(status, SPLITKV_DEV_BAD_PLAN);
        tr.ntiles = 0;
        return;
    }
    const Item it = decode_item(m, id);
    tr.id = id;
    tr.s = it.s;
    tr.c = it.c;
    tr.g = it.g;
    tr.j = it.j;
    tr.nbt = it.nbt;
    tr.nvis = visible_in_chunk(m, it.s, it.c, a);
    tr.ntiles = (tr.nvis + kKeysPerTile - 1) / kKeysPerTile;
}

// Next valid item (ntiles > 0); false at the end of the CTA's work.
__device__ __forceinline__ bool next_item(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                          const int32_t* queue_items, ItemStream& st, TileRef& tr, int32_t* status) {
    while (stream_more(st)) {
        stream_next(m, anchors, item_id, queue_items, st, tr, status);
        if (tr.ntiles > 0) return true;
    }
    return false;
}

// The two softmax warps of one SM sub-partition (warp q of each lane) take turns in the
// exponential pass: the MUFU unit is the sub-partition's bottleneck, and when the passes alternate,
// each lane's exponentials overlap the other lane's matrix products. Lane 0 of the warp takes the
// slot; false on abort or after the time limit.
__device__ __forceinline__ bool exp_slot_take(int32_t* slot, volatile int* abort_flag, uint64_t limit_ns) {
    bool got = false;
    if ((threadIdx.x & 31) == 0) {
        const uint64_t t0 = globaltimer();
        for (uint32_t n = 0;; ++n) {
            if (atomicCAS(slot, 0, 1) == 0) {
                got = true;
                break;
            }
            __nanosleep(32);
            if ((n & 63u) == 63u && (*abort_flag || globaltimer() - t0 > limit_ns)) break;
        }
    }
    return __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ void exp_slot_give(int32_t* slot) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) atomicExch(slot, 0);
}

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

// O_L *= alpha for this thread's row (128 columns).
__device__ __forceinline__ void rescale_o(uint32_t to, float alpha) {
#pragma unroll 1
    for (int cc = 0; cc < 8; ++cc) {
        uint32_t ov[16];
        tmem_ld16(to + cc * 16, ov);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * alpha);
        tmem_st16(to + cc * 16, ov);
    }
}

// ---------------------------------------------------------------- item ring
// The CTA's work is its LPT queue, in queue order, then self items (one key tile each, outside the
// plan) claimed one at a time through a global counter once its own work runs low, so that SMs that
// finish their queue early take more of them. (Also putting the smallest quarter of every queue into
// that pool was measured slower: 310 vs 295 us on the 32k-context drafter shape.) One thread, the
// claimer, turns this into the CTA's item sequence: it deals each item to the lane with fewer key
// tiles so far and writes the decoded item into a ring in shared memory that every role reads.

// Next ring entry for lane L, or for either lane if L < 0. blocking: wait for the entry; otherwise
// return 0 at once if none has been written. Returns 1 (entry in t, its lane in *lane_out), or -1 at
// the end of the sequence or on abort/timeout. `slot` is this reader's progress word; a warp-wide
// reader (all 32 lanes in step) publishes after __syncwarp.
__device__ __forceinline__ int ring_next(const Meta& m, Bars* bars, int32_t& idx, int slot, int L, bool blocking,
                                         bool warp_wide, TileRef& t, int* lane_out, volatile int* abort_flag) {
    volatile int32_t* rw = &bars->ring_w;
    uint64_t t0 = 0;
    for (uint32_t spin = 0;; ++spin) {
        if (idx < *rw) {
            const int e = idx % kRing;
            const int32_t id = ((volatile int32_t*)bars->ring_id)[e];
            const int lane = ((volatile int32_t*)bars->ring_lane)[e];
            const int32_t nvis = ((volatile int32_t*)bars->ring_nvis)[e];
            const int32_t jj = ((volatile int32_t*)bars->ring_j)[e];
            const int32_t cc = ((volatile int32_t*)bars->ring_c)[e];
            const int32_t sgn = ((volatile int32_t*)bars->ring_sgn)[e];
            if (id == kRingEnd) return -1;  // the end entry stays: every later call sees it again
            ++idx;
            if (warp_wide) __syncwarp();
            if (!warp_wide || (threadIdx.x & 31) == 0) ((volatile int32_t*)bars->ring_r)[slot] = idx;
            if (L >= 0 && lane != L) continue;
            *lane_out = lane;
            t.nvis = nvis;
            t.ntiles = (nvis + kKeysPerTile - 1) / kKeysPerTile;
            t.id = id;
            t.self_item = id >= m.n_items ? 1 : 0;
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
            else if (globaltimer() - t0 > kTimeoutNs) {
                *abort_flag = 1;
                return -1;
            }
        }
        __nanosleep(32);
    }
}

// The claimer: the CTA's queue, then self items while a producer runs low, then the end entry.
// One thread.
__device__ void claim_items(const Meta& m, Bars* bars, const int32_t* __restrict__ anchors,
                            const int32_t* __restrict__ item_id, const int32_t* __restrict__ queue_off,
                            const int32_t* __restrict__ queue_items, int32_t* pool,
                            int32_t* status, volatile int* abort_flag) {
    const int32_t q0 = queue_off[blockIdx.x], q1 = queue_off[blockIdx.x + 1];
    volatile int32_t* rr = bars->ring_r;
    int32_t tiles[2] = {0, 0};
    int32_t w = 0;
    bool ok = true;
    // Wait until slot w is free (every reader is past entry w - kRing) and, if ahead > 0, until one of
    // the producers has fewer than `ahead` entries left to read (pool items are claimed when needed).
    auto wait_room = [&](int ahead) -> bool {
        const uint64_t t0 = globaltimer();
        for (uint32_t spin = 0;; ++spin) {
            int32_t lo = rr[0];
            for (int x = 1; x < kReaders; ++x) lo = min(lo, rr[x]);
            const bool room = lo > w - kRing;
            const bool low = ahead <= 0 || max(rr[0], rr[1]) > w - ahead;  // a producer is running low
            if (room && low) return true;
            if ((spin & 63u) == 63u && (*abort_flag || globaltimer() - t0 > kTimeoutNs)) {
                *abort_flag = 1;
                return false;
            }
            __nanosleep(64);
        }
    };
    auto put = [&](int32_t id, int lane, int32_t nvis) {
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
        ((volatile int32_t*)bars->ring_lane)[e] = lane;
        ((volatile int32_t*)bars->ring_nvis)[e] = nvis;
        ((volatile int32_t*)bars->ring_j)[e] = j;
        ((volatile int32_t*)bars->ring_c)[e] = c;
        ((volatile int32_t*)bars->ring_sgn)[e] = sgn;
        __threadfence_block();
        ++w;
        ((volatile int32_t*)&bars->ring_w)[0] = w;
    };
    // Emits queue entry `pos` (if the item is visible) or a self item; ahead as in wait_room.
    auto emit = [&](int32_t id, int32_t nvis, int ahead) -> bool {
        if (nvis <= 0) return true;
        if (!wait_room(ahead)) return false;
        const int lane = tiles[0] <= tiles[1] ? 0 : 1;
        tiles[lane] += (nvis + kKeysPerTile - 1) / kKeysPerTile;
        put(id, lane, nvis);
        return true;
    };
    auto queue_entry = [&](int32_t pos, int ahead) -> bool {
        const int32_t id = __ldg(item_id + __ldg(queue_items + pos));
        if (id < 0 || id >= m.n_items) {
            raise_status(status, SPLITKV_DEV_BAD_PLAN);
            return true;
        }
        const Item it = decode_item(m, id);
        return emit(id, visible_in_chunk(m, it.s, it.c, __ldg(anchors + it.j + it.nbt - 1)), ahead);
    };
    for (int32_t pos = q0; ok && pos < q1; ++pos) ok = queue_entry(pos, 0);
    const int64_t n_self = m.n_blocks * m.hkv;
    while (ok) {
        // Claim when a producer has fewer than 2 entries left to read.
        if (!wait_room(2)) {
            ok = false;
            break;
        }
        const int64_t p = atomicAdd(pool, 1);
        if (p >= n_self) break;
        ok = emit((int32_t)(m.n_items + p), m.block, 0);
    }
    if (ok && wait_room(0)) put(kRingEnd, 0, 0);
}

__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ Meta m, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
                  const int32_t* __restrict__ anchors, const int32_t* __restrict__ item_id,
                  const int32_t* __restrict__ queue_off, const int32_t* __restrict__ queue_items,
                  __nv_bfloat16* __restrict__ o_part, float* __restrict__ lse_part, int32_t* __restrict__ pool,
                  int32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* stat = reinterpret_cast<float*>(smem + kOffStat);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
            mbar_init(&bars->k_full[b], 1);
            mbar_init(&bars->k_empty[b], 1);
            mbar_init(&bars->v_full[b], 1);
            mbar_init(&bars->v_empty[b], 1);
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->p_full[b], kWgThreads);
            mbar_init(&bars->o_ready[b], 1);
            mbar_init(&bars->o_free[b][0], kWgThreads);
            mbar_init(&bars->o_free[b][1], kWgThreads);
            mbar_init(&bars->stat_full[b][0], kWgThreads);
            mbar_init(&bars->stat_full[b][1], kWgThreads);
            mbar_init(&bars->drain[b], 1);
        }
        for (int q = 0; q < 4; ++q) bars->exp_slot[q] = 0;
        bars->ring_w = 0;
        for (int x = 0; x < kReaders; ++x) bars->ring_r[x] = 0;
        bars->abort_flag = 0;
        bars->status0 = status_bad(status) ? 1 : 0;
        fence_barrier_init();
    }
    // Rows of the Q buffers beyond block*G are never loaded: keep them finite (zero).
    for (int i = threadIdx.x; i < 2 * kTileBytes / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem + kOffQ)[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == kMmaWarp0) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const bool skip = bars->status0 != 0;  // every CTA may take pool items
    const int G = m.group, R = m.rows_item;

    if (warp >= kLoadWarp0) {
        // ------------------------------------------------------------ control warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kControlRegs));
        if (!skip && (warp == kLoadWarp0 || warp == kLoadWarp1) && lane == 0) {
            // Lane L: Q of item k, then K(n) and V(n) for each of its key tiles.
            const int L = warp == kLoadWarp0 ? 0 : 1;
            tma_prefetch_desc(L ? &tmK : &tmQ);
            tma_prefetch_desc(L ? &tmKb : &tmV);
            const uint32_t q_bytes = 2u * 64u * (uint32_t)G * (uint32_t)(m.block * m.pack) * 2u;
            uint8_t* qdst = smem + kOffQ + L * kTileBytes;
            uint8_t* kdst = smem + kOffK + L * kTileBytes;
            uint8_t* vdst = smem + kOffV + L * kTileBytes;
            int32_t ridx = 0;
            int rlane;
            TileRef t;
            uint32_t k = 0, n = 0;
            uint32_t inflight = 0;  // 1: Q(k-1), 2: K(n-1), 4: V(n-1) may still be landing
            bool ok = true;
            while (ok && ring_next(m, bars, ridx, L, L, true, false, t, &rlane, abort_flag) == 1) {
                if (k >= 1 && !mbar_wait(&bars->q_empty[L], (k - 1) & 1u, abort_flag, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars->q_full[L], q_bytes);
                tma_load_3d(qdst, &tmQ, &bars->q_full[L], 0, t.g * G, m.block * t.j);
                tma_load_3d(qdst + kHalfBytes, &tmQ, &bars->q_full[L], 64, t.g * G, m.block * t.j);
                ++k;
                inflight = 1;
                const CUtensorMap* mk = t.self_item ? &tmKb : &tmK;
                const CUtensorMap* mv = t.self_item ? &tmVb : &tmV;
                for (int32_t tt = 0; tt < t.ntiles; ++tt, ++n) {
                    const uint32_t ph = (n & 1u) ^ 1u;
                    const int32_t row = t.self_item ? m.block * t.j
                                                    : (int32_t)(m.key_off[t.s] + (int64_t)t.c * m.chunk +
                                                                (int64_t)tt * kKeysPerTile);
                    if (!mbar_wait(&bars->k_empty[L], ph, abort_flag, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->k_full[L], kTileBytes);
                    tma_load_3d(kdst, mk, &bars->k_full[L], 0, t.g, row);
                    tma_load_3d(kdst + kHalfBytes, mk, &bars->k_full[L], 64, t.g, row);
                    inflight = 3;
                    if (!mbar_wait(&bars->v_empty[L], ph, abort_flag, kTimeoutNs)) {
                        ++n;
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->v_full[L], kTileBytes);
                    tma_load_3d(vdst, mv, &bars->v_full[L], 0, t.g, row);
                    tma_load_3d(vdst + kHalfBytes, mv, &bars->v_full[L], 64, t.g, row);
                    inflight = 7;
                }
            }
            if (!ok) *abort_flag = 1;
            // Drain: the most recent copy into each buffer has landed before the CTA exits.
            volatile int never = 0;
            if (k > 0) mbar_wait(&bars->q_full[L], (k - 1) & 1u, &never, kTimeoutNs);
            if (n > 0 && (inflight & 2)) mbar_wait(&bars->k_full[L], (n - 1) & 1u, &never, kTimeoutNs);
            if (n > 0 && (inflight & 4)) mbar_wait(&bars->v_full[L], (n - 1) & 1u, &never, kTimeoutNs);
        } else if (!skip && warp == kLoadWarp0 && lane == 1) {
            claim_items(m, bars, anchors, item_id, queue_off, queue_items, pool, status, abort_flag);
        } else if (!skip && (warp == kMmaWarp0 || warp == kMmaWarp1) && lane == 0) {
            // Issuer L: QK(n) -> wait P(n) -> PV(n) -> QK(n+1) -> ...
            const int L = warp == kMmaWarp0 ? 0 : 1;
            constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, 128, false, true);
            // Descriptor bases; a K step only adds a constant to the (16-byte unit) start address.
            const uint64_t dq = umma_desc_sw128(smem_u32(smem + kOffQ + L * kTileBytes), 16, 1024);
            const uint64_t dk = umma_desc_sw128(smem_u32(smem + kOffK + L * kTileBytes), 16, 1024);
            const uint64_t dv = umma_desc_sw128(smem_u32(smem + kOffV + L * kTileBytes), kHalfBytes, 1024);
            const uint32_t ts = tmem + kColS + 128u * L, to = tmem + kColO + 128u * L;
            int32_t ridx = 0;
            int rlane;
            TileRef t;
            uint32_t k = 0, n = 0;
            bool ok = true;
            while (ok && ring_next(m, bars, ridx, 2 + L, L, true, false, t, &rlane, abort_flag) == 1) {
                if (!mbar_wait(&bars->q_full[L], k & 1u, abort_flag, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                for (int32_t tt = 0; tt < t.ntiles; ++tt, ++n) {
                    const uint32_t ph = n & 1u;
                    if (!mbar_wait(&bars->k_full[L], ph, abort_flag, kTimeoutNs)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t off = (uint64_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) / 16);
                        mma_ss(ts, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&bars->s_full[L]);
                    mma_commit(&bars->k_empty[L]);
                    if (tt == t.ntiles - 1) mma_commit(&bars->q_empty[L]);
                    if (!mbar_wait(&bars->p_full[L], ph, abort_flag, kTimeoutNs)) { ok = false; break; }
                    // The first PV of item k overwrites O_L once the epilogue has read item k-1.
                    if (tt == 0 && k >= 1 &&
                        !mbar_wait(&bars->o_free[L][(k - 1) & 1], ((k - 1) >> 1) & 1u, abort_flag, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&bars->v_full[L], ph, abort_flag, kTimeoutNs)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(to, ts + (uint32_t)(kk * 8), dv + (uint64_t)(kk * 2048 / 16), idesc_pv,
                               (tt > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&bars->v_empty[L]);
                    if (tt == t.ntiles - 1) mma_commit(&bars->o_ready[L]);
                }
                ++k;
            }
            if (!ok) *abort_flag = 1;
            // Drain: all MMAs issued by this thread complete before TMEM is released.
            mma_commit(&bars->drain[L]);
            volatile int never = 0;
            mbar_wait(&bars->drain[L], 0, &never, kTimeoutNs);
        }
        __syncwarp();
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------------ epilogue warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kEpilogueRegs));
        if (!skip) {
            // Each warp serves its 32 rows of both lanes, taking whichever lane has an item ready.
            const int quad = warp & 3;
            const int r = quad * 32 + lane;
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            // Per lane: 1 = holding its next item, 0 = none read yet, -1 = its sequence ended.
            int32_t idx0 = 0, idx1 = 0;
            int rlane;
            TileRef t0, t1;
            int has0 = 0, has1 = 0;
            uint32_t k0 = 0, k1 = 0;
            uint64_t deadline = globaltimer() + kTimeoutNs;
            bool ok = true;
            const int slot0 = 12 + 2 * quad;
            while (has0 >= 0 || has1 >= 0) {
                if (has0 == 0)
                    has0 = __shfl_sync(0xffffffffu,
                                       ring_next(m, bars, idx0, slot0, 0, false, true, t0, &rlane, abort_flag), 0);
                if (has1 == 0)
                    has1 = __shfl_sync(0xffffffffu,
                                       ring_next(m, bars, idx1, slot0 + 1, 1, false, true, t1, &rlane, abort_flag), 0);
                if (*abort_flag) {
                    ok = false;
                    break;
                }
                int pick = -1;
                if (has0 == 1 && mbar_try_wait(&bars->stat_full[0][k0 & 1], (k0 >> 1) & 1u) &&
                    mbar_try_wait(&bars->o_ready[0], k0 & 1u))
                    pick = 0;
                else if (has1 == 1 && mbar_try_wait(&bars->stat_full[1][k1 & 1], (k1 >> 1) & 1u) &&
                         mbar_try_wait(&bars->o_ready[1], k1 & 1u))
                    pick = 1;
                pick = __shfl_sync(0xffffffffu, pick, 0);
                if (pick < 0) {
                    if (*abort_flag || globaltimer() > deadline) {
                        ok = false;
                        break;
                    }
                    continue;
                }
                const uint32_t k = pick ? k1 : k0;
                // Lane 0 saw both phases complete; every thread observes them too (acquire), at once.
                mbar_wait(&bars->stat_full[pick][k & 1], (k >> 1) & 1u, abort_flag, kTimeoutNs);
                mbar_wait(&bars->o_ready[pick], k & 1u, abort_flag, kTimeoutNs);
                tc_fence_after();
                const TileRef& t = pick ? t1 : t0;
                const float* sp = stat + (pick * 2 + (int)(k & 1)) * 256;
                const float m_l = sp[r], l = sp[128 + r];
                const float inv = l > 0.f ? 1.f / l : 0.f;  // a row that sees no key: O = 0, LSE = -inf
                __nv_bfloat16* op = o_part + t.id * (int64_t)R * 128;  // [d/8][R][8] bf16
                const uint32_t to = tmem + kColO + 128u * pick + lane_off;
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    uint32_t ov[16];
                    tmem_ld16(to + cc * 16, ov);
                    tmem_wait_ld();
                    if (cc == 7) {  // O_L fully read: issuer L may start the lane's next item in it
                        tc_fence_before();
                        mbar_arrive(&bars->o_free[pick][k & 1]);
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
                if (r < R) lse_part[t.id * R + r] = l > 0.f ? (m_l + lg2_approx(l)) * 0.6931471805599453f : -INFINITY;
                if (pick) {
                    ++k1;
                    has1 = 0;
                } else {
                    ++k0;
                    has0 = 0;
                }
                deadline = globaltimer() + kTimeoutNs;
            }
            if (!ok) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
        if (!skip) {
            const int L = warp >> 2;                // lane
            const int quad = warp & 3;              // TMEM lane quadrant
            const int r = quad * 32 + lane;         // query-tile row
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const uint32_t ts = tmem + kColS + 128u * L + lane_off;  // S_L / P_L, this row
            const uint32_t to = tmem + kColO + 128u * L + lane_off;  // O_L, this row
            const float c = m.scale * 1.4426950408889634f;  // log2(e)
            const uint64_t c2 = f2_pack(c, c);
            uint32_t k = 0, n = 0;
            bool ok = true;
            int32_t ridx = 0;
            int rlane;
            TileRef t;
            while (ok && ring_next(m, bars, ridx, 4 + warp, L, true, true, t, &rlane, abort_flag) == 1) {
                float m_l = -INFINITY, l = 0.f;  // reference max and row sum (relative to m_l)
                // Keys of the chunk this row sees: its own block's prefix (a row of no block of the tile,
                // or of a self item beyond the block's own rows, sees none). A row's keys lie in the
                // item's first tiles, so a row that sees nothing in tile 0 sees nothing at all.
                int32_t row_nvis = 0;
                {
                    const int32_t x = r / m.rows;
                    if (t.self_item) row_nvis = x == 0 ? m.block : 0;
                    else if (x < t.nbt) row_nvis = visible_in_chunk(m, t.s, t.c, __ldg(anchors + t.j + x));
                }
                for (int32_t tt = 0; tt < t.ntiles; ++tt, ++n) {
                    // The whole warp leaves together on a timeout: the TMEM accesses below are collective.
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[L], n & 1u, abort_flag, kTimeoutNs))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int valid = row_nvis - tt * kKeysPerTile;  // keys of the tile this row sees
                    // Pass 1: row max over the visible keys, 64 columns per TMEM wait. tcgen05.ld/st are
                    // warp-collective, so the rescale below is decided by a warp vote (rows that do not
                    // move scale by 1).
                    uint32_t ra[32], rb[32];
                    float mx = -INFINITY;
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        load_half(ts, h, valid, ra, rb);
                        mx = fmaxf(mx, max_half(ra, rb));
                    }
                    mx *= c;
                    if (tt == 0) {
                        m_l = mx;
                    } else {
                        const bool move = mx > m_l + kRescaleLog2;
                        if (__any_sync(0xffffffffu, move)) {
                            // The max moved: rescale O_L (PV of the previous tile is complete) and the sum.
                            const float alpha = move ? ex2_approx(m_l - mx) : 1.f;
                            rescale_o(to, alpha);
                            l *= alpha;
                            if (move) m_l = mx;
                        }
                    }
                    // Pass 2: P = 2^(s*c - m) as bf16 pairs over the first 64 columns of S_L (keys 2u, 2u+1
                    // -> column u). Half h reads S columns 64h.. and writes P columns 32h.., which it has
                    // already read.
                    if (!exp_slot_take(&bars->exp_slot[quad], abort_flag, kTimeoutNs)) {
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    const float m_use = m_l == -INFINITY ? 0.f : m_l;  // fully masked row: P = 2^-inf = 0
                    const uint64_t negm2 = f2_pack(-m_use, -m_use);
                    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        load_half(ts, h, valid, ra, rb);
                        uint32_t pk[32];
                        exp_half(ra, rb, c2, negm2, acc, pk);
                        tmem_st32(ts + h * 32, pk);
                    }
                    exp_slot_give(&bars->exp_slot[quad]);
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
                    mbar_arrive(&bars->p_full[L]);
                }
                if (!ok) break;
                // Hand (m, l) of item k to the epilogue; stat[L][k % 2] was last read for item k-2.
                if (k >= 2 && !mbar_wait(&bars->o_free[L][k & 1], ((k >> 1) - 1) & 1u, abort_flag, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                float* sp = stat + (L * 2 + (int)(k & 1)) * 256;
                sp[r] = m_l;
                sp[128 + r] = l;
                mbar_arrive(&bars->stat_full[L][k & 1]);
                ++k;
            }
            if (!ok) *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && bars->abort_flag) raise_status(status, SPLITKV_DEV_TIMEOUT);
    if (warp == kMmaWarp0) {
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
                          int32_t* status, void* ws, cudaStream_t st) {
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
    fwd_tc_kernel<<<n_workers, kThreads, kSmemBytes, st>>>(m, tq, tk, tv, tkb, tvb, anchors, item_id, queue_off,
                                                           queue_items, (__nv_bfloat16*)o_part, lse_part, pool, status);
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
