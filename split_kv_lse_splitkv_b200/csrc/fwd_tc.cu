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
// Roles (512 threads, four warpgroups; registers moved with setmaxnreg):
//   WG0 / WG1 (warps 0-7)  softmax of the even / odd key tiles: row r = 32*(warp%4) + lane
//   WG2 (warps 8-11)       epilogue: normalises O of a finished item and stores O_c, LSE_c
//   warp 12                TMA producer: Q per item (2 buffers), K(n) and V(n) (2 buffers each)
//   warp 13                QK^T issuer (one thread) and TMEM owner
//   warp 14                PV issuer (one thread)
//
// TMEM (all 512 columns): S[2] = Q K^T (128 fp32 columns each, tile n in S[n % 2]), P[2] (bf16
// pairs, 64 columns each) and O (128 fp32 columns). A thread issuing tcgen05.mma waits while the
// tensor core works through its previous instruction, and back-to-back MMAs into one accumulator
// wait on each other; two threads issuing independent chains at the same moment keep the tensor
// core busy. So both issuers start on the same event: when P(n) is written, one issues PV(n) and
// the other QK^T(n+2) (S[n % 2] is free: the softmax of tile n has finished with it). The two
// softmax warpgroups work on consecutive tiles at the same time, so one evaluates exponentials
// while the other loads and reduces, and the epilogue warpgroup drains O while the next item's
// scores are computed. The issuers only commit S-ready and PV-done; the softmax threads release
// the K, V and Q buffers once those commits say the reads are over.
//
// Online softmax in log2 units (x = s * scale * log2 e). The running reference max m of a row only
// moves when a tile's max exceeds it by more than 8 (so P <= 256); tile n publishes its m to tile
// n+1 through shared memory, and a move rescales O (after PV(n-1)) and the row sums. Each
// warpgroup sums P over its own tiles, relative to its latest m; the epilogue combines the two sums.
// LSE = (m + log2 l) * ln 2.
//
// Every wait is bounded (2 s); on expiry the CTA raises SPLITKV_DEV_TIMEOUT, drains its copies and
// MMAs in flight, frees TMEM and returns.
#include <cstdio>

#include "common.cuh"
#include "sm100.cuh"

namespace splitkv {

namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int kEpiWarp0 = 8;
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;  // QK^T issuer, TMEM owner
constexpr int kPvWarp = 14;
constexpr int kSoftmaxRegs = 152;  // per SM sub-partition: 152 + 152 + 104 + 96 = 504 <= 4 x 128 launched
constexpr int kEpilogueRegs = 104;
constexpr int kControlRegs = 96;
constexpr int kTileBytes = 32768;    // 128 x 128 bf16, as two 128-byte-wide halves
constexpr int kHalfBytes = 16384;
constexpr int kKeysPerTile = 128;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kWgThreads = 128;

constexpr uint32_t kColS0 = 0, kColP0 = 256, kColO = 384;  // S[b] at 128 b, P[b] at 256 + 64 b

constexpr int kOffQ = 0;                                  // Q[2]
constexpr int kOffK = 2 * kTileBytes;                     // K[2]
constexpr int kOffV = 4 * kTileBytes;                     // V[2]
constexpr int kOffMdec = 6 * kTileBytes;                  // float [2][128]: reference max of tile n (n % 2)
constexpr int kOffStat = kOffMdec + 2 * 128 * 4;          // float [2][2][2][128]: item parity, wg, (m, l)
constexpr int kOffBar = kOffStat + 2 * 2 * 2 * 128 * 4;

struct Bars {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2];     // QK^T(n) complete, by n % 2
    uint64_t p_full[2];     // P(n) written, by n % 2
    uint64_t pv_done[2];    // PV(n) complete, by n % 2
    uint64_t mdec[2];       // reference max of tile n published, by n % 2
    uint64_t stat_full[2];  // m and l of item i written (by item parity)
    uint64_t o_ready[2];    // last PV of item i complete (by item parity)
    uint64_t o_free[2];     // epilogue has read O for item i (by item parity)
    uint64_t drain[2];      // all MMAs of the QK^T / PV issuer complete
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

constexpr int kSmemBytes = kOffBar + (int)sizeof(Bars) + 1024;  // + alignment slack

struct TileRef {
    int64_t id;                // partial slot: item id, or n_items + j*Hkv + g for a self item
    int32_t s, c, g, j;
    int32_t nvis, ntiles, t;
    int32_t self_item;         // 1: keys are the block's own (Kb/Vb rows block*j ..)
};

// The CTA's items (queue positions first, first+1, ...), fetched ahead: each call hands out the
// next (item id, anchor) and issues the loads one link further for the three items after it
// (anchor of n+1, id of n+2, queue entry of n+3), so no role waits on a dependent global load
// chain when it moves to a new item.
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
    return (id >= 0 && id < m.n_items) ? __ldg(anchors + decode_item(m, id).j) : 0;
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
    tr.t = 0;
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
    tr.nvis = visible_in_chunk(m, it.s, it.c, a);
    tr.ntiles = (tr.nvis + kKeysPerTile - 1) / kKeysPerTile;
    tr.t = 0;
}

// The CTA's items as one sequence of key tiles.
struct Cursor {
    ItemStream st;
    bool has;
    TileRef cur;
};

__device__ __forceinline__ void cursor_fetch(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                             const int32_t* queue_items, Cursor& c, int32_t* status) {
    while (stream_more(c.st)) {
        stream_next(m, anchors, item_id, queue_items, c.st, c.cur, status);
        if (c.cur.ntiles > 0) {
            c.has = true;
            return;
        }
    }
    c.has = false;
}

__device__ __forceinline__ void cursor_init(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                            const int32_t* queue_items, int32_t first, int32_t end, Cursor& c,
                                            int32_t* status) {
    stream_init(m, anchors, item_id, queue_items, first, end, c.st);
    cursor_fetch(m, anchors, item_id, queue_items, c, status);
}

__device__ __forceinline__ void cursor_advance(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                               const int32_t* queue_items, Cursor& c, int32_t* status) {
    if (++c.cur.t < c.cur.ntiles) return;
    cursor_fetch(m, anchors, item_id, queue_items, c, status);
}

__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ Meta m, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
                  const int32_t* __restrict__ anchors, const int32_t* __restrict__ item_id,
                  const int32_t* __restrict__ queue_off, const int32_t* __restrict__ queue_items,
                  float* __restrict__ o_part, float* __restrict__ lse_part, int32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* mdec = reinterpret_cast<float*>(smem + kOffMdec);
    float* stat = reinterpret_cast<float*>(smem + kOffStat);
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t q0 = queue_off[blockIdx.x], q1 = queue_off[blockIdx.x + 1];

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
            mbar_init(&bars->pv_done[b], 1);
            mbar_init(&bars->mdec[b], kWgThreads);
            mbar_init(&bars->stat_full[b], 2 * kWgThreads);
            mbar_init(&bars->o_ready[b], 1);
            mbar_init(&bars->o_free[b], kWgThreads);
        }
        mbar_init(&bars->drain[0], 1);
        mbar_init(&bars->drain[1], 1);
        bars->abort_flag = 0;
        bars->status0 = status_bad(status) ? 1 : 0;
        fence_barrier_init();
    }
    // Rows of the Q buffers beyond block*G are never loaded: keep them finite (zero).
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
    const bool skip = bars->status0 != 0 || (q0 >= q1 && (int64_t)blockIdx.x >= m.n_blocks * m.hkv);
    const int G = m.group, R = m.rows;

    if (warp >= kProducerWarp) {
        // ------------------------------------------------------------ control warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kControlRegs));
        if (!skip && warp == kProducerWarp && lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmKb);
            tma_prefetch_desc(&tmVb);
            const uint32_t q_bytes = 2u * 64u * (uint32_t)G * (uint32_t)m.block * 2u;
            Cursor cur;
            TileRef prev;
            uint32_t n = 0, item_seq = 0;
            bool ok = true;
            cursor_init(m, anchors, item_id, queue_items, q0, q1, cur, status);
            auto load_tile = [&](const CUtensorMap* map, uint64_t* full, uint64_t* empty, uint32_t idx, int off,
                                 const TileRef& t) -> bool {
                const int b = idx & 1;
                if (!mbar_wait(&empty[b], ((idx >> 1) & 1u) ^ 1u, abort_flag, kTimeoutNs)) return false;
                mbar_arrive_expect_tx(&full[b], kTileBytes);
                const int32_t row = t.self_item ? m.block * t.j
                                                : (int32_t)(m.key_off[t.s] + (int64_t)t.c * m.chunk +
                                                            (int64_t)t.t * kKeysPerTile);
                uint8_t* dst = smem + off + b * kTileBytes;
                tma_load_3d(dst, map, &full[b], 0, t.g, row);
                tma_load_3d(dst + kHalfBytes, map, &full[b], 64, t.g, row);
                return true;
            };
            // Order: Q (new item), K(n), V(n-1).
            while (ok && cur.has) {
                const TileRef t = cur.cur;
                if (t.t == 0) {
                    const int qb = item_seq & 1;
                    if (!mbar_wait(&bars->q_empty[qb], ((item_seq >> 1) & 1u) ^ 1u, abort_flag, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->q_full[qb], q_bytes);
                    uint8_t* dst = smem + kOffQ + qb * kTileBytes;
                    tma_load_3d(dst, &tmQ, &bars->q_full[qb], 0, t.g * G, m.block * t.j);
                    tma_load_3d(dst + kHalfBytes, &tmQ, &bars->q_full[qb], 64, t.g * G, m.block * t.j);
                    ++item_seq;
                }
                ok = load_tile(t.self_item ? &tmKb : &tmK, bars->k_full, bars->k_empty, n, kOffK, t);
                if (ok && n > 0)
                    ok = load_tile(prev.self_item ? &tmVb : &tmV, bars->v_full, bars->v_empty, n - 1, kOffV, prev);
                if (!ok) break;
                prev = t;
                ++n;
                cursor_advance(m, anchors, item_id, queue_items, cur, status);
            }
            if (ok && n > 0)
                ok = load_tile(prev.self_item ? &tmVb : &tmV, bars->v_full, bars->v_empty, n - 1, kOffV, prev);
            // Drain: the most recent copy into every buffer has landed before the CTA exits.
            volatile int never = 0;
            for (uint32_t x = (n > 2 ? n - 2 : 0); x < n; ++x) {
                mbar_wait(&bars->k_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
                mbar_wait(&bars->v_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
            }
            for (uint32_t x = (item_seq > 2 ? item_seq - 2 : 0); x < item_seq; ++x)
                mbar_wait(&bars->q_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
        } else if (!skip && warp == kMmaWarp && lane == 0) {
            // QK^T(0), QK^T(1) at once; QK^T(n) for n >= 2 when P(n-2) is written.
            constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(128, 128, false, false);
            // Descriptor bases; a K step only adds a constant to the (16-byte unit) start address.
            uint64_t dq[2], dk[2];
            for (int b = 0; b < 2; ++b) {
                dq[b] = umma_desc_sw128(smem_u32(smem + kOffQ + b * kTileBytes), 16, 1024);
                dk[b] = umma_desc_sw128(smem_u32(smem + kOffK + b * kTileBytes), 16, 1024);
            }
            Cursor cur;
            uint32_t n = 0, item_seq = 0, qb = 0;
            cursor_init(m, anchors, item_id, queue_items, q0, q1, cur, status);
            while (cur.has) {
                const TileRef t = cur.cur;
                const int sb = n & 1;
                if (n >= 2 && !mbar_wait(&bars->p_full[sb], ((n >> 1) - 1) & 1u, abort_flag, kTimeoutNs)) break;
                if (t.t == 0) {
                    qb = item_seq & 1;
                    if (!mbar_wait(&bars->q_full[qb], (item_seq >> 1) & 1u, abort_flag, kTimeoutNs)) break;
                    ++item_seq;
                }
                if (!mbar_wait(&bars->k_full[sb], (n >> 1) & 1u, abort_flag, kTimeoutNs)) break;
                tc_fence_after();
                const uint32_t ts = tmem + kColS0 + 128u * sb;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) / 16);
                    mma_ss(ts, dq[qb] + off, dk[sb] + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[sb]);
                ++n;
                cursor_advance(m, anchors, item_id, queue_items, cur, status);
            }
            // Drain: all MMAs issued by this thread complete before TMEM is released.
            mma_commit(&bars->drain[0]);
            volatile int never = 0;
            mbar_wait(&bars->drain[0], 0, &never, kTimeoutNs);
        } else if (!skip && warp == kPvWarp && lane == 0) {
            // PV(n): O (+)= P(n) V(n), A = P[n % 2] from TMEM (bf16 pairs), B = V, MN-major. The first
            // PV of item i overwrites O once the epilogue of item i-1 has read it.
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, 128, false, true);
            uint64_t dv[2];
            for (int b = 0; b < 2; ++b)
                dv[b] = umma_desc_sw128(smem_u32(smem + kOffV + b * kTileBytes), kHalfBytes, 1024);
            const uint32_t to = tmem + kColO;
            Cursor cur;
            uint32_t n = 0, item = 0;
            cursor_init(m, anchors, item_id, queue_items, q0, q1, cur, status);
            while (cur.has) {
                const TileRef t = cur.cur;
                const bool first = t.t == 0, last = t.t == t.ntiles - 1;
                const int sb = n & 1;
                if (!mbar_wait(&bars->p_full[sb], (n >> 1) & 1u, abort_flag, kTimeoutNs)) break;
                if (first && item >= 1 &&
                    !mbar_wait(&bars->o_free[(item - 1) & 1], ((item - 1) >> 1) & 1u, abort_flag, kTimeoutNs))
                    break;
                if (!mbar_wait(&bars->v_full[sb], (n >> 1) & 1u, abort_flag, kTimeoutNs)) break;
                tc_fence_after();
                const uint32_t tp = tmem + kColP0 + 64u * sb;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(to, tp + (uint32_t)(kk * 8), dv[sb] + (uint64_t)(kk * 2048 / 16), idesc_pv,
                           (!first || kk > 0) ? 1u : 0u);
                mma_commit(&bars->pv_done[sb]);
                if (last) {
                    mma_commit(&bars->o_ready[item & 1]);
                    ++item;
                }
                ++n;
                cursor_advance(m, anchors, item_id, queue_items, cur, status);
            }
            mma_commit(&bars->drain[1]);
            volatile int never = 0;
            mbar_wait(&bars->drain[1], 0, &never, kTimeoutNs);
        }
        __syncwarp();
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------------ epilogue warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kEpilogueRegs));
        if (!skip) {
            const int quad = warp & 3;
            const int r = quad * 32 + lane;
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            uint32_t i = 0;
            ItemStream st;
            stream_init(m, anchors, item_id, queue_items, q0, q1, st);
            while (stream_more(st)) {
                TileRef t;
                stream_next(m, anchors, item_id, queue_items, st, t, status);
                if (t.ntiles == 0) continue;
                const int ob = i & 1;
                if (!mbar_wait(&bars->stat_full[ob], (i >> 1) & 1u, abort_flag, kTimeoutNs)) break;
                if (!mbar_wait(&bars->o_ready[ob], (i >> 1) & 1u, abort_flag, kTimeoutNs)) break;
                tc_fence_after();
                // Both warpgroups' sums, moved to the final reference max (the larger m: m only grows).
                const float* sp = stat + ob * 512;
                const float m0 = sp[r], l0 = sp[128 + r], m1 = sp[256 + r], l1 = sp[384 + r];
                const float m_fin = fmaxf(m0, m1);
                const float l_row = (l0 > 0.f ? l0 * ex2_approx(m0 - m_fin) : 0.f) +
                                    (l1 > 0.f ? l1 * ex2_approx(m1 - m_fin) : 0.f);
                const float inv_l = 1.f / l_row;
                float* op = o_part + t.id * (int64_t)R * 128;
                const uint32_t to = tmem + kColO + lane_off;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t ov[32];
                    tmem_ld32(to + cc * 32, ov);
                    tmem_wait_ld();
                    if (cc == 3) {  // O fully read: the issuer may start item i+1 in it
                        tc_fence_before();
                        mbar_arrive(&bars->o_free[ob]);
                    }
                    if (r < R) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            float4 x = make_float4(__uint_as_float(ov[4 * u]) * inv_l,
                                                   __uint_as_float(ov[4 * u + 1]) * inv_l,
                                                   __uint_as_float(ov[4 * u + 2]) * inv_l,
                                                   __uint_as_float(ov[4 * u + 3]) * inv_l);
                            *reinterpret_cast<float4*>(op + ((int64_t)(cc * 8 + u) * R + r) * 4) = x;
                        }
                    }
                }
                if (r < R) lse_part[t.id * R + r] = (m_fin + lg2_approx(l_row)) * 0.6931471805599453f;
                ++i;
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
        if (!skip) {
            const int wg = warp >> 2;               // this warpgroup takes the tiles n with n % 2 == wg
            const int quad = warp & 3;              // TMEM lane quadrant
            const int r = quad * 32 + lane;         // query-tile row
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const uint32_t ts = tmem + kColS0 + 128u * wg + lane_off;  // S[wg], this row
            const uint32_t tp = tmem + kColP0 + 64u * wg + lane_off;   // P[wg], this row
            const float c = m.scale * 1.4426950408889634f;  // log2(e)
            const uint64_t c2 = f2_pack(c, c);
            const bool leader = (threadIdx.x & (kWgThreads - 1)) == 0;
            uint32_t n = 0, i = 0;
            bool ok = true;
            ItemStream st;
            stream_init(m, anchors, item_id, queue_items, q0, q1, st);
            while (stream_more(st) && ok) {
                TileRef t;
                stream_next(m, anchors, item_id, queue_items, st, t, status);
                if (t.ntiles == 0) continue;
                const int ob = i & 1;
                const uint32_t to = tmem + kColO + lane_off;
                float m_l = -INFINITY, l = 0.f;  // this warpgroup's row sum, relative to m_l
                for (int tt = 0; tt < t.ntiles; ++tt, ++n) {
                    if ((int)(n & 1) != wg) continue;
                    if (!mbar_wait(&bars->s_full[wg], (n >> 1) & 1u, abort_flag, kTimeoutNs)) { ok = false; break; }
                    tc_fence_after();
                    if (leader) {  // QK^T(n) complete: K(n) is free, and Q after the item's last tile
                        mbar_arrive(&bars->k_empty[wg]);
                        if (tt == t.ntiles - 1) mbar_arrive(&bars->q_empty[i & 1]);
                    }
                    const int valid = t.nvis - tt * kKeysPerTile;  // keys of this tile the block sees (>= 1)
                    // Pass 1: row max over the visible keys, 64 columns per TMEM wait.
                    float mx;
                    {
                        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll 1
                        for (int h = 0; h < 2; ++h) {
                            uint32_t ra[32], rb[32];
                            tmem_ld32(ts + h * 64, ra);
                            tmem_ld32(ts + h * 64 + 32, rb);
                            tmem_wait_ld();
                            if (valid >= kKeysPerTile) {
#pragma unroll
                                for (int u = 0; u < 32; u += 4) {
                                    m0 = max3f(m0, __uint_as_float(ra[u]), __uint_as_float(ra[u + 1]));
                                    m1 = max3f(m1, __uint_as_float(ra[u + 2]), __uint_as_float(ra[u + 3]));
                                    m2 = max3f(m2, __uint_as_float(rb[u]), __uint_as_float(rb[u + 1]));
                                    m3 = max3f(m3, __uint_as_float(rb[u + 2]), __uint_as_float(rb[u + 3]));
                                }
                            } else {
#pragma unroll
                                for (int u = 0; u < 32; ++u) {
                                    if (h * 64 + u < valid) m0 = fmaxf(m0, __uint_as_float(ra[u]));
                                    if (h * 64 + 32 + u < valid) m1 = fmaxf(m1, __uint_as_float(rb[u]));
                                }
                            }
                        }
                        mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * c;
                    }
                    // Reference max: tile n-1 publishes its m to tile n (every tile waits, which also
                    // keeps a warpgroup from overwriting a slot its partner has not read yet).
                    float m_prev = -INFINITY;
                    if (n > 0) {
                        if (!mbar_wait(&bars->mdec[(n - 1) & 1], ((n - 1) >> 1) & 1u, abort_flag, kTimeoutNs)) {
                            ok = false;
                            break;
                        }
                        if (tt > 0) m_prev = mdec[((n - 1) & 1) * 128 + r];
                    }
                    const float m_new = (tt == 0 || mx > m_prev + kRescaleLog2) ? mx : m_prev;
                    mdec[(n & 1) * 128 + r] = m_new;
                    mbar_arrive(&bars->mdec[n & 1]);
                    if (tt > 0 && m_new != m_prev) {
                        // The max moved: rescale this row of O once PV(n-1) has landed in it.
                        if (!mbar_wait(&bars->pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1u, abort_flag, kTimeoutNs)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const float alpha = ex2_approx(m_prev - m_new);
#pragma unroll 1
                        for (int cc = 0; cc < 4; ++cc) {
                            uint32_t ov[32];
                            tmem_ld32(to + cc * 32, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int u = 0; u < 32; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * alpha);
                            tmem_st32(to + cc * 32, ov);
                        }
                    }
                    if (m_l != m_new) {
                        l = (m_l == -INFINITY) ? 0.f : l * ex2_approx(m_l - m_new);
                        m_l = m_new;
                    }
                    // P[wg] was last read by PV(n-2); once that completed, V(n-2) is free as well.
                    if (n >= 2) {
                        if (!mbar_wait(&bars->pv_done[wg], ((n >> 1) - 1) & 1u, abort_flag, kTimeoutNs)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        if (leader) mbar_arrive(&bars->v_empty[wg]);
                    }
                    // Pass 2: P = 2^(s*c - m) in bf16 pairs into P[wg] (keys 64h.. -> columns 32h..).
                    const uint64_t negm2 = f2_pack(-m_new, -m_new);
                    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        uint32_t ra[32], rb[32];
                        tmem_ld32(ts + h * 64, ra);
                        tmem_ld32(ts + h * 64 + 32, rb);
                        tmem_wait_ld();
                        if (valid < kKeysPerTile) {
#pragma unroll
                            for (int u = 0; u < 32; ++u) {
                                if (h * 64 + u >= valid) ra[u] = __float_as_uint(-INFINITY);
                                if (h * 64 + 32 + u >= valid) rb[u] = __float_as_uint(-INFINITY);
                            }
                        }
                        uint32_t pk[32];
#pragma unroll
                        for (int u = 0; u < 32; ++u) {
                            const uint32_t* src = u < 16 ? ra : rb;
                            const int v = (u & 15) * 2;
                            float t0, t1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(src[v]), __uint_as_float(src[v + 1])), c2, negm2),
                                      t0, t1);
                            const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
                            acc[u & 3] = f2_add(acc[u & 3], f2_pack(p0, p1));
                            __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);  // .x (low half) = even key
                            pk[u] = *reinterpret_cast<uint32_t*>(&hp);
                        }
                        tmem_st32(tp + h * 32, pk);
                    }
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
                    mbar_arrive(&bars->p_full[wg]);
                }
                if (!ok) break;
                // Hand this warpgroup's (m, l) to the epilogue; stat[i % 2] was last read by the
                // epilogue of item i-2.
                if (i >= 2 && !mbar_wait(&bars->o_free[ob], ((i >> 1) - 1) & 1u, abort_flag, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                float* sp = stat + ob * 512 + wg * 256;
                sp[r] = m_l;
                sp[128 + r] = l;
                mbar_arrive(&bars->stat_full[ob]);
                ++i;
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

// 3-D bf16 map over [rows][heads][d] with a 128-byte swizzled box {64, box_heads, box_rows}.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int heads, int d, int box_heads, int box_rows) {
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

}  // namespace

bool fwd_tc_supported(const Meta& m) {
    return m.dtype == SPLITKV_BF16 && m.d == 128 && m.rows <= 128 && m.block <= 256 && m.group <= 256 &&
           m.total_keys < INT32_MAX && m.n_queries < INT32_MAX;
}

cudaError_t launch_fwd_tc(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                          const int32_t* anchors, const int32_t* item_id, const int32_t* queue_off,
                          const int32_t* queue_items, int32_t n_workers, float* o_part, float* lse_part,
                          int32_t* status, cudaStream_t st) {
    CUtensorMap tq, tk, tv, tkb, tvb;
    if (m.n_queries == 0 || m.total_keys == 0) return cudaSuccess;
    if (!make_map(&tq, q, m.n_queries, m.hq, m.d, m.group, m.block) ||
        !make_map(&tk, k, m.total_keys, m.hkv, m.d, 1, kKeysPerTile) ||
        !make_map(&tv, v, m.total_keys, m.hkv, m.d, 1, kKeysPerTile) ||
        !make_map(&tkb, kb, m.n_queries, m.hkv, m.d, 1, kKeysPerTile) ||
        !make_map(&tvb, vb, m.n_queries, m.hkv, m.d, 1, kKeysPerTile))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(fwd_tc_kernel, smem)");
    fwd_tc_kernel<<<n_workers, kThreads, kSmemBytes, st>>>(m, tq, tk, tv, tkb, tvb, anchors, item_id, queue_off,
                                                           queue_items, o_part, lse_part, status);
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
