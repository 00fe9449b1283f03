// Chunk-partial forward on the 5th-generation tensor cores (sm_100a): TMA -> tcgen05.mma -> TMEM.
//
// Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, Abstract: exact
// attention over context chunks, each producing a query-sized partial output and a per-row
// log-sum-exp; the chunks are placed by the cost-aware LPT plan. Here one persistent CTA per SM
// walks the SM's LPT queue. A work item (s, c, g, b) is one 128-row query tile — the block*G rows
// (query i, head g*G+hl) of block b at kv head g, shared by the G query heads of the GQA group —
// against the ceil(nvis/128) key tiles of chunk c that the block sees. The CTA's key tiles form
// one sequence n = 0, 1, ... across its items i = 0, 1, ...
//
// Roles (512 threads, four warpgroups; registers moved with setmaxnreg):
//   WG0 / WG1 (warps 0-7)  softmax: row r = 32*(warp%4) + lane, key columns 0-63 / 64-127
//   WG2 (warps 8-11)       epilogue: normalises O of a finished item and stores O_c, LSE_c
//   warp 12                TMA producer: Q per item (2 buffers), K(n) and V(n) (2 buffers each)
//   warp 13                MMA issuer (one thread) and TMEM owner
//
// TMEM (448 of 512 columns): S = Q K^T (128 fp32 columns), P (bf16 pairs, 64 columns) and
// O[2] (128 fp32 columns each, one per item parity). The MMA thread issues QK^T(n) and then
// PV(n-1): while the softmax turns S(n) into P(n), the tensor core runs PV(n-1) and, as soon as
// the softmax holds S(n) in registers, QK^T(n+1). No MMA waits for another MMA, and an item's
// epilogue overlaps the next item's tiles. The MMA thread only commits S-ready and PV-done; the
// softmax warps release the K, V and Q buffers once those commits tell them the reads are over.
//
// Online softmax in log2 units (x = s * scale * log2 e); the two halves of a row exchange their
// maxima through shared memory. The running reference max only moves when a tile's max exceeds it
// by more than 8 (so P <= 256), which keeps O and l consistent and rescales O rarely.
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
constexpr int kMmaWarp = 13;
constexpr int kSoftmaxRegs = 152;  // per SM sub-partition: 152 + 152 + 104 + 96 = 504 <= 4 x 128 launched
constexpr int kEpilogueRegs = 104;
constexpr int kControlRegs = 96;
constexpr int kTileBytes = 32768;    // 128 x 128 bf16, as two 128-byte-wide halves
constexpr int kHalfBytes = 16384;
constexpr int kKeysPerTile = 128;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kSoftmaxThreads = 256;
constexpr int kEpiThreads = 128;

constexpr uint32_t kColS = 0, kColP = 128, kColO0 = 256;  // O[b] at kColO0 + 128 b

constexpr int kOffQ = 0;                                  // Q[2]
constexpr int kOffK = 2 * kTileBytes;                     // K[2]
constexpr int kOffV = 4 * kTileBytes;                     // V[2]
constexpr int kOffRed = 6 * kTileBytes;                   // float [2][2][128]: row-max halves by tile parity
constexpr int kOffStat = kOffRed + 2 * 2 * 128 * 4;       // float [2][3][128]: m, l0, l1 by item parity
constexpr int kOffBar = kOffStat + 2 * 3 * 128 * 4;

struct Bars {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full, s_free;
    uint64_t p_full, pv_done;
    uint64_t red_bar[2];    // row-max halves of tile n written (by tile parity)
    uint64_t stat_full[2];  // m and l of item i written (by item parity)
    uint64_t o_ready[2];    // last PV of item i complete (by item parity)
    uint64_t o_free[2];     // epilogue has read O[i % 2]
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

constexpr int kSmemBytes = kOffBar + (int)sizeof(Bars) + 1024;  // + alignment slack

struct TileRef {
    int64_t id;
    int32_t s, c, g, j;
    int32_t nvis, ntiles, t;
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
}

// Next item as a tile reference (ntiles == 0 for an invalid entry, which raises BAD_PLAN).
__device__ __forceinline__ void stream_next(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                            const int32_t* queue_items, ItemStream& st, TileRef& tr, int32_t* status) {
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
    while (c.st.left > 0) {
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
                  const int32_t* __restrict__ anchors, const int32_t* __restrict__ item_id,
                  const int32_t* __restrict__ queue_off, const int32_t* __restrict__ queue_items,
                  float* __restrict__ o_part, float* __restrict__ lse_part, int32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* red = reinterpret_cast<float*>(smem + kOffRed);
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
            mbar_init(&bars->red_bar[b], kSoftmaxThreads);
            mbar_init(&bars->stat_full[b], kSoftmaxThreads);
            mbar_init(&bars->o_ready[b], 1);
            mbar_init(&bars->o_free[b], kEpiThreads);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, kSoftmaxThreads);
        mbar_init(&bars->p_full, kSoftmaxThreads);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->drain, 1);
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
    const bool skip = bars->status0 != 0 || q0 >= q1;
    const int G = m.group, R = m.rows;
    const uint32_t tS = tmem + kColS, tP = tmem + kColP;

    if (warp >= kProducerWarp) {
        // ------------------------------------------------------------ control warpgroup
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kControlRegs));
        if (!skip && warp == kProducerWarp && lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
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
                const int32_t row = (int32_t)(m.key_off[t.s] + (int64_t)t.c * m.chunk + (int64_t)t.t * kKeysPerTile);
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
                ok = load_tile(&tmK, bars->k_full, bars->k_empty, n, kOffK, t);
                if (ok && n > 0) ok = load_tile(&tmV, bars->v_full, bars->v_empty, n - 1, kOffV, prev);
                prev = t;
                ++n;
                cursor_advance(m, anchors, item_id, queue_items, cur, status);
            }
            if (ok && n > 0) ok = load_tile(&tmV, bars->v_full, bars->v_empty, n - 1, kOffV, prev);
            // Drain: the most recent copy into every buffer has landed before the CTA exits.
            volatile int never = 0;
            for (uint32_t x = (n > 2 ? n - 2 : 0); x < n; ++x) {
                mbar_wait(&bars->k_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
                mbar_wait(&bars->v_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
            }
            for (uint32_t x = (item_seq > 2 ? item_seq - 2 : 0); x < item_seq; ++x)
                mbar_wait(&bars->q_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
        } else if (!skip && warp == kMmaWarp && lane == 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, 128, false, true);
            // Descriptor bases; a K step only adds a constant to the (16-byte unit) start address.
            uint64_t dq[2], dk[2], dv[2];
            for (int b = 0; b < 2; ++b) {
                dq[b] = umma_desc_sw128(smem_u32(smem + kOffQ + b * kTileBytes), 16, 1024);
                dk[b] = umma_desc_sw128(smem_u32(smem + kOffK + b * kTileBytes), 16, 1024);
                dv[b] = umma_desc_sw128(smem_u32(smem + kOffV + b * kTileBytes), kHalfBytes, 1024);
            }
            Cursor cur;
            uint32_t n = 0, item_seq = 0, qb = 0, cur_item = 0;
            bool pending = false, pv_first = false, pv_last = false;
            uint32_t pv_n = 0, pv_item = 0;
            bool ok = true;
            cursor_init(m, anchors, item_id, queue_items, q0, q1, cur, status);
            auto issue_pv = [&]() -> bool {
                // PV(pv_n): O[item % 2] (+)= P V, A = P from TMEM (bf16 pairs), B = V, MN-major.
                if (!mbar_wait(&bars->p_full, pv_n & 1u, abort_flag, kTimeoutNs)) return false;
                const int ob = pv_item & 1;
                if (pv_first && pv_item >= 2 &&
                    !mbar_wait(&bars->o_free[ob], ((pv_item >> 1) - 1) & 1u, abort_flag, kTimeoutNs))
                    return false;
                const int vb = pv_n & 1;
                if (!mbar_wait(&bars->v_full[vb], (pv_n >> 1) & 1u, abort_flag, kTimeoutNs)) return false;
                tc_fence_after();
                const uint32_t to = tmem + kColO0 + 128u * ob;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(to, tP + (uint32_t)(kk * 8), dv[vb] + (uint64_t)(kk * 2048 / 16), idesc_pv,
                           (!pv_first || kk > 0) ? 1u : 0u);
                mma_commit(&bars->pv_done);
                if (pv_last) mma_commit(&bars->o_ready[ob]);
                return true;
            };
            while (ok && cur.has) {
                const TileRef t = cur.cur;
                // QK^T(n) into S: the softmax must hold S(n-1) in registers already.
                if (n >= 1 && !mbar_wait(&bars->s_free, (n - 1) & 1u, abort_flag, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                if (t.t == 0) {
                    qb = item_seq & 1;
                    if (!mbar_wait(&bars->q_full[qb], (item_seq >> 1) & 1u, abort_flag, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    cur_item = item_seq++;
                }
                const int kb = n & 1;
                if (!mbar_wait(&bars->k_full[kb], (n >> 1) & 1u, abort_flag, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) / 16);
                    mma_ss(tS, dq[qb] + off, dk[kb] + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full);
                // PV(n-1) once its P is ready.
                if (pending && !(ok = issue_pv())) break;
                pending = true;
                pv_n = n;
                pv_item = cur_item;
                pv_first = (t.t == 0);
                pv_last = (t.t == t.ntiles - 1);
                ++n;
                cursor_advance(m, anchors, item_id, queue_items, cur, status);
            }
            if (ok && pending) ok = issue_pv();
            if (!ok) *abort_flag = 1;
            // Drain: all MMAs issued by this thread complete before TMEM is released.
            mma_commit(&bars->drain);
            volatile int never = 0;
            mbar_wait(&bars->drain, 0, &never, kTimeoutNs);
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
            while (st.left > 0) {
                TileRef t;
                stream_next(m, anchors, item_id, queue_items, st, t, status);
                if (t.ntiles == 0) continue;
                const int ob = i & 1;
                if (!mbar_wait(&bars->stat_full[ob], (i >> 1) & 1u, abort_flag, kTimeoutNs)) break;
                if (!mbar_wait(&bars->o_ready[ob], (i >> 1) & 1u, abort_flag, kTimeoutNs)) break;
                tc_fence_after();
                const float* sp = stat + ob * 384;
                const float m_used = sp[r];
                const float l_row = sp[128 + r] + sp[256 + r];
                const float inv_l = 1.f / l_row;
                float* op = o_part + t.id * (int64_t)R * 128;
                const uint32_t to = tmem + kColO0 + 128u * ob + lane_off;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t ov[32];
                    tmem_ld32(to + cc * 32, ov);
                    tmem_wait_ld();
                    if (cc == 3) {  // O[ob] fully read: the MMA may start item i+2 in it
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
                if (r < R) lse_part[t.id * R + r] = (m_used + lg2_approx(l_row)) * 0.6931471805599453f;
                ++i;
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
        if (!skip) {
            const int wg = warp >> 2;               // key-column half
            const int quad = warp & 3;              // TMEM lane quadrant
            const int r = quad * 32 + lane;         // query-tile row
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const float c = m.scale * 1.4426950408889634f;  // log2(e)
            const uint64_t c2 = f2_pack(c, c);
            const bool leader = threadIdx.x == 0;
            uint32_t n = 0, i = 0;
            bool ok = true;
            ItemStream st;
            stream_init(m, anchors, item_id, queue_items, q0, q1, st);
            while (st.left > 0 && ok) {
                TileRef t;
                stream_next(m, anchors, item_id, queue_items, st, t, status);
                if (t.ntiles == 0) continue;
                const int ob = i & 1;
                const uint32_t to = tmem + kColO0 + 128u * ob + lane_off + wg * 64;
                float m_used = -INFINITY, l = 0.f;
                for (int tt = 0; tt < t.ntiles; ++tt, ++n) {
                    if (!mbar_wait(&bars->s_full, n & 1u, abort_flag, kTimeoutNs)) { ok = false; break; }
                    tc_fence_after();
                    uint32_t sr[64];
                    tmem_ld32(tS + lane_off + wg * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld32(tS + lane_off + wg * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(&bars->s_free);  // S(n) is in registers: QK^T(n+1) may overwrite it
                    if (leader) {                // QK^T(n) is complete: K(n), and Q after the item's last tile
                        mbar_arrive(&bars->k_empty[n & 1]);
                        if (tt == t.ntiles - 1) mbar_arrive(&bars->q_empty[i & 1]);
                    }
                    const int valid = t.nvis - tt * kKeysPerTile - wg * 64;  // visible keys in this half
                    if (valid < 64) {                                        // only an item's last tile
#pragma unroll
                        for (int u = 0; u < 64; ++u)
                            if (u >= valid) sr[u] = __float_as_uint(-INFINITY);
                    }
                    float mx;
                    {
                        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
                        for (int u = 0; u < 64; u += 8) {
                            m0 = max3f(m0, __uint_as_float(sr[u]), __uint_as_float(sr[u + 1]));
                            m1 = max3f(m1, __uint_as_float(sr[u + 2]), __uint_as_float(sr[u + 3]));
                            m2 = max3f(m2, __uint_as_float(sr[u + 4]), __uint_as_float(sr[u + 5]));
                            m3 = max3f(m3, __uint_as_float(sr[u + 6]), __uint_as_float(sr[u + 7]));
                        }
                        // Exchange with the thread holding the other half of the row (bounded wait).
                        const float mine = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
                        float* rp = red + (n & 1) * 256;
                        rp[wg * 128 + r] = mine;
                        mbar_arrive(&bars->red_bar[n & 1]);
                        if (!mbar_wait(&bars->red_bar[n & 1], (n >> 1) & 1u, abort_flag, kTimeoutNs)) {
                            ok = false;
                            break;
                        }
                        mx = fmaxf(mine, rp[(1 - wg) * 128 + r]) * c;
                    }
                    bool pv_prev_done = (n == 0);
                    if (tt == 0) {
                        m_used = mx;
                    } else if (mx > m_used + kRescaleLog2) {
                        // Rescale this half of O once PV(n-1) has landed in it.
                        if (!mbar_wait(&bars->pv_done, (n - 1) & 1u, abort_flag, kTimeoutNs)) { ok = false; break; }
                        tc_fence_after();
                        pv_prev_done = true;
                        const float alpha = ex2_approx(m_used - mx);
                        l *= alpha;
#pragma unroll 1
                        for (int cc = 0; cc < 2; ++cc) {
                            uint32_t ov[32];
                            tmem_ld32(to + cc * 32, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int u = 0; u < 32; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * alpha);
                            tmem_st32(to + cc * 32, ov);
                        }
                        m_used = mx;
                    }
                    // P = 2^(s*c - m) in bf16 pairs: keys 64wg.. -> P columns 32wg..
                    const uint64_t negm2 = f2_pack(-m_used, -m_used);
                    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
                    uint32_t pk[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        float t0, t1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * u]), __uint_as_float(sr[2 * u + 1])), c2, negm2),
                                  t0, t1);
                        const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
                        acc[u & 3] = f2_add(acc[u & 3], f2_pack(p0, p1));
                        __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);  // .x (low half) = even key
                        pk[u] = *reinterpret_cast<uint32_t*>(&hp);
                    }
                    {
                        float a0, a1, b0, b1, c0, c1, d0, d1;
                        f2_unpack(acc[0], a0, a1);
                        f2_unpack(acc[1], b0, b1);
                        f2_unpack(acc[2], c0, c1);
                        f2_unpack(acc[3], d0, d1);
                        l += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
                    }
                    // P is single-buffered: PV(n-1), its last reader, must have completed.
                    if (!pv_prev_done) {
                        if (!mbar_wait(&bars->pv_done, (n - 1) & 1u, abort_flag, kTimeoutNs)) { ok = false; break; }
                        tc_fence_after();
                    }
                    if (leader && n > 0) mbar_arrive(&bars->v_empty[(n - 1) & 1]);  // V(n-1) read
                    tmem_st32(tP + lane_off + wg * 32, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&bars->p_full);
                }
                if (!ok) break;
                // Hand m and l to the epilogue; stat[i % 2] was last read by the epilogue of item i-2.
                if (i >= 2 && !mbar_wait(&bars->o_free[ob], ((i >> 1) - 1) & 1u, abort_flag, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                float* sp = stat + ob * 384;
                if (wg == 0) sp[r] = m_used;
                sp[128 + wg * 128 + r] = l;
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

cudaError_t launch_fwd_tc(const Meta& m, const void* q, const void* k, const void* v, const int32_t* anchors,
                          const int32_t* item_id, const int32_t* queue_off, const int32_t* queue_items,
                          int32_t n_workers, float* o_part, float* lse_part, int32_t* status, cudaStream_t st) {
    CUtensorMap tq, tk, tv;
    if (m.n_queries == 0 || m.total_keys == 0) return cudaSuccess;
    if (!make_map(&tq, q, m.n_queries, m.hq, m.d, m.group, m.block) ||
        !make_map(&tk, k, m.total_keys, m.hkv, m.d, 1, kKeysPerTile) ||
        !make_map(&tv, v, m.total_keys, m.hkv, m.d, 1, kKeysPerTile))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(fwd_tc_kernel, smem)");
    fwd_tc_kernel<<<n_workers, kThreads, kSmemBytes, st>>>(m, tq, tk, tv, anchors, item_id, queue_off, queue_items,
                                                           o_part, lse_part, status);
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
