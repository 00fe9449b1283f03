// Chunk-partial forward on the 5th-generation tensor cores (sm_100a): TMA -> tcgen05.mma -> TMEM.
//
// Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, Abstract: exact
// attention over context chunks, each producing a query-sized partial output and a per-row
// log-sum-exp; the chunks are placed by the cost-aware LPT plan. Here one persistent CTA per SM
// walks the SM's LPT queue. A work item (s, c, g, b) is one 128-row query tile — the block*G rows
// (query i, head g*G+hl) of block b at kv head g, shared by the G query heads of the GQA group —
// against the ceil(nvis/128) key tiles of chunk c that the block sees.
//
// Roles (384 threads, three warpgroups):
//   warps 0-3 / 4-7  softmax warpgroups of slot 0 / slot 1 (one query-tile row per thread); they
//                    raise their register budget to 200 so a whole S row stays in registers
//   warp 8           TMA producer: Q tile per item, K then V tile per key tile, 5-deep ring
//   warp 9           MMA issuer (one thread) and TMEM owner (512 columns)
//   warps 8-11       lower their budget to 104 registers (warps 10-11 only do that)
// The two slots take alternate items of the queue and ping-pong on the tensor core: while one
// slot's warpgroup runs the softmax of its tile, the tensor core runs the other slot's QK^T / PV.
//
// TMEM: S_k = Q K^T (128 x 128 fp32) at columns 128k; P_k (bf16, 64 columns) written over the first
// half of S_k; O_k (128 x 128 fp32) at columns 256 + 128k. The next QK^T of a slot is issued only
// after that slot's PV has completed, because P aliases S.
//
// Online softmax in log2 units (x = s * scale * log2 e); the running reference max is only moved
// when a tile's max exceeds it by more than 8 (so P <= 256), which keeps O and l consistent and
// rescales O rarely. LSE = (m + log2 l) * ln 2.
//
// Every wait is bounded (2 s); on expiry the CTA raises SPLITKV_DEV_TIMEOUT, drains its copies and
// MMAs in flight, frees TMEM and returns.
#include <cstdio>

#include "common.cuh"
#include "sm100.cuh"

namespace splitkv {

namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kSoftmaxRegs = 200;  // per SM sub-partition: 200 + 200 + 104 = 504 = 3 x 168 launched
constexpr int kControlRegs = 104;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kNB = 5;               // K/V ring depth (32 KB buffers)
constexpr int kTileBytes = 32768;    // 128 x 128 bf16, as two 128-byte-wide halves
constexpr int kHalfBytes = 16384;
constexpr int kKeysPerTile = 128;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;

constexpr int kOffQ = 0;                                   // 2 x 32 KB
constexpr int kOffKV = 2 * kTileBytes;                     // kNB x 32 KB
constexpr int kOffBar = kOffKV + kNB * kTileBytes;
constexpr int kNumBars = 2 * kNB + 2 * 5 + 1;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 64 + 1024;  // + alignment slack

struct Bars {
    uint64_t kv_full[kNB];
    uint64_t kv_empty[kNB];
    uint64_t q_full[2];
    uint64_t q_empty[2];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t pv_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

struct TileRef {
    int64_t id;
    int32_t s, c, g, j;
    int32_t nvis, ntiles, t;
};

// The items of one slot (queue positions first, first+2, ...), fetched ahead: each call hands out
// the next (item id, anchor) and issues the loads one link further for the three items after it
// (anchor of n+1, id of n+2, queue entry of n+3), so no role waits on a dependent global load
// chain when it moves to a new item.
struct ItemStream {
    int32_t pos, end, left;
    int64_t id1;  // item n+1 (loaded)
    int32_t a1;   // anchor of item n+1 (in flight)
    int64_t id2;  // item n+2 (in flight)
    int32_t k3;   // queue entry of item n+3 (in flight)
};

__device__ __forceinline__ int64_t load_id(const Meta& m, const int32_t* __restrict__ item_id, int32_t k) {
    return k >= 0 ? (int64_t)__ldg(item_id + k) : -1;
}
__device__ __forceinline__ int32_t load_anchor(const Meta& m, const int32_t* __restrict__ anchors, int64_t id) {
    return (id >= 0 && id < m.n_items) ? __ldg(anchors + decode_item(m, id).j) : 0;
}

__device__ __forceinline__ void stream_init(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                            const int32_t* queue_items, int32_t first, int32_t end, ItemStream& st) {
    st.end = end;
    st.left = first < end ? (end - first + 1) / 2 : 0;
    const int32_t k0 = st.left > 0 ? __ldg(queue_items + first) : -1;
    const int32_t k1 = st.left > 1 ? __ldg(queue_items + first + 2) : -1;
    st.k3 = st.left > 2 ? __ldg(queue_items + first + 4) : -1;
    st.id1 = load_id(m, item_id, k0);
    st.id2 = load_id(m, item_id, k1);
    st.a1 = load_anchor(m, anchors, st.id1);
    st.pos = first + 6;
}

// Next item as a tile reference (ntiles == 0 for an invalid entry, which raises BAD_PLAN).
__device__ __forceinline__ void stream_next(const Meta& m, const int32_t* anchors, const int32_t* item_id,
                                            const int32_t* queue_items, ItemStream& st, TileRef& tr, int32_t* status) {
    const int64_t id = st.id1;
    const int32_t a = st.a1;
    --st.left;
    st.a1 = load_anchor(m, anchors, st.id2);
    st.id1 = st.id2;
    st.id2 = load_id(m, item_id, st.k3);
    st.k3 = st.pos < st.end ? __ldg(queue_items + st.pos) : -1;
    st.pos += 2;
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

// Items of one slot as a sequence of key tiles.
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
    uint8_t* q_smem = smem + kOffQ;
    uint8_t* kv_smem = smem + kOffKV;
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t q0 = queue_off[blockIdx.x], q1 = queue_off[blockIdx.x + 1];

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNB; ++i) {
            mbar_init(&bars->kv_full[i], 1);
            mbar_init(&bars->kv_empty[i], 1);
        }
        for (int k = 0; k < 2; ++k) {
            mbar_init(&bars->q_full[k], 1);
            mbar_init(&bars->q_empty[k], 1);
            mbar_init(&bars->s_full[k], 1);
            mbar_init(&bars->p_full[k], 128);
            mbar_init(&bars->pv_done[k], 1);
        }
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        bars->status0 = status_bad(status) ? 1 : 0;
        fence_barrier_init();
    }
    // Rows of the Q buffers beyond block*G are never loaded: keep them finite (zero).
    for (int i = threadIdx.x; i < 2 * kTileBytes / 16; i += kThreads)
        reinterpret_cast<uint4*>(q_smem)[i] = make_uint4(0, 0, 0, 0);
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
    const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
    const uint32_t tO[2] = {tmem + 256u, tmem + 384u};

    if (warp >= 8) {
        // Control warpgroup: give registers to the softmax warpgroups.
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kControlRegs));
        if (!skip && warp == kProducerWarp) {
            if (lane == 0) {
                tma_prefetch_desc(&tmQ);
                tma_prefetch_desc(&tmK);
                tma_prefetch_desc(&tmV);
                const uint32_t q_bytes = 2u * 64u * (uint32_t)G * (uint32_t)m.block * 2u;
                Cursor cur[2];
                TileRef pv_tile[2];
                bool pending[2] = {false, false};
                uint32_t kv_seq = 0, qseq[2] = {0, 0};
                int32_t last_kv_parity[kNB];
                bool issued[kNB];
                for (int i = 0; i < kNB; ++i) { issued[i] = false; last_kv_parity[i] = 0; }
                bool q_issued[2] = {false, false};
                uint32_t q_last_parity[2] = {0, 0};
                bool ok = true;
                for (int k = 0; k < 2; ++k) cursor_init(m, anchors, item_id, queue_items, q0 + k, q1, cur[k], status);
                auto load_kv = [&](const CUtensorMap* map, const TileRef& t) -> bool {
                    const int buf = kv_seq % kNB;
                    const uint32_t ph = (kv_seq / kNB) & 1u;
                    if (!mbar_wait(&bars->kv_empty[buf], ph ^ 1u, abort_flag, kTimeoutNs)) return false;
                    mbar_arrive_expect_tx(&bars->kv_full[buf], kTileBytes);
                    const int32_t row = (int32_t)(m.key_off[t.s] + (int64_t)t.c * m.chunk + (int64_t)t.t * kKeysPerTile);
                    uint8_t* dst = kv_smem + buf * kTileBytes;
                    tma_load_3d(dst, map, &bars->kv_full[buf], 0, t.g, row);
                    tma_load_3d(dst + kHalfBytes, map, &bars->kv_full[buf], 64, t.g, row);
                    issued[buf] = true;
                    last_kv_parity[buf] = (int32_t)ph;
                    ++kv_seq;
                    return true;
                };
                auto emit_qk = [&](int k) -> bool {
                    const TileRef t = cur[k].cur;
                    if (t.t == 0) {
                        if (!mbar_wait(&bars->q_empty[k], (qseq[k] & 1u) ^ 1u, abort_flag, kTimeoutNs)) return false;
                        mbar_arrive_expect_tx(&bars->q_full[k], q_bytes);
                        uint8_t* dst = q_smem + k * kTileBytes;
                        tma_load_3d(dst, &tmQ, &bars->q_full[k], 0, t.g * G, m.block * t.j);
                        tma_load_3d(dst + kHalfBytes, &tmQ, &bars->q_full[k], 64, t.g * G, m.block * t.j);
                        q_issued[k] = true;
                        q_last_parity[k] = qseq[k] & 1u;
                        ++qseq[k];
                    }
                    if (!load_kv(&tmK, t)) return false;
                    pv_tile[k] = t;
                    pending[k] = true;
                    cursor_advance(m, anchors, item_id, queue_items, cur[k], status);
                    return true;
                };
                for (int k = 0; k < 2 && ok; ++k)
                    if (cur[k].has) ok = emit_qk(k);
                while (ok && (pending[0] || pending[1])) {
                    for (int k = 0; k < 2 && ok; ++k) {
                        if (pending[k]) {
                            ok = load_kv(&tmV, pv_tile[k]);
                            pending[k] = false;
                        }
                        if (ok && cur[k].has) ok = emit_qk(k);
                    }
                }
                // Drain: every copy this warp issued must have landed before the CTA exits.
                for (int i = 0; i < kNB; ++i)
                    if (issued[i]) {
                        volatile int never = 0;
                        mbar_wait(&bars->kv_full[i], (uint32_t)last_kv_parity[i], &never, kTimeoutNs);
                    }
                for (int k = 0; k < 2; ++k)
                    if (q_issued[k]) {
                        volatile int never = 0;
                        mbar_wait(&bars->q_full[k], q_last_parity[k], &never, kTimeoutNs);
                    }
            }
            __syncwarp();
        } else if (!skip && warp == kMmaWarp) {
            if (lane == 0) {
                constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(128, 128, false, false);
                constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, 128, false, true);
                const uint32_t q_base = smem_u32(q_smem), kv_base = smem_u32(kv_smem);
                Cursor cur[2];
                bool pending[2] = {false, false}, pv_first[2] = {false, false};
                uint32_t kv_seq = 0, qseq[2] = {0, 0}, tile_seq[2] = {0, 0};
                bool ok = true;
                for (int k = 0; k < 2; ++k) cursor_init(m, anchors, item_id, queue_items, q0 + k, q1, cur[k], status);
                auto emit_qk = [&](int k) -> bool {
                    const TileRef t = cur[k].cur;
                    if (tile_seq[k] > 0 &&
                        !mbar_wait(&bars->pv_done[k], (tile_seq[k] - 1) & 1u, abort_flag, kTimeoutNs))
                        return false;
                    if (t.t == 0) {
                        if (!mbar_wait(&bars->q_full[k], qseq[k] & 1u, abort_flag, kTimeoutNs)) return false;
                        ++qseq[k];
                    }
                    const int buf = kv_seq % kNB;
                    if (!mbar_wait(&bars->kv_full[buf], (kv_seq / kNB) & 1u, abort_flag, kTimeoutNs)) return false;
                    tc_fence_after();
                    const uint32_t qa = q_base + k * kTileBytes, kb = kv_base + buf * kTileBytes;
    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                        mma_ss(tS[k], umma_desc_sw128(qa + off, 16, 1024), umma_desc_sw128(kb + off, 16, 1024),
                               idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&bars->s_full[k]);
                    mma_commit(&bars->kv_empty[buf]);
                    if (t.t == t.ntiles - 1) mma_commit(&bars->q_empty[k]);
                    ++kv_seq;
                    pv_first[k] = (t.t == 0);
                    pending[k] = true;
                    ++tile_seq[k];
                    cursor_advance(m, anchors, item_id, queue_items, cur[k], status);
                    return true;
                };
                auto emit_pv = [&](int k) -> bool {
                    if (!mbar_wait(&bars->p_full[k], (tile_seq[k] - 1) & 1u, abort_flag, kTimeoutNs)) return false;
                    const int buf = kv_seq % kNB;
                    if (!mbar_wait(&bars->kv_full[buf], (kv_seq / kNB) & 1u, abort_flag, kTimeoutNs)) return false;
                    tc_fence_after();
                    const uint32_t vb = kv_base + buf * kTileBytes;
    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        // A = P[:, 16kk .. 16kk+16) packed two bf16 per column; B = V rows 16kk.., MN-major.
                        mma_ts(tO[k], tS[k] + (uint32_t)(kk * 8), umma_desc_sw128(vb + kk * 2048, kHalfBytes, 1024),
                               idesc_pv, (!pv_first[k] || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&bars->pv_done[k]);
                    mma_commit(&bars->kv_empty[buf]);
                    ++kv_seq;
                    pending[k] = false;
                    return true;
                };
                for (int k = 0; k < 2 && ok; ++k)
                    if (cur[k].has) ok = emit_qk(k);
                while (ok && (pending[0] || pending[1])) {
                    for (int k = 0; k < 2 && ok; ++k) {
                        if (pending[k]) ok = emit_pv(k);
                        if (ok && cur[k].has) ok = emit_qk(k);
                    }
                }
                // Drain: all MMAs issued by this thread complete before TMEM is released.
                mma_commit(&bars->drain);
                volatile int never = 0;
                mbar_wait(&bars->drain, 0, &never, kTimeoutNs);
            }
            __syncwarp();
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
        if (!skip) {
            const int k = warp >> 2;                // slot
            const int quad = warp & 3;              // TMEM lane quadrant
            const int r = quad * 32 + lane;         // query-tile row
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const float c = m.scale * 1.4426950408889634f;  // log2(e)
            const uint64_t c2 = f2_pack(c, c);
            uint32_t tile_seq = 0;
            bool ok = true;
            ItemStream st;
            stream_init(m, anchors, item_id, queue_items, q0 + k, q1, st);
            while (st.left > 0 && ok) {
                TileRef t;
                stream_next(m, anchors, item_id, queue_items, st, t, status);
                if (t.ntiles == 0) continue;
                float m_used = -INFINITY, l = 0.f;
                for (int tt = 0; tt < t.ntiles; ++tt) {
                    if (!mbar_wait(&bars->s_full[k], tile_seq & 1u, abort_flag, kTimeoutNs)) { ok = false; break; }
                    tc_fence_after();
                    // The whole S row in registers: one TMEM round trip.
                    uint32_t sr[128];
    #pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        tmem_ld32(tS[k] + lane_off + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[cc * 32]));
                    tmem_wait_ld();
                    const int valid = t.nvis - tt * kKeysPerTile;  // keys of this tile the block sees (>= 1)
                    if (valid < kKeysPerTile) {                    // only an item's last tile can be partial
    #pragma unroll
                        for (int u = 0; u < 128; ++u)
                            if (u >= valid) sr[u] = __float_as_uint(-INFINITY);
                    }
                    float mx;
                    {
                        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
    #pragma unroll
                        for (int u = 0; u < 128; u += 8) {
                            m0 = max3f(m0, __uint_as_float(sr[u]), __uint_as_float(sr[u + 1]));
                            m1 = max3f(m1, __uint_as_float(sr[u + 2]), __uint_as_float(sr[u + 3]));
                            m2 = max3f(m2, __uint_as_float(sr[u + 4]), __uint_as_float(sr[u + 5]));
                            m3 = max3f(m3, __uint_as_float(sr[u + 6]), __uint_as_float(sr[u + 7]));
                        }
                        mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * c;
                    }
                    if (tt == 0) {
                        m_used = mx;
                    } else if (mx > m_used + kRescaleLog2) {
                        // The previous PV of this slot completed before this tile's QK^T was issued.
                        const float alpha = ex2_approx(m_used - mx);
                        l *= alpha;
    #pragma unroll 1
                        for (int cc = 0; cc < 4; ++cc) {
                            uint32_t ov[32];
                            tmem_ld32(tO[k] + lane_off + cc * 32, ov);
                            tmem_wait_ld();
    #pragma unroll
                            for (int u = 0; u < 32; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * alpha);
                            tmem_st32(tO[k] + lane_off + cc * 32, ov);
                        }
                        m_used = mx;
                    }
                    // P = 2^(s*c - m) in bf16, packed two per column over the first 64 columns of S.
                    const uint64_t negm2 = f2_pack(-m_used, -m_used);
                    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
    #pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        uint32_t pk[16];
    #pragma unroll
                        for (int u = 0; u < 16; ++u) {
                            const int v = h * 32 + 2 * u;
                            float t0, t1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[v]), __uint_as_float(sr[v + 1])), c2, negm2), t0,
                                      t1);
                            const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
                            acc[u & 3] = f2_add(acc[u & 3], f2_pack(p0, p1));
                            __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);  // .x (low half) = even key
                            pk[u] = *reinterpret_cast<uint32_t*>(&hp);
                        }
                        tmem_st16(tS[k] + lane_off + h * 16, pk);
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
                    mbar_arrive(&bars->p_full[k]);
                    ++tile_seq;
                }
                if (!ok) break;
                // Epilogue: wait for the item's last PV, normalise, store partial O and LSE.
                if (!mbar_wait(&bars->pv_done[k], (tile_seq - 1) & 1u, abort_flag, kTimeoutNs)) { ok = false; break; }
                tc_fence_after();
                const float inv_l = 1.f / l;
                float* op = o_part + t.id * (int64_t)R * 128;
    #pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t ov[32];
                    tmem_ld32(tO[k] + lane_off + cc * 32, ov);
                    tmem_wait_ld();
                    if (r < R) {
    #pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            float4 x = make_float4(__uint_as_float(ov[4 * u]) * inv_l, __uint_as_float(ov[4 * u + 1]) * inv_l,
                                                   __uint_as_float(ov[4 * u + 2]) * inv_l,
                                                   __uint_as_float(ov[4 * u + 3]) * inv_l);
                            *reinterpret_cast<float4*>(op + ((int64_t)(cc * 8 + u) * R + r) * 4) = x;
                        }
                    }
                }
                if (r < R) lse_part[t.id * R + r] = (m_used + lg2_approx(l)) * 0.6931471805599453f;
            }
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
