// Backward on the 5th-generation tensor cores (sm_100a): TMA -> tcgen05.mma -> TMEM, in one pass.
//
// Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, title and Abstract: the
// method trains diffusion drafters, so gradients flow back through the same exact attention. With
// P = exp(s - LSE) recomputed from the stored natural-log LSE, D = rowsum(dO * O) and
// dS = scale P (dP - D), dP = dO V^T:
//   dV = P^T dO,  dK = dS^T Q,  dQ = dS K
// One CTA per 128-key tile (key-stationary): S^T and dP^T are computed once per (key tile, block)
// pair, dV and dK accumulate in TMEM over the blocks that see the tile, and each pair's dQ^T = K^T dS^T
// (head dim x query rows) is added into the zeroed float32 dq with coalesced reductions (one 128-byte
// line per store instruction). Five GEMMs per pair, the useful work of the backward.
//
// Per pair: S^T = K Q_b^T and dP^T = V dO_b^T (M = 128 keys, N = 64 query rows per step, K = d) into
// TMEM; two threads per key (query rows 0-31 / 32-63 of the step, in two warps of the same SM
// sub-partition, so that the MUFU unit has two warps to interleave) form P^T and dS^T in bf16, P^T
// back into TMEM over S^T's columns and dS^T into shared memory (128-byte swizzle), where it serves
// both as the K-major A operand of dK += dS^T Q_b and as the MN-major B operand of dQ^T = K^T dS^T.
// Two issuing threads: one thread gets one tcgen05.mma per ~120 cycles, two interleave.
// (Measured on the backward of train_4x16k: 1085 -> 1042 us for two threads per key, and on
// train_4x64k 13.65 -> 12.98 ms for two issuers, in the earlier two-kernel form.)
//
// Every wait is bounded (2 s); on expiry the CTA raises SPLITKV_DEV_TIMEOUT, drains its copies and
// MMAs in flight, frees TMEM and returns.
#include <cstdio>

#include "common.cuh"
#include "scan.cuh"
#include "sm100.cuh"
#include "tma_map.cuh"

namespace splitkv {

namespace {

using namespace sm100;

constexpr int kTileBytes = 32768;  // 128 x 128 bf16, as two 128-byte-wide halves
constexpr int kHalfBytes = 16384;
constexpr int kKeys = 128;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kIdescSS64 = umma_idesc_bf16_f32(128, 64, false, false);  // N = 64 query rows (one step)
constexpr uint32_t kIdescTS = umma_idesc_bf16_f32(128, 128, false, true);   // B MN-major

// Per-row constants of one (block j, kv head g) query tile, rows r = i*G + hl contiguous, negated so
// that each enters one fused multiply-add: l2 = -LSE * log2 e and dvec = -scale * rowsum(dO * O).
// One warp per row.
template <typename T>
__global__ void __launch_bounds__(256) rows_kernel(Meta m, const T* __restrict__ o, const T* __restrict__ dout,
                                                   const float* __restrict__ lse, float* __restrict__ l2,
                                                   float* __restrict__ dvec) {
    const int lane = threadIdx.x & 31;
    const int64_t q = ((int64_t)blockIdx.x * 256 + threadIdx.x) >> 5;
    if (q >= m.n_blocks * m.hkv * m.rows) return;
    const int64_t jg = q / m.rows;
    const int r = (int)(q % m.rows);
    const int64_t j = jg / m.hkv;
    const int g = (int)(jg % m.hkv);
    const int64_t orow = ((int64_t)m.block * j + r / m.group) * m.hq + (int64_t)g * m.group + r % m.group;
    float acc = 0.f;
    for (int dd = lane; dd < m.d; dd += 32) acc = fmaf(to_f32(o[orow * m.d + dd]), to_f32(dout[orow * m.d + dd]), acc);
    acc = warp_reduce_sum(acc);
    if (lane == 0) {
        l2[q] = -lse[orow] * kLog2e;
        dvec[q] = -m.scale * acc;
    }
}

// ------------------------------------------------------------------ one pass: dK, dV and dQ
constexpr int kKvThreads = 608;  // warps 0-7: elementwise (key row x query half); warp 8: TMA producer;
                                 // warps 9, 10: MMA issuers (S^T, dV, dK; dP^T, dQ^T); warps 11-18: dQ out
constexpr int kKvLoadWarp = 8, kKvMmaWarp = 9, kKvMma2Warp = 10, kKvDqWarp0 = 11;
constexpr int kDsBytes = 16384;              // dS^T of one step: 128 keys x 64 query rows, bf16
constexpr int kKvOffK = 0;
constexpr int kKvOffV = kTileBytes;
constexpr int kKvOffQ = 2 * kTileBytes;      // Q_b[2]
constexpr int kKvOffDo = 4 * kTileBytes;     // dO_b[2]
constexpr int kKvOffDs = 6 * kTileBytes;     // dS^T[2], by step parity
constexpr int kKvOffRows = kKvOffDs + 2 * kDsBytes;  // float [2 slots][-LSE log2 e, -scale D][128]
constexpr int kKvOffBar = kKvOffRows + 2 * 2 * 128 * 4;
constexpr uint32_t kIdescDQ = umma_idesc_bf16_f32(128, 64, true, true);  // dQ^T = K^T dS^T, both MN-major

struct KvBars {
    uint64_t kv_full;
    uint64_t qd_full[2], qd_empty[2];  // Q_b, dO_b, rows of pair p in slot p % 2
    uint64_t s_full[2];                // S^T, dP^T of step u (parity u % 2) complete (one commit per issuer)
    uint64_t dp_read;                  // dP^T of step u loaded into registers (8 elementwise warps)
    uint64_t p_full[2];                // P^T (TMEM) and dS^T (shared memory) of step u written (8 warps)
    uint64_t dq_full, dq_free;         // dQ^T of step u complete / read out of TMEM (8 dQ warps)
    uint64_t acc_done;                 // every MMA complete: dV, dK final
    uint64_t epi_staged;               // all 8 elementwise warps staged their dV / dK rows
    uint64_t drain[2];
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

// No padding for alignment: the dynamic shared memory window starts 1024-byte aligned (checked at run
// time), and the tiles need all but a few hundred bytes of the 227 KB a CTA may hold.
constexpr int kKvSmemBytes = kKvOffBar + (int)sizeof(KvBars);
static_assert(kKvSmemBytes <= 227 * 1024, "backward tiles exceed the shared memory of one CTA");

// Adds the 32 values x[j] (query rows rbase + j of one block, head-dim index fixed per thread) into their
// dq rows: row r is query r / G of the block at head g * G + r % G, so query rows come in runs of G
// consecutive heads (G * 512 contiguous bytes of dq). With G a compile-time constant each run is one
// pointer and G reductions at constant offsets; rows r >= R (blocks of fewer than 64 rows) are
// predicated off. `row0` points at row rbase's head-dim index.
template <int G>
__device__ __forceinline__ void dq_add_rows(float* row0, int64_t query_stride, const uint32_t (&x)[32], int valid) {
    static_assert(32 % G == 0, "32 rows hold whole queries");
#pragma unroll
    for (int i = 0; i < 32 / G; ++i) {
        float* qp = row0 + i * query_stride;
#pragma unroll
        for (int hl = 0; hl < G; ++hl) {
            const int j = i * G + hl;
            red_add_f32_if(qp + hl * 128, __uint_as_float(x[j]), j < valid);
        }
    }
}

// Unit u: context key tile (t, sample s, kv head g) with g fastest and t slowest, so that the
// costliest tiles (small t: seen by the most blocks) start first; then the self tiles (block j,
// kv head g): the block's own 16 keys.
//
// Per pair (key tile, block b seeing it), in steps of 64 query rows (two for a block of more than 64
// rows), so that the tensor core computes step u + 1 while the elementwise warps work on step u.
// TMEM (512 columns): S^T / P^T of steps u and u + 1 (2 x 64), dP^T (64, free once the elementwise
// warps hold step u's values in registers), dQ^T (64), dV (128), dK (128).
//   issuer A: S^T(u) = K Q_h^T; then, once P^T(u) / dS^T(u) are written, dV += P^T(u) dO_h (P^T in
//             TMEM over S^T(u)'s columns) and dK += dS^T(u) Q_h (dS^T from shared memory);
//   issuer B: dP^T(u) = V dO_h^T; then dQ^T(u) = K^T dS^T(u) (d x 64 rows), which eight dQ warps (two
//             per TMEM lane quadrant, 32 query rows each) read out and add into dq.
// dS carries the softmax scale (dS = scale P (dP - D)), so dK and dQ need no further scaling.
__global__ void __launch_bounds__(kKvThreads, 1)
    bwd_tc_kernel(const __grid_constant__ Meta m, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmDo, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                  const __grid_constant__ CUtensorMap tmVb, int32_t tiles_max, const int32_t* __restrict__ anchors,
                  const float* __restrict__ l2, const float* __restrict__ dvec, float* __restrict__ dq,
                  float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dkb, float* __restrict__ dvb,
                  int32_t* __restrict__ status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
        if (threadIdx.x == 0) raise_status(status, SPLITKV_DEV_SMEM_ALIGN);
        return;
    }
    const int64_t n_ctx = (int64_t)tiles_max * m.batch * m.hkv;
    const int64_t unit = blockIdx.x;
    const bool self = unit >= n_ctx;
    int s = 0, g, lo, hi, nk;
    int64_t key0 = 0, krow;  // first key of the tile within its sample; its row in k/v (or kb/vb)
    if (!self) {
        g = (int)(unit % m.hkv);
        const int64_t rest = unit / m.hkv;
        s = (int)(rest % m.batch);
        const int64_t t = rest / m.batch;
        if (t * kKeys >= m.seq_len[s]) return;  // the sample is shorter: no such tile
        key0 = t * kKeys;
        nk = (int)min((int64_t)kKeys, m.seq_len[s] - key0);
        krow = m.key_off[s] + key0;
        // Blocks of sample s whose anchor exceeds key0 (a suffix: anchors ascend).
        hi = m.anchor_off[s + 1];
        int32_t a = m.anchor_off[s], b = hi;
        while (a < b) {
            const int32_t mid = (a + b) >> 1;
            if ((int64_t)__ldg(anchors + mid) > key0) b = mid;
            else a = mid + 1;
        }
        lo = a;
        if (!owns_chunk(m, s, (int32_t)(key0 / m.chunk))) hi = lo;  // another rank's chunk: zeros here
    } else {
        const int64_t sid = unit - n_ctx;
        const int32_t j = (int32_t)(sid / m.hkv);
        g = (int)(sid % m.hkv);
        lo = j;
        hi = owns_self(m, j) ? j + 1 : j;  // another rank's block: zeros here
        nk = m.block;
        krow = (int64_t)m.block * j;
    }
    const int32_t np = hi - lo;
    const int32_t steps = m.rows > 64 ? 2 : 1;
    const int32_t U = np * steps;

    float* rows = reinterpret_cast<float*>(smem + kKvOffRows);
    KvBars* bars = reinterpret_cast<KvBars*>(smem + kKvOffBar);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = m.group, R = m.rows;

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->qd_full[b], 1);
            mbar_init(&bars->qd_empty[b], 2);
            mbar_init(&bars->s_full[b], 2);
            mbar_init(&bars->p_full[b], 8);
        }
        mbar_init(&bars->dp_read, 8);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_free, 8);
        mbar_init(&bars->acc_done, 2);
        mbar_init(&bars->epi_staged, 8);
        mbar_init(&bars->drain[0], 1);
        mbar_init(&bars->drain[1], 1);
        bars->abort_flag = 0;
        bars->status0 = status_bad(status) ? 1 : 0;
        fence_barrier_init();
    }
    // Query rows beyond block*G are never loaded: keep Q_b, dO_b and the row constants finite (zero).
    if (R < 128)
        for (int i = threadIdx.x; i < 4 * kTileBytes / 16; i += kKvThreads)
            reinterpret_cast<uint4*>(smem + kKvOffQ)[i] = make_uint4(0, 0, 0, 0);
    for (int i = threadIdx.x; i < 2 * 2 * 128; i += kKvThreads) rows[i] = 0.f;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == kKvMmaWarp) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 192, tdV = tmem + 256, tdK = tmem + 384;
    const bool skip = bars->status0 != 0;

    if (warp == kKvLoadWarp) {
        if (!skip && lane == 0 && np > 0) {
            const CUtensorMap* mk = self ? &tmKb : &tmK;
            const CUtensorMap* mv = self ? &tmVb : &tmV;
            const uint32_t q_bytes = 2u * 64u * (uint32_t)G * (uint32_t)m.block * 2u;
            mbar_arrive_expect_tx(&bars->kv_full, 2 * kTileBytes);
            tma_load_3d(smem + kKvOffK, mk, &bars->kv_full, 0, g, (int32_t)krow);
            tma_load_3d(smem + kKvOffK + kHalfBytes, mk, &bars->kv_full, 64, g, (int32_t)krow);
            tma_load_3d(smem + kKvOffV, mv, &bars->kv_full, 0, g, (int32_t)krow);
            tma_load_3d(smem + kKvOffV + kHalfBytes, mv, &bars->kv_full, 64, g, (int32_t)krow);
            int32_t issued = 0;
            for (int32_t p = 0; p < np; ++p) {
                const int slot = p & 1;
                if (!mbar_wait(&bars->qd_empty[slot], ((p >> 1) & 1u) ^ 1u, abort_flag, kTimeoutNs)) break;
                const int32_t b = lo + p;
                mbar_arrive_expect_tx(&bars->qd_full[slot], 2 * q_bytes + 2u * (uint32_t)R * 4u);
                uint8_t* dqs = smem + kKvOffQ + slot * kTileBytes;
                uint8_t* ddo = smem + kKvOffDo + slot * kTileBytes;
                tma_load_3d(dqs, &tmQ, &bars->qd_full[slot], 0, g * G, m.block * b);
                tma_load_3d(dqs + kHalfBytes, &tmQ, &bars->qd_full[slot], 64, g * G, m.block * b);
                tma_load_3d(ddo, &tmDo, &bars->qd_full[slot], 0, g * G, m.block * b);
                tma_load_3d(ddo + kHalfBytes, &tmDo, &bars->qd_full[slot], 64, g * G, m.block * b);
                const int64_t rb = ((int64_t)b * m.hkv + g) * R;
                bulk_load(rows + slot * 256, l2 + rb, (uint32_t)R * 4u, &bars->qd_full[slot]);
                bulk_load(rows + slot * 256 + 128, dvec + rb, (uint32_t)R * 4u, &bars->qd_full[slot]);
                issued = p + 1;
            }
            // Drain: every copy this thread started has landed before the CTA exits.
            volatile int never = 0;
            mbar_wait(&bars->kv_full, 0, &never, kTimeoutNs);
            for (int32_t p = (issued > 2 ? issued - 2 : 0); p < issued; ++p)
                mbar_wait(&bars->qd_full[p & 1], (p >> 1) & 1u, &never, kTimeoutNs);
        }
    } else if (warp == kKvMmaWarp || warp == kKvMma2Warp) {
        // Two issuers with 16 MMAs per step each (one thread issues one tcgen05.mma per ~120 cycles, two
        // interleave). Each issuer's MMAs execute in its issue order: S^T(u + 2) overwrites P^T(u) only
        // after dV(u) has read it. dP^T(u) overwrites dP^T(u - 1) once the elementwise warps hold it in
        // registers (dp_read), dQ^T(u) overwrites dQ^T(u - 1) once the dQ warps have read it (dq_free). The
        // shared-memory dS^T of step u is rewritten by the elementwise pass of step u + 2, which starts
        // after S^T(u + 2) and dP^T(u + 2), issued after dK(u) and dQ^T(u).
        const bool isA = warp == kKvMmaWarp;
        if (!skip && lane == 0 && np > 0) {
            bool ok = mbar_wait(&bars->kv_full, 0, abort_flag, kTimeoutNs);
            tc_fence_after();
            const uint64_t dA1 = umma_desc_sw128(smem_u32(smem + (isA ? kKvOffK : kKvOffV)), 16, 1024);
            // K^T as an MN-major A operand: head-dim halves 16 KB apart, 8-key groups 1024 bytes apart.
            const uint64_t dKt = umma_desc_sw128(smem_u32(smem + kKvOffK), kHalfBytes, 1024);
            // First GEMM of step u: S^T(u) = K Q_h^T  /  dP^T(u) = V dO_h^T into buffer u % 2 (64 columns),
            // B = the step's 64 query rows of Q_b / dO_b (K-major, rows 64h .. of the slot's tile).
            auto first = [&](int32_t u) -> bool {
                const int32_t p = u / steps, h = u % steps;
                const int slot = p & 1;
                if (h == 0 && !mbar_wait(&bars->qd_full[slot], (p >> 1) & 1u, abort_flag, kTimeoutNs)) return false;
                if (!isA && u >= 1 && !mbar_wait(&bars->dp_read, (u - 1) & 1u, abort_flag, kTimeoutNs))
                    return false;
                tc_fence_after();
                const uint32_t src = smem_u32(smem + (isA ? kKvOffQ : kKvOffDo) + slot * kTileBytes) + 8192u * h;
                const uint64_t dB1 = umma_desc_sw128(src, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) / 16);
                    mma_ss(isA ? tS + 64u * (u & 1) : tdP, dA1 + off, dB1 + off, kIdescSS64, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[u & 1]);
                if (!isA && h == steps - 1) mma_commit(&bars->qd_empty[slot]);  // dO_b read for the last time
                return true;
            };
            // Second half of step u once P^T(u) / dS^T(u) are written (16 query rows or keys per MMA).
            auto second = [&](int32_t u) -> bool {
                const int32_t p = u / steps, h = u % steps;
                const int slot = p & 1;
                if (!mbar_wait(&bars->p_full[u & 1], (u >> 1) & 1u, abort_flag, kTimeoutNs)) return false;
                tc_fence_after();
                const uint32_t ds = smem_u32(smem + kKvOffDs + (u & 1) * kDsBytes);
                if (isA) {
                    // dV += P^T(u) dO_h: rows 32w' + 16i of the step are bf16 pairs at columns 32w' + 8i of
                    // S^T(u)'s buffer. dK += dS^T(u) Q_h: dS^T K-major (keys x 64 rows, 32 bytes per 16 rows).
                    const uint64_t dDo = umma_desc_sw128(smem_u32(smem + kKvOffDo + slot * kTileBytes), kHalfBytes, 1024);
                    const uint64_t dQh = umma_desc_sw128(smem_u32(smem + kKvOffQ + slot * kTileBytes), kHalfBytes, 1024);
                    const uint64_t dDs = umma_desc_sw128(ds, 16, 1024);
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)
                        mma_ts(tdV, tS + 64u * (u & 1) + 32u * (kq >> 1) + 8u * (kq & 1),
                               dDo + (uint64_t)((4 * h + kq) * 2048 / 16), kIdescTS, (u > 0 || kq > 0) ? 1u : 0u);
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)
                        mma_ss(tdK, dDs + (uint64_t)(kq * 32 / 16), dQh + (uint64_t)((4 * h + kq) * 2048 / 16),
                               kIdescTS, (u > 0 || kq > 0) ? 1u : 0u);
                    if (h == steps - 1) mma_commit(&bars->qd_empty[slot]);  // Q_b / dO_b read for the last time
                } else {
                    // dQ^T(u) = K^T dS^T(u): 16 keys per MMA, dS^T MN-major (64 query rows per 128-byte row).
                    if (u >= 1 && !mbar_wait(&bars->dq_free, (u - 1) & 1u, abort_flag, kTimeoutNs)) return false;
                    tc_fence_after();
                    const uint64_t dDs = umma_desc_sw128(ds, 8192, 1024);
#pragma unroll
                    for (int kq = 0; kq < 8; ++kq)
                        mma_ss(tdQ, dKt + (uint64_t)(kq * 2048 / 16), dDs + (uint64_t)(kq * 2048 / 16), kIdescDQ,
                               kq > 0 ? 1u : 0u);
                    mma_commit(&bars->dq_full);
                }
                return true;
            };
            for (int32_t u = 0; ok && u < U; ++u) {
                ok = first(u);
                if (ok && u >= 1) ok = second(u - 1);
            }
            if (ok) ok = second(U - 1);
            if (ok) mma_commit(&bars->acc_done);
            else *abort_flag = 1;
            uint64_t* dr = &bars->drain[isA ? 0 : 1];
            mma_commit(dr);
            volatile int never = 0;
            mbar_wait(dr, 0, &never, kTimeoutNs);
        }
    } else if (warp >= kKvDqWarp0) {
        // ------------------------------------------------ dQ out: one thread per head-dim index
        // dQ^T(u) in TMEM: lane = head-dim index (this warp's quadrant), column = query row of the step.
        // Two warps per quadrant take 32 columns each, free the buffer for dQ^T(u + 1), then add row r of
        // the step (block lo + u / steps, row 64h + r) into dq: each reduction instruction covers 128
        // contiguous bytes (32 head-dim values of one query row); rows past the block are predicated off.
        const int quad = warp & 3, cpart = (warp - kKvDqWarp0) >> 2;
        const int dd = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        bool ok = true;
        for (int32_t u = 0; !skip && ok && u < U; ++u) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->dq_full, u & 1u, abort_flag, kTimeoutNs))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t x[32];
            tmem_ld32(tdQ + lane_off + 32u * cpart, x);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dq_free);
            const int32_t b = lo + u / steps;
            const int rbase = 64 * (u % steps) + 32 * cpart;
            const int valid = R - rbase;  // rows of these 32 inside the block
            if (valid <= 0) continue;
            if (G == 8 || G == 4 || G == 2 || G == 1) {
                float* row0 = dq + (((int64_t)m.block * b + rbase / G) * m.hq + (int64_t)g * G) * 128 + dd;
                const int64_t qs = (int64_t)m.hq * 128;
                if (G == 8) dq_add_rows<8>(row0, qs, x, valid);
                else if (G == 4) dq_add_rows<4>(row0, qs, x, valid);
                else if (G == 2) dq_add_rows<2>(row0, qs, x, valid);
                else dq_add_rows<1>(row0, qs, x, valid);
            } else {
                // Any other group size: walk the rows with a running (query, head) position.
                int i = rbase / G, hl = rbase - i * G;
                float* ptr = dq + (((int64_t)m.block * b + i) * m.hq + (int64_t)g * G + hl) * 128 + dd;
                const int64_t wrap = (int64_t)(m.hq - G + 1) * 128;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    red_add_f32_if(ptr, __uint_as_float(x[j]), j < valid);
                    const bool next_query = ++hl == G;
                    hl = next_query ? 0 : hl;
                    ptr += next_query ? wrap : 128;
                }
            }
        }
        if (!ok) *abort_flag = 1;
    } else if (!skip) {
        // ------------------------------------------------ one thread per (key kr, 32 query rows of a step)
        // Warps w and w+4 share key rows 32 (w % 4) .. (their TMEM lane quadrant) and take the step's query
        // rows 0-31 / 32-63: two warps per SM sub-partition keep the MUFU unit busy.
        const int quad = warp & 3, half = warp >> 2;
        const int kr = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float c = m.scale * kLog2e;
        const float sc = m.scale;
        bool ok = true;
        bool kvis = false;
        for (int32_t u = 0; u < U; ++u) {
            const int32_t p = u / steps, h = u % steps;
            if (h == 0) {
                const int32_t b = lo + p;
                kvis = self ? kr < nk : key0 + kr < (int64_t)__ldg(anchors + b);
            }
            // S^T(u) ready; the row constants of the slot landed with Q_b (waited here too, for visibility).
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[u & 1], (u >> 1) & 1u, abort_flag, kTimeoutNs) &&
                                             mbar_wait(&bars->qd_full[p & 1], (p >> 1) & 1u, abort_flag,
                                                       kTimeoutNs))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float* L2s = rows + (p & 1) * 256;  // -LSE log2 e per row
            const float* Ds = L2s + 128;               // -scale D per row
            const uint32_t col = 64u * (u & 1) + 32u * half;  // this warp's 32 query rows of the step
            uint32_t sv[32], pv[32];
            tmem_ld32(tS + lane_off + col, sv);
            tmem_ld32(tdP + lane_off + 32u * half, pv);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dp_read);  // dP^T(u + 1) may overwrite it now
            // P = 2^(s c - LSE log2 e), dS = P (scale dP - scale D), two rows per packed f32x2 operation.
            uint32_t pk[16], dk2[16];
            const int rb = 64 * h + 32 * half;
            if (kvis && rb + 32 <= R) {
                const uint64_t* L2v = reinterpret_cast<const uint64_t*>(L2s + rb);
                const uint64_t* Dv = reinterpret_cast<const uint64_t*>(Ds + rb);
                const uint64_t c2 = f2_pack(c, c), sc2 = f2_pack(sc, sc);
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    float t0, t1, d0, d1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * x]), __uint_as_float(sv[2 * x + 1])), c2, L2v[x]),
                              t0, t1);
                    const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
                    const uint64_t q2 =
                        f2_fma(f2_pack(__uint_as_float(pv[2 * x]), __uint_as_float(pv[2 * x + 1])), sc2, Dv[x]);
                    f2_unpack(f2_mul(f2_pack(p0, p1), q2), d0, d1);
                    __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);  // .x (low half) = even row
                    __nv_bfloat162 hd = __floats2bfloat162_rn(d0, d1);
                    pk[x] = *reinterpret_cast<uint32_t*>(&hp);
                    dk2[x] = *reinterpret_cast<uint32_t*>(&hd);
                }
            } else {
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int r0 = rb + 2 * x, r1 = r0 + 1;
                    const bool v0 = kvis && r0 < R, v1 = kvis && r1 < R;
                    const float p0 = v0 ? ex2_approx(fmaf(__uint_as_float(sv[2 * x]), c, L2s[r0])) : 0.f;
                    const float p1 = v1 ? ex2_approx(fmaf(__uint_as_float(sv[2 * x + 1]), c, L2s[r1])) : 0.f;
                    const float d0 = v0 ? p0 * fmaf(__uint_as_float(pv[2 * x]), sc, Ds[r0]) : 0.f;
                    const float d1 = v1 ? p1 * fmaf(__uint_as_float(pv[2 * x + 1]), sc, Ds[r1]) : 0.f;
                    __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
                    __nv_bfloat162 hd = __floats2bfloat162_rn(d0, d1);
                    pk[x] = *reinterpret_cast<uint32_t*>(&hp);
                    dk2[x] = *reinterpret_cast<uint32_t*>(&hd);
                }
            }
            // P^T over the first 16 of this warp's 32 columns of S^T(u) (read above by this warp alone);
            // dS^T into the key's 128-byte row of the step's shared buffer: query rows 32 half .. + 31 are
            // 16-byte groups 4 half .. 4 half + 3, XOR-swizzled by kr % 8 (the 128-byte swizzle).
            tmem_st16(tS + lane_off + col, pk);
            uint8_t* dsrow = smem + kKvOffDs + (u & 1) * kDsBytes + kr * 128;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4*>(dsrow + (((4 * half + q4) ^ (kr & 7)) << 4)) =
                    make_uint4(dk2[4 * q4], dk2[4 * q4 + 1], dk2[4 * q4 + 2], dk2[4 * q4 + 3]);
            tmem_wait_st();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // dS^T visible to the tensor core
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[u & 1]);
        }
        // Epilogue: dV and dK of this key, fp32, overwritten (zero if no block sees the tile).
        if (ok && np > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(&bars->acc_done, 0, abort_flag, kTimeoutNs)))
            ok = false;
        if (ok) {
            tc_fence_after();
            // Stage the tile's dV and dK rows in shared memory (the Q_b / dO_b slots, free now that every
            // MMA is complete): 16-byte groups of key kr at group index g4 ^ (kr % 32), so that the 32 rows a
            // warp writes at once fall in different banks. Then every warp stores whole 512-byte rows: a
            // thread per key writing its own row touched 32 rows' sectors per store instruction.
            float4* stv = reinterpret_cast<float4*>(smem + kKvOffQ);  // [128 keys][32 groups] dV
            float4* stk = stv + 128 * 32;                             // [128 keys][32 groups] dK
#pragma unroll 1
            for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
                uint32_t xv[32], xk[32];
                if (np > 0) {
                    tmem_ld32(tdV + lane_off + cc * 32, xv);
                    tmem_ld32(tdK + lane_off + cc * 32, xk);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) xv[e] = xk[e] = 0u;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int at = kr * 32 + ((cc * 8 + e) ^ (kr & 31));
                    stv[at] = make_float4(__uint_as_float(xv[4 * e]), __uint_as_float(xv[4 * e + 1]),
                                          __uint_as_float(xv[4 * e + 2]), __uint_as_float(xv[4 * e + 3]));
                    stk[at] = make_float4(__uint_as_float(xk[4 * e]), __uint_as_float(xk[4 * e + 1]),
                                          __uint_as_float(xk[4 * e + 2]), __uint_as_float(xk[4 * e + 3]));
                }
            }
            // Every elementwise warp staged its rows (bounded wait; a warp that gave up earlier never arrives).
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->epi_staged);
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->epi_staged, 0, abort_flag, kTimeoutNs));
            if (ok) {
                float* dv_t = (self ? dvb : dv) + (krow * m.hkv + g) * (int64_t)m.d;
                float* dk_t = (self ? dkb : dk) + (krow * m.hkv + g) * (int64_t)m.d;
                const int64_t rstride = (int64_t)m.hkv * m.d;
#pragma unroll 2
                for (int k = warp; k < nk; k += 8) {
                    const int at = k * 32 + (lane ^ (k & 31));
                    *reinterpret_cast<float4*>(dv_t + k * rstride + 4 * lane) = stv[at];
                    *reinterpret_cast<float4*>(dk_t + k * rstride + 4 * lane) = stk[at];
                }
            }
        }
        if (!ok) *abort_flag = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && bars->abort_flag) raise_status(status, SPLITKV_DEV_TIMEOUT);
    if (warp == kKvMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

bool bwd_tc_supported(const Meta& m) {
    return m.dtype == SPLITKV_BF16 && m.d == 128 && m.rows_item <= 128 && m.group >= 1 && m.total_keys < INT32_MAX &&
           m.n_queries < INT32_MAX;
}

size_t bwd_tc_workspace(const Meta& m) { return 2 * sizeof(float) * (size_t)m.n_queries * m.hq + 256; }

cudaError_t launch_bwd_tc(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                          const void* o, const float* lse, const void* dout, const int32_t* anchors, float* dq,
                          float* dk, float* dv, float* dkb, float* dvb, int32_t* status, void* ws, cudaStream_t st) {
    const size_t nrows = (size_t)m.n_queries * m.hq;
    cudaError_t e;
    if (m.n_queries == 0) {
        // No query (the query-side buffers are empty): every key gradient is zero.
        e = cudaMemsetAsync(dk, 0, sizeof(float) * (size_t)m.total_keys * m.hkv * m.d, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, sizeof(float) * (size_t)m.total_keys * m.hkv * m.d, st);
        return note_error(e, "cudaMemsetAsync(dk, dv)");
    }
    e = cudaMemsetAsync(dq, 0, sizeof(float) * nrows * m.d, st);
    if (e != cudaSuccess) return note_error(e, "cudaMemsetAsync(dq)");
    float* l2 = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
    float* dvec = l2 + nrows;
    rows_kernel<__nv_bfloat16><<<(unsigned)((nrows * 32 + 255) / 256), 256, 0, st>>>(
        m, (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, lse, l2, dvec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return note_error(e, "launch rows_kernel");
    CUtensorMap tq, tdo, tk, tv, tkb, tvb;
    if (!make_bf16_map(&tq, q, m.n_queries, m.hq, m.d, m.group, m.block) ||
        !make_bf16_map(&tdo, dout, m.n_queries, m.hq, m.d, m.group, m.block) ||
        !make_bf16_map(&tk, k, m.total_keys, m.hkv, m.d, 1, kKeys) ||
        !make_bf16_map(&tv, v, m.total_keys, m.hkv, m.d, 1, kKeys) ||
        !make_bf16_map(&tkb, kb, m.n_queries, m.hkv, m.d, 1, kKeys) ||
        !make_bf16_map(&tvb, vb, m.n_queries, m.hkv, m.d, 1, kKeys))
        return cudaErrorInvalidValue;
    int32_t tiles_max = 0;
    for (int s = 0; s < m.batch; ++s) {
        const int32_t t = (int32_t)((m.seq_len[s] + kKeys - 1) / kKeys);
        tiles_max = t > tiles_max ? t : tiles_max;
    }
    e = cudaFuncSetAttribute(bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmemBytes);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(bwd_tc_kernel)");
    const int64_t kv_grid = (int64_t)tiles_max * m.batch * m.hkv + m.n_blocks * m.hkv;
    if (kv_grid > 0x7fffffff) return note_error(cudaErrorInvalidConfiguration, "bwd_tc_kernel: grid too large");
    bwd_tc_kernel<<<(unsigned)kv_grid, kKvThreads, kKvSmemBytes, st>>>(m, tq, tdo, tk, tv, tkb, tvb, tiles_max, anchors,
                                                                       l2, dvec, dq, dk, dv, dkb, dvb, status);
    return note_error(cudaGetLastError(), "launch bwd_tc_kernel");
}

}  // namespace splitkv
