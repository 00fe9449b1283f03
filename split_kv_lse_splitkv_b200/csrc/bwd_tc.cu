// Backward on the 5th-generation tensor cores (sm_100a): TMA -> tcgen05.mma -> TMEM.
//
// Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, title and Abstract: the
// method trains diffusion drafters, so gradients flow back through the same exact attention. With
// P = exp(s - LSE) recomputed from the stored natural-log LSE, D = rowsum(dO * O) and
// dS = P (dP - D), dP = dO V^T:
//   dV = P^T dO,  dK = scale dS^T Q   (key-stationary kernel: one CTA per 128-key tile)
//   dQ = scale dS K                   (query-stationary kernel: the forward's LPT queues)
// Each kernel recomputes S and dP for its (key tile, block) pairs, so neither needs atomics for
// the tensors it owns; dQ of an item (one block against one chunk) is added once, with vector
// atomics, into the zeroed dq.
//
// Key-stationary kernel (bwd_kv_kernel), per pair (key tile, block b seeing it):
//   S^T = K Q_b^T and dP^T = V dO_b^T (M = 128 keys, N = 128 query rows, K = d) into TMEM; two
//   threads per key (query rows 0-63 / 64-127, in two warps of the same SM sub-partition, so that
//   the MUFU unit has two warps to interleave) form P^T and dS^T in bf16 over the first 32 columns
//   of their half of each (two rows per column); dV += P^T dO_b and dK += dS^T Q_b with P^T / dS^T
//   as the TMEM operand and Q_b / dO_b read MN-major from shared memory, each query half as soon as
//   it is written. Two issuing threads, one per accumulator pair (S^T then dV, dP^T then dK): one
//   thread gets one tcgen05.mma per ~120 cycles, two interleave; each issuer's MMAs execute in its
//   issue order, so the next pair's S^T (dP^T) overwrites P^T (dS^T) only after dV (dK) has read it.
//   (Measured on the backward of train_4x16k: 1085 -> 1042 us for two threads per key, and on
//   train_4x64k 13.65 -> 12.98 ms for two issuers here and in the dQ kernel.)
// Query-stationary kernel (bwd_q_kernel), per item key tile: S = Q K^T and dP = dO V^T into TMEM,
//   from two issuing threads; two threads per query row (keys 0-63 / 64-127, two warps per SM
//   sub-partition) form dS in bf16 over the first 32 columns of their half of S; dQ += dS K, each key
//   half as soon as it is written. (Measured: the backward of train_4x64k 14.10 -> 13.62 ms against
//   one thread per row.)
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

// Per-row constants of one (block j, kv head g) query tile, rows r = i*G + hl contiguous:
// l2 = LSE * log2 e and dvec = rowsum(dO * O). One warp per row.
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
        l2[q] = lse[orow] * kLog2e;
        dvec[q] = acc;
    }
}

// ------------------------------------------------------------------ key-stationary: dK, dV
constexpr int kKvThreads = 352;  // warps 0-7: elementwise (key row x query half); warp 8: TMA producer;
                                 // warps 9, 10: MMA issuers (S^T then dV; dP^T then dK)
constexpr int kKvLoadWarp = 8, kKvMmaWarp = 9, kKvMma2Warp = 10;
constexpr int kKvOffK = 0;
constexpr int kKvOffV = kTileBytes;
constexpr int kKvOffQ = 2 * kTileBytes;     // Q_b[2]
constexpr int kKvOffDo = 4 * kTileBytes;    // dO_b[2]
constexpr int kKvOffRows = 6 * kTileBytes;  // float [2 slots][l2, dvec][128]
constexpr int kKvOffBar = kKvOffRows + 2 * 2 * 128 * 4;

struct KvBars {
    uint64_t kv_full;
    uint64_t qd_full[2], qd_empty[2];  // Q_b, dO_b, rows of pair p in slot p % 2
    uint64_t s_full[2];                // S^T, dP^T of step u (parity u % 2) complete (one commit per issuer)
    uint64_t p_full[2];                // P^T, dS^T of step u written (8 elementwise warps)
    uint64_t acc_done;                 // every MMA complete: dV, dK final
    uint64_t epi_staged;               // all 8 elementwise warps staged their dV / dK rows
    uint64_t drain[2];
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

constexpr int kKvSmemBytes = kKvOffBar + (int)sizeof(KvBars) + 1024;

// Unit u: context key tile (t, sample s, kv head g) with g fastest and t slowest, so that the
// costliest tiles (small t: seen by the most blocks) start first; then the self tiles (block j,
// kv head g): the block's own 16 keys.
__global__ void __launch_bounds__(kKvThreads, 1)
    bwd_kv_kernel(const __grid_constant__ Meta m, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmDo, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                  const __grid_constant__ CUtensorMap tmVb, int32_t tiles_max, const int32_t* __restrict__ anchors,
                  const float* __restrict__ l2, const float* __restrict__ dvec, float* __restrict__ dk,
                  float* __restrict__ dv, float* __restrict__ dkb, float* __restrict__ dvb,
                  int32_t* __restrict__ status) {
    const int64_t n_ctx = (int64_t)tiles_max * m.batch * m.hkv;
    const int64_t u = blockIdx.x;
    const bool self = u >= n_ctx;
    int s = 0, g, lo, hi, nk;
    int64_t key0 = 0, krow;  // first key of the tile within its sample; its row in k/v (or kb/vb)
    if (!self) {
        g = (int)(u % m.hkv);
        const int64_t rest = u / m.hkv;
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
    } else {
        const int64_t sid = u - n_ctx;
        const int32_t j = (int32_t)(sid / m.hkv);
        g = (int)(sid % m.hkv);
        lo = j;
        hi = j + 1;
        nk = m.block;
        krow = (int64_t)m.block * j;
    }
    const int32_t np = hi - lo;
    // Each pair runs as steps of 64 query rows (two for a block of more than 64 rows), so that S^T and
    // dP^T are double-buffered in TMEM and the tensor core computes step u while the elementwise warps
    // work on step u - 1.
    const int32_t steps = m.rows > 64 ? 2 : 1;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->s_full[b], 2);
            mbar_init(&bars->p_full[b], 8);
        }
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
    const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384;
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
                uint8_t* dq = smem + kKvOffQ + slot * kTileBytes;
                uint8_t* ddo = smem + kKvOffDo + slot * kTileBytes;
                tma_load_3d(dq, &tmQ, &bars->qd_full[slot], 0, g * G, m.block * b);
                tma_load_3d(dq + kHalfBytes, &tmQ, &bars->qd_full[slot], 64, g * G, m.block * b);
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
        // Two issuers, each with its own pair of accumulators, so that the tensor core interleaves two
        // instruction streams (one thread issues one tcgen05.mma per ~120 cycles): A: S^T = K Q_b^T, then
        // dV += P^T dO_b reading P^T from S^T's columns; B: dP^T = V dO_b^T, then dK += dS^T Q_b. Each
        // issuer's MMAs execute in its issue order, so the next pair's S^T (dP^T) overwrites P^T (dS^T)
        // only after dV (dK) has read it.
        const bool isA = warp == kKvMmaWarp;
        if (!skip && lane == 0 && np > 0) {
            bool ok = mbar_wait(&bars->kv_full, 0, abort_flag, kTimeoutNs);
            tc_fence_after();
            const uint64_t dA1 = umma_desc_sw128(smem_u32(smem + (isA ? kKvOffK : kKvOffV)), 16, 1024);
            const uint32_t t1 = isA ? tS : tdP, t2 = isA ? tdV : tdK;
            // First GEMM of step u: S^T(u) = K Q_h^T  /  dP^T(u) = V dO_h^T into buffer u % 2 (64 columns),
            // B = the step's 64 query rows of Q_b / dO_b (K-major, rows 64h .. of the slot's tile).
            auto first = [&](int32_t u) -> bool {
                const int32_t p = u / steps, h = u % steps;
                const int slot = p & 1;
                if (h == 0 && !mbar_wait(&bars->qd_full[slot], (p >> 1) & 1u, abort_flag, kTimeoutNs)) return false;
                tc_fence_after();
                const uint32_t src = smem_u32(smem + (isA ? kKvOffQ : kKvOffDo) + slot * kTileBytes) + 8192u * h;
                const uint64_t dB1 = umma_desc_sw128(src, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) / 16);
                    mma_ss(t1 + 64u * (u & 1), dA1 + off, dB1 + off, kIdescSS64, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[u & 1]);
                return true;
            };
            // Second GEMM of step u once its P^T / dS^T are written: dV += P^T(u) dO_h  /  dK += dS^T(u) Q_h,
            // 16 query rows per MMA: rows 32w' + 16i of the step are bf16 pairs at columns 32w' + 8i of the
            // buffer (each elementwise warp half w' writes its 32 rows into its own 32 columns).
            auto second = [&](int32_t u) -> bool {
                const int32_t p = u / steps, h = u % steps;
                const int slot = p & 1;
                if (!mbar_wait(&bars->p_full[u & 1], (u >> 1) & 1u, abort_flag, kTimeoutNs)) return false;
                tc_fence_after();
                const uint32_t src = smem_u32(smem + (isA ? kKvOffDo : kKvOffQ) + slot * kTileBytes);
                const uint64_t dB2 = umma_desc_sw128(src, kHalfBytes, 1024);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)
                    mma_ts(t2, t1 + 64u * (u & 1) + 32u * (kq >> 1) + 8u * (kq & 1),
                           dB2 + (uint64_t)((4 * h + kq) * 2048 / 16), kIdescTS, (u > 0 || kq > 0) ? 1u : 0u);
                if (h == steps - 1) mma_commit(&bars->qd_empty[slot]);  // pair p's Q_b / dO_b read for the last time
                return true;
            };
            // S^T(u) / dP^T(u) run while the elementwise warps work on step u - 1: the buffer u % 2 they
            // overwrite held step u - 2, whose second GEMM this thread issued before (its MMAs run in order).
            const int32_t U = np * steps;
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
    } else if (!skip) {
        // ------------------------------------------------ one thread per (key kr, 32 query rows of a step)
        // Warps w and w+4 share key rows 32 (w % 4) .. (their TMEM lane quadrant) and take the step's query
        // rows 0-31 / 32-63: two warps per SM sub-partition keep the MUFU unit busy.
        const int quad = warp & 3, half = warp >> 2;
        const int kr = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float c = m.scale * kLog2e;
        bool ok = true;
        bool kvis = false;
        for (int32_t u = 0; u < np * steps; ++u) {
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
            const float* L2s = rows + (p & 1) * 256;
            const float* Ds = L2s + 128;
            const uint32_t col = 64u * (u & 1) + 32u * half;  // this warp's 32 query rows of the step
            uint32_t sv[32], pv[32];
            tmem_ld32(tS + lane_off + col, sv);
            tmem_ld32(tdP + lane_off + col, pv);
            tmem_wait_ld();
            uint32_t pk[16], dk2[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const int r0 = 64 * h + 32 * half + 2 * x, r1 = r0 + 1;
                const bool v0 = kvis && r0 < R, v1 = kvis && r1 < R;
                const float p0 = v0 ? ex2_approx(fmaf(__uint_as_float(sv[2 * x]), c, -L2s[r0])) : 0.f;
                const float p1 = v1 ? ex2_approx(fmaf(__uint_as_float(sv[2 * x + 1]), c, -L2s[r1])) : 0.f;
                const float d0 = v0 ? p0 * (__uint_as_float(pv[2 * x]) - Ds[r0]) : 0.f;
                const float d1 = v1 ? p1 * (__uint_as_float(pv[2 * x + 1]) - Ds[r1]) : 0.f;
                __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);  // .x (low half) = even row
                __nv_bfloat162 hd = __floats2bfloat162_rn(d0, d1);
                pk[x] = *reinterpret_cast<uint32_t*>(&hp);
                dk2[x] = *reinterpret_cast<uint32_t*>(&hd);
            }
            // The first 16 of this warp's 32 columns: read above by this warp alone.
            tmem_st16(tS + lane_off + col, pk);
            tmem_st16(tdP + lane_off + col, dk2);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[u & 1]);
        }
        // Epilogue: dV and scale * dK of this key, fp32, overwritten (zero if no block sees the tile).
        if (ok && np > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(&bars->acc_done, 0, abort_flag, kTimeoutNs)))
            ok = false;
        if (ok) {
            tc_fence_after();
            // Stage the tile's dV and scale * dK rows in shared memory (the Q_b / dO_b slots, free now that
            // every MMA is complete): 16-byte groups of key kr at group index g4 ^ (kr % 32), so that the 32
            // rows a warp writes at once fall in different banks. Then every warp stores whole 512-byte rows:
            // a thread per key writing its own row touched 32 rows' sectors per store instruction.
            float4* stv = reinterpret_cast<float4*>(smem + kKvOffQ);  // [128 keys][32 groups] dV
            float4* stk = stv + 128 * 32;                             // [128 keys][32 groups] scale * dK
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
                    stk[at] = make_float4(__uint_as_float(xk[4 * e]) * m.scale, __uint_as_float(xk[4 * e + 1]) * m.scale,
                                          __uint_as_float(xk[4 * e + 2]) * m.scale,
                                          __uint_as_float(xk[4 * e + 3]) * m.scale);
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

// ------------------------------------------------------------------ query-stationary: dQ
constexpr int kQThreads = 352;  // warps 0-7: elementwise (query row x key half); warp 8: TMA producer;
                                // warps 9, 10: MMA issuers (S then dQ; dP)
constexpr int kQLoadWarp = 8, kQMmaWarp = 9, kQMma2Warp = 10;
constexpr int kQOffQ = 0;                   // Q of the current item
constexpr int kQOffDo = kTileBytes;         // dO of the current item
constexpr int kQOffK = 2 * kTileBytes;      // K[2], by key tile parity
constexpr int kQOffV = 4 * kTileBytes;      // V[2]
constexpr int kQOffBar = 6 * kTileBytes;

struct QBars {
    uint64_t qd_full, qd_empty;      // Q, dO of item i landed / every S, dP of item i complete
    uint64_t kv_full[2], kv_empty[2];
    uint64_t s_full[2];              // S, dP of step u (parity u % 2) complete (one commit per issuer)
    uint64_t p_full[2];              // dS of step u written (8 elementwise warps)
    uint64_t dq_ready, dq_free;      // last dQ MMA of item i complete / dQ read by the epilogue
    uint64_t drain[2];
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t status0;
};

constexpr int kQSmemBytes = kQOffBar + (int)sizeof(QBars) + 1024;

struct QItem {
    int64_t id;
    int32_t s, c, g, j;       // j: first block of the query tile
    int32_t nbt;              // blocks in the tile
    int32_t nvis, ntiles, self_item;  // nvis: keys the tile's last (largest-anchor) block sees
};

// The CTA's items: its queue (positions pos .. end-1), then self items blockIdx.x, blockIdx.x +
// gridDim.x, ... (block j, kv head g against the block's own keys). Items the block cannot see
// are skipped; an invalid queue entry raises SPLITKV_DEV_BAD_PLAN.
__device__ __forceinline__ bool q_next(const Meta& m, const int32_t* __restrict__ anchors,
                                       const int32_t* __restrict__ item_id, const int32_t* __restrict__ queue_items,
                                       int32_t& pos, int32_t end, int64_t& self_pos, QItem& t, int32_t* status) {
    while (pos < end) {
        const int64_t id = __ldg(item_id + __ldg(queue_items + pos));
        ++pos;
        if (id < 0 || id >= m.n_items) {
            raise_status(status, SPLITKV_DEV_BAD_PLAN);
            continue;
        }
        const Item it = decode_item(m, id);
        t.id = id;
        t.s = it.s;
        t.c = it.c;
        t.g = it.g;
        t.j = it.j;
        t.nbt = it.nbt;
        t.nvis = visible_in_chunk(m, it.s, it.c, __ldg(anchors + it.j + it.nbt - 1));
        t.ntiles = (t.nvis + kKeys - 1) / kKeys;
        t.self_item = 0;
        if (t.ntiles > 0) return true;
    }
    if (self_pos < m.n_blocks * m.hkv) {
        const int64_t sid = self_pos;
        self_pos += gridDim.x;
        t.id = m.n_items + sid;
        t.j = (int32_t)(sid / m.hkv);
        t.g = (int32_t)(sid % m.hkv);
        t.s = sample_of_block(m, t.j);
        t.c = 0;
        t.nbt = 1;
        t.nvis = m.block;
        t.ntiles = 1;
        t.self_item = 1;
        return true;
    }
    return false;
}

__global__ void __launch_bounds__(kQThreads, 1)
    bwd_q_kernel(const __grid_constant__ Meta m, const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmDo, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                 const __grid_constant__ CUtensorMap tmVb, const int32_t* __restrict__ anchors,
                 const int32_t* __restrict__ item_id, const int32_t* __restrict__ queue_off,
                 const int32_t* __restrict__ queue_items, const float* __restrict__ l2,
                 const float* __restrict__ dvec, float* __restrict__ dq, int32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    QBars* bars = reinterpret_cast<QBars*>(smem + kQOffBar);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = m.group, RB = m.rows;  // rows of one block
    const int32_t q0 = queue_off[blockIdx.x], q1 = queue_off[blockIdx.x + 1];

    if (threadIdx.x == 0) {
        mbar_init(&bars->qd_full, 1);
        mbar_init(&bars->qd_empty, 2);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->kv_full[b], 1);
            mbar_init(&bars->kv_empty[b], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->s_full[b], 2);
            mbar_init(&bars->p_full[b], 8);
        }
        mbar_init(&bars->dq_ready, 1);
        mbar_init(&bars->dq_free, 256);
        mbar_init(&bars->drain[0], 1);
        mbar_init(&bars->drain[1], 1);
        bars->abort_flag = 0;
        bars->status0 = status_bad(status) ? 1 : 0;
        fence_barrier_init();
    }
    // Query rows beyond the tile's are never loaded: keep Q and dO finite (zero).
    if (m.rows_item < 128)
        for (int i = threadIdx.x; i < 2 * kTileBytes / 16; i += kQThreads)
            reinterpret_cast<uint4*>(smem + kQOffQ)[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == kQMmaWarp) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;
    const bool skip = bars->status0 != 0;

    if (warp == kQLoadWarp) {
        if (!skip && lane == 0) {
            const uint32_t q_bytes = 2u * 64u * (uint32_t)G * (uint32_t)(m.block * m.pack) * 2u;
            int32_t pos = q0;
            int64_t self_pos = blockIdx.x;
            QItem t;
            uint32_t i = 0, n = 0, q_inflight = 0, kv_inflight = 0;
            bool ok = true;
            while (ok && q_next(m, anchors, item_id, queue_items, pos, q1, self_pos, t, status)) {
                if (i >= 1 && !mbar_wait(&bars->qd_empty, (i - 1) & 1u, abort_flag, kTimeoutNs)) break;
                mbar_arrive_expect_tx(&bars->qd_full, 2 * q_bytes);
                tma_load_3d(smem + kQOffQ, &tmQ, &bars->qd_full, 0, t.g * G, m.block * t.j);
                tma_load_3d(smem + kQOffQ + kHalfBytes, &tmQ, &bars->qd_full, 64, t.g * G, m.block * t.j);
                tma_load_3d(smem + kQOffDo, &tmDo, &bars->qd_full, 0, t.g * G, m.block * t.j);
                tma_load_3d(smem + kQOffDo + kHalfBytes, &tmDo, &bars->qd_full, 64, t.g * G, m.block * t.j);
                ++i;
                q_inflight = 1;
                const CUtensorMap* mk = t.self_item ? &tmKb : &tmK;
                const CUtensorMap* mv = t.self_item ? &tmVb : &tmV;
                for (int32_t tt = 0; tt < t.ntiles; ++tt, ++n) {
                    const int b = n & 1;
                    if (!mbar_wait(&bars->kv_empty[b], ((n >> 1) & 1u) ^ 1u, abort_flag, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    const int32_t row = t.self_item ? m.block * t.j
                                                    : (int32_t)(m.key_off[t.s] + (int64_t)t.c * m.chunk +
                                                                (int64_t)tt * kKeys);
                    mbar_arrive_expect_tx(&bars->kv_full[b], 2 * kTileBytes);
                    uint8_t* kd = smem + kQOffK + b * kTileBytes;
                    uint8_t* vd = smem + kQOffV + b * kTileBytes;
                    tma_load_3d(kd, mk, &bars->kv_full[b], 0, t.g, row);
                    tma_load_3d(kd + kHalfBytes, mk, &bars->kv_full[b], 64, t.g, row);
                    tma_load_3d(vd, mv, &bars->kv_full[b], 0, t.g, row);
                    tma_load_3d(vd + kHalfBytes, mv, &bars->kv_full[b], 64, t.g, row);
                    kv_inflight = 1;
                }
            }
            // Drain: the most recent copies into every buffer have landed before the CTA exits.
            volatile int never = 0;
            if (q_inflight) mbar_wait(&bars->qd_full, (i - 1) & 1u, &never, kTimeoutNs);
            if (kv_inflight)
                for (uint32_t x = (n > 2 ? n - 2 : 0); x < n; ++x)
                    mbar_wait(&bars->kv_full[x & 1], (x >> 1) & 1u, &never, kTimeoutNs);
        }
    } else if (warp == kQMmaWarp || warp == kQMma2Warp) {
        // Two issuers, so that the tensor core interleaves two instruction streams. Each key tile runs as
        // two steps of 64 keys (u = 2n + kh), with S and dP double-buffered by step parity (64 columns
        // each): A: S(u) = Q K_kh^T, then dQ += dS(u-1) K_kh' of the previous step (reading dS from its S
        // buffer; this thread's MMAs run in order, so S(u+1) overwrites it only after); B: dP(u) = dO V_kh^T
        // once the elementwise pass has read dP(u-2) out of the same buffer.
        const bool isA = warp == kQMmaWarp;
        if (!skip && lane == 0) {
            const uint64_t dA1 = umma_desc_sw128(smem_u32(smem + (isA ? kQOffQ : kQOffDo)), 16, 1024);
            int32_t pos = q0;
            int64_t self_pos = blockIdx.x;
            QItem t;
            uint32_t i = 0, n = 0, u = 0;
            bool ok = true;
            // The previous step, whose dQ MMAs issuer A issues after the next step's S.
            uint32_t pu = 0, pn = 0, pi = 0;
            int pkh = 0;
            bool have_prev = false, p_first = false, p_last = false;
            auto dq_step = [&]() -> bool {
                if (!mbar_wait(&bars->p_full[pu & 1], (pu >> 1) & 1u, abort_flag, kTimeoutNs)) return false;
                // The first dQ MMA of item i overwrites dQ once the epilogue has read item i-1.
                if (p_first && pi >= 1 && !mbar_wait(&bars->dq_free, (pi - 1) & 1u, abort_flag, kTimeoutNs))
                    return false;
                tc_fence_after();
                const uint64_t dKmn = umma_desc_sw128(smem_u32(smem + kQOffK + (pn & 1) * kTileBytes), kHalfBytes, 1024);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)  // keys 32w' + 16i of the step: dS pairs at columns 32w' + 8i
                    mma_ts(tdQ, tS + 64u * (pu & 1) + 32u * (kq >> 1) + 8u * (kq & 1),
                           dKmn + (uint64_t)((4 * pkh + kq) * 2048 / 16), kIdescTS, (!p_first || kq > 0) ? 1u : 0u);
                if (pkh == 1) mma_commit(&bars->kv_empty[pn & 1]);  // K(n) read for the last time
                if (p_last) mma_commit(&bars->dq_ready);
                return true;
            };
            while (ok && q_next(m, anchors, item_id, queue_items, pos, q1, self_pos, t, status)) {
                if (!mbar_wait(&bars->qd_full, i & 1u, abort_flag, kTimeoutNs)) { ok = false; break; }
                for (int32_t tt = 0; ok && tt < t.ntiles; ++tt, ++n) {
                    const int b = n & 1;
                    if (!mbar_wait(&bars->kv_full[b], (n >> 1) & 1u, abort_flag, kTimeoutNs)) { ok = false; break; }
                    for (int kh = 0; kh < 2; ++kh, ++u) {
                        // B: dP(u) overwrites dP(u-2) once the elementwise pass has read it.
                        if (!isA && u >= 2 &&
                            !mbar_wait(&bars->p_full[u & 1], ((u >> 1) - 1) & 1u, abort_flag, kTimeoutNs)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t src = smem_u32(smem + (isA ? kQOffK : kQOffV) + b * kTileBytes) + 8192u * kh;
                        const uint64_t dB1 = umma_desc_sw128(src, 16, 1024);
                        const uint32_t t1 = (isA ? tS : tdP) + 64u * (u & 1);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {  // S = Q K_kh^T  /  dP = dO V_kh^T, 64 keys
                            const uint64_t off = (uint64_t)(((kk >> 2) * kHalfBytes + (kk & 3) * 32) / 16);
                            mma_ss(t1, dA1 + off, dB1 + off, kIdescSS64, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&bars->s_full[u & 1]);
                        const bool last_of_item = tt == t.ntiles - 1 && kh == 1;
                        if (last_of_item) mma_commit(&bars->qd_empty);  // Q, dO free once these complete
                        if (isA) {
                            if (have_prev && !dq_step()) { ok = false; break; }
                            pu = u;
                            pn = n;
                            pi = i;
                            pkh = kh;
                            p_first = tt == 0 && kh == 0;
                            p_last = last_of_item;
                            have_prev = true;
                        } else if (kh == 1) {
                            mma_commit(&bars->kv_empty[b]);  // V(n) read for the last time
                        }
                    }
                }
                ++i;
            }
            if (ok && isA && have_prev && !dq_step()) ok = false;
            if (!ok) *abort_flag = 1;
            uint64_t* dr = &bars->drain[isA ? 0 : 1];
            mma_commit(dr);
            volatile int never = 0;
            mbar_wait(dr, 0, &never, kTimeoutNs);
        }
    } else if (!skip) {
        // ------------------------------------------------ one thread per (query row r, key half)
        // Warps w and w+4 share rows 32 (w % 4) .. (their TMEM lane quadrant) and take key columns
        // 0-63 / 64-127: two warps per SM sub-partition keep the MUFU unit busy.
        const int quad = warp & 3, half = warp >> 2;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float c = m.scale * kLog2e;
        int32_t pos = q0;
        int64_t self_pos = blockIdx.x;
        QItem t;
        uint32_t i = 0, u = 0;
        bool ok = true;
        while (ok && q_next(m, anchors, item_id, queue_items, pos, q1, self_pos, t, status)) {
            // Row r belongs to block t.j + x of the tile; it sees that block's prefix of the chunk (a
            // self item: its own keys, rows of its block only).
            const int32_t x = r / RB;
            const bool live = x < t.nbt && (!t.self_item || x == 0);
            const int32_t row_nvis =
                !live ? 0 : t.self_item ? m.block : visible_in_chunk(m, t.s, t.c, __ldg(anchors + t.j + x));
            const int64_t rb = ((int64_t)(t.j + x) * m.hkv + t.g) * RB + r % RB;
            const float L2 = live ? l2[rb] : 0.f, Dr = live ? dvec[rb] : 0.f;
            for (int32_t tt = 0; ok && tt < t.ntiles; ++tt) {
                for (int kh = 0; kh < 2; ++kh, ++u) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[u & 1], (u >> 1) & 1u, abort_flag, kTimeoutNs))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int valid = row_nvis - tt * kKeys - 64 * kh - 32 * half;  // keys of my 32 this row sees
                    const uint32_t col = 64u * (u & 1) + 32u * half;
                    uint32_t sv[32], pv[32];
                    tmem_ld32(tS + lane_off + col, sv);
                    tmem_ld32(tdP + lane_off + col, pv);
                    tmem_wait_ld();
                    uint32_t dk2[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const int k0 = 2 * x;
                        const float p0 = k0 < valid ? ex2_approx(fmaf(__uint_as_float(sv[2 * x]), c, -L2)) : 0.f;
                        const float p1 =
                            k0 + 1 < valid ? ex2_approx(fmaf(__uint_as_float(sv[2 * x + 1]), c, -L2)) : 0.f;
                        const float d0 = k0 < valid ? p0 * (__uint_as_float(pv[2 * x]) - Dr) : 0.f;
                        const float d1 = k0 + 1 < valid ? p1 * (__uint_as_float(pv[2 * x + 1]) - Dr) : 0.f;
                        __nv_bfloat162 hd = __floats2bfloat162_rn(d0, d1);  // .x (low half) = even key
                        dk2[x] = *reinterpret_cast<uint32_t*>(&hd);
                    }
                    // The first 16 of this warp's 32 columns: read above by this warp alone.
                    tmem_st16(tS + lane_off + col, dk2);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->p_full[u & 1]);
                }
            }
            if (!ok) break;
            // Epilogue of item i: add scale * dQ into dq (zeroed before the launch).
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->dq_ready, i & 1u, abort_flag, kTimeoutNs))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int64_t orow = ((int64_t)m.block * t.j + r / G) * m.hq + (int64_t)t.g * G + r % G;
            float* dst = dq + orow * (int64_t)m.d;
#pragma unroll 1
            for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
                uint32_t xq[32];
                tmem_ld32(tdQ + lane_off + cc * 32, xq);
                tmem_wait_ld();
                if (cc == 2 * half + 1) {
                    tc_fence_before();
                    mbar_arrive(&bars->dq_free);
                }
                if (live) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        atomicAdd(reinterpret_cast<float4*>(dst + cc * 32 + e),
                                  make_float4(__uint_as_float(xq[e]) * m.scale, __uint_as_float(xq[e + 1]) * m.scale,
                                              __uint_as_float(xq[e + 2]) * m.scale,
                                              __uint_as_float(xq[e + 3]) * m.scale));
                }
            }
            ++i;
        }
        if (!ok) *abort_flag = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && bars->abort_flag) raise_status(status, SPLITKV_DEV_TIMEOUT);
    if (warp == kQMmaWarp) {
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
                          const void* o, const float* lse, const void* dout, const int32_t* anchors,
                          const int32_t* item_id, const int32_t* queue_off, const int32_t* queue_items,
                          int32_t n_workers, float* dq, float* dk, float* dv, float* dkb, float* dvb,
                          int32_t* status, void* ws, cudaStream_t st) {
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
    // Per-block Q/dO boxes for the key-stationary kernel, per-item (P blocks) boxes for the dQ kernel.
    CUtensorMap tq, tdo, tqi, tdoi, tk, tv, tkb, tvb;
    if (!make_bf16_map(&tq, q, m.n_queries, m.hq, m.d, m.group, m.block) ||
        !make_bf16_map(&tdo, dout, m.n_queries, m.hq, m.d, m.group, m.block) ||
        !make_bf16_map(&tqi, q, m.n_queries, m.hq, m.d, m.group, m.block * m.pack) ||
        !make_bf16_map(&tdoi, dout, m.n_queries, m.hq, m.d, m.group, m.block * m.pack) ||
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
    e = cudaFuncSetAttribute(bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmemBytes);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(bwd_kv_kernel)");
    e = cudaFuncSetAttribute(bwd_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(bwd_q_kernel)");
    const int64_t kv_grid = (int64_t)tiles_max * m.batch * m.hkv + m.n_blocks * m.hkv;
    if (kv_grid > 0x7fffffff) return note_error(cudaErrorInvalidConfiguration, "bwd_kv_kernel: grid too large");
    bwd_kv_kernel<<<(unsigned)kv_grid, kKvThreads, kKvSmemBytes, st>>>(m, tq, tdo, tk, tv, tkb, tvb, tiles_max, anchors,
                                                                       l2, dvec, dk, dv, dkb, dvb, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return note_error(e, "launch bwd_kv_kernel");
    bwd_q_kernel<<<(unsigned)n_workers, kQThreads, kQSmemBytes, st>>>(m, tqi, tdoi, tk, tv, tkb, tvb, anchors, item_id,
                                                                      queue_off, queue_items, l2, dvec, dq, status);
    return note_error(cudaGetLastError(), "launch bwd_q_kernel");
}

}  // namespace splitkv
