// Backward of the anchor-block cross-attention (Split-KV: Efficient Context Parallelism for
// Training Diffusion Drafters — the method exists to train diffusion drafters, so gradients flow
// through the same exact attention).
//
// With P = exp(s - LSE) recomputed from the stored natural-log LSE and D = rowsum(dO * O):
//   dV_j += P_j dO,   dS_j = P_j (dO.v_j - D),   dQ += scale dS_j k_j,   dK_j += scale dS_j q.
// Key-stationary on CUDA cores (fp32 FMA): one CTA owns a tile of 32 keys of one kv head and
// loops over the blocks that see it (anchor > first key), 32 query rows at a time, so dK/dV are
// written once without atomics; dQ is accumulated with fp32 atomics. A second kernel does the
// same for each block's own 16 keys (dKb, dVb). dq is zeroed first.
#include "common.cuh"
#include "scan.cuh"

namespace splitkv {

namespace {

constexpr int kThreads = 256;
constexpr int kBK = 32;  // keys per CTA tile
constexpr int kBR = 32;  // query rows per step
constexpr int kMaxAcc = kBK * 128 / kThreads;  // dK/dV elements per thread at d = 128

struct TileMap {
    int64_t tile_base[kMaxBatch + 1];  // first key tile (per kv head) of each sample
};

template <typename T>
__global__ void __launch_bounds__(kThreads) dvec_kernel(Meta m, const T* __restrict__ o, const T* __restrict__ dout,
                                                        float* __restrict__ dvec) {
    const int lane = threadIdx.x & 31;
    const int64_t row = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    if (row >= m.n_queries * m.hq) return;
    float acc = 0.f;
    for (int dd = lane; dd < m.d; dd += 32) acc = fmaf(to_f32(o[row * m.d + dd]), to_f32(dout[row * m.d + dd]), acc);
    acc = warp_reduce_sum(acc);
    if (lane == 0) dvec[row] = acc;
}

// Shared body: `nk` keys (rows of kp/vp with stride kstride) seen by the R rows of global block j
// at kv head g, the first `nvis` of them visible. Accumulates into dk/dv registers, dQ via atomics.
template <typename T>
__device__ void tile_rows(const Meta& m, int32_t j, int g, int nvis, const float* Ks, const float* Vs,
                          const T* __restrict__ q, const T* __restrict__ dout, const float* __restrict__ lse,
                          const float* __restrict__ dvec, float* __restrict__ dq, float* Qc, float* dOc, float* Ps,
                          float* dSs, float* Lc, float* Dc, float (&adk)[kMaxAcc], float (&adv)[kMaxAcc]) {
    const int R = m.rows, d = m.d, G = m.group, dp = d + 1;
    const int tid = threadIdx.x;
    for (int r0 = 0; r0 < R; r0 += kBR) {
        const int nr = min(kBR, R - r0);
        for (int e = tid; e < kBR * d; e += kThreads) {
            int rr = e / d, dd = e % d;
            float qv = 0.f, gv = 0.f;
            if (rr < nr) {
                int r = r0 + rr, i = r / G, hl = r % G;
                int64_t orow = ((int64_t)m.block * j + i) * m.hq + (int64_t)g * G + hl;
                qv = to_f32(q[orow * d + dd]);
                gv = to_f32(dout[orow * d + dd]);
            }
            Qc[rr * dp + dd] = qv;
            dOc[rr * dp + dd] = gv;
        }
        for (int rr = tid; rr < kBR; rr += kThreads) {
            float L = INFINITY, D = 0.f;
            if (rr < nr) {
                int r = r0 + rr, i = r / G, hl = r % G;
                int64_t orow = ((int64_t)m.block * j + i) * m.hq + (int64_t)g * G + hl;
                L = lse[orow];
                D = dvec[orow];
            }
            Lc[rr] = L;
            Dc[rr] = D;
        }
        __syncthreads();
        for (int e = tid; e < kBR * kBK; e += kThreads) {
            int rr = e / kBK, jj = e % kBK;
            float p = 0.f, ds = 0.f;
            if (rr < nr && jj < nvis) {
                float sacc = 0.f, dpacc = 0.f;
                for (int dd = 0; dd < d; ++dd) {
                    sacc = fmaf(Qc[rr * dp + dd], Ks[jj * dp + dd], sacc);
                    dpacc = fmaf(dOc[rr * dp + dd], Vs[jj * dp + dd], dpacc);
                }
                p = expf(sacc * m.scale - Lc[rr]);
                ds = p * (dpacc - Dc[rr]);
            }
            Ps[rr * (kBK + 1) + jj] = p;
            dSs[rr * (kBK + 1) + jj] = ds;
        }
        __syncthreads();
        // dK, dV for this thread's (key, dim) elements.
#pragma unroll
        for (int u = 0; u < kMaxAcc; ++u) {
            int e = tid + u * kThreads;
            if (e < kBK * d) {
                int jj = e / d, dd = e % d;
                float sv = 0.f, sk = 0.f;
                for (int rr = 0; rr < nr; ++rr) {
                    sv = fmaf(Ps[rr * (kBK + 1) + jj], dOc[rr * dp + dd], sv);
                    sk = fmaf(dSs[rr * (kBK + 1) + jj], Qc[rr * dp + dd], sk);
                }
                adv[u] += sv;
                adk[u] += sk * m.scale;
            }
        }
        // dQ for (row, dim) elements.
        for (int e = tid; e < nr * d; e += kThreads) {
            int rr = e / d, dd = e % d;
            float acc = 0.f;
            for (int jj = 0; jj < nvis && jj < kBK; ++jj) acc = fmaf(dSs[rr * (kBK + 1) + jj], Ks[jj * dp + dd], acc);
            int r = r0 + rr, i = r / G, hl = r % G;
            int64_t orow = ((int64_t)m.block * j + i) * m.hq + (int64_t)g * G + hl;
            atomicAdd(&dq[orow * d + dd], acc * m.scale);
        }
        __syncthreads();
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_context_kernel(Meta m, TileMap tm, const T* __restrict__ q,
                                                               const T* __restrict__ k, const T* __restrict__ v,
                                                               const T* __restrict__ dout,
                                                               const float* __restrict__ lse,
                                                               const float* __restrict__ dvec,
                                                               const int32_t* __restrict__ anchors,
                                                               float* __restrict__ dq, float* __restrict__ dk,
                                                               float* __restrict__ dv,
                                                               const int32_t* __restrict__ status) {
    extern __shared__ float smem[];
    if (status_bad(status)) return;
    const int d = m.d, dp = d + 1;
    float* Ks = smem;
    float* Vs = Ks + kBK * dp;
    float* Qc = Vs + kBK * dp;
    float* dOc = Qc + kBR * dp;
    float* Ps = dOc + kBR * dp;
    float* dSs = Ps + kBR * (kBK + 1);
    float* Lc = dSs + kBR * (kBK + 1);
    float* Dc = Lc + kBR;
    const int tid = threadIdx.x;
    const int64_t t = blockIdx.x / m.hkv;
    const int g = blockIdx.x % m.hkv;
    int s = 0;
    while (s + 1 < m.batch && t >= tm.tile_base[s + 1]) ++s;
    const int64_t k0 = (t - tm.tile_base[s]) * kBK;
    const int nk = (int)min((int64_t)kBK, m.seq_len[s] - k0);
    const int64_t krow0 = m.key_off[s] + k0;
    for (int e = tid; e < kBK * d; e += kThreads) {
        int jj = e / d, dd = e % d;
        float kv = 0.f, vv = 0.f;
        if (jj < nk) {
            int64_t off = ((krow0 + jj) * m.hkv + g) * d + dd;
            kv = to_f32(k[off]);
            vv = to_f32(v[off]);
        }
        Ks[jj * dp + dd] = kv;
        Vs[jj * dp + dd] = vv;
    }
    float adk[kMaxAcc], adv[kMaxAcc];
#pragma unroll
    for (int u = 0; u < kMaxAcc; ++u) adk[u] = adv[u] = 0.f;
    __syncthreads();
    // Blocks of sample s whose anchor exceeds k0 (a suffix, anchors ascending).
    const int32_t b_lo = m.anchor_off[s], b_hi = m.anchor_off[s + 1];
    int32_t lo = b_lo, hi = b_hi;
    while (lo < hi) {
        int32_t mid = (lo + hi) >> 1;
        if ((int64_t)anchors[mid] > k0) hi = mid; else lo = mid + 1;
    }
    // Context parallelism: a rank computes only the key tiles of its own chunks (zeros elsewhere).
    const int32_t j_end = owns_chunk(m, s, (int32_t)(k0 / m.chunk)) ? b_hi : lo;
    for (int32_t j = lo; j < j_end; ++j) {
        const int64_t a = anchors[j];
        const int nvis = (int)min((int64_t)nk, a - k0);
        tile_rows<T>(m, j, g, nvis, Ks, Vs, q, dout, lse, dvec, dq, Qc, dOc, Ps, dSs, Lc, Dc, adk, adv);
    }
#pragma unroll
    for (int u = 0; u < kMaxAcc; ++u) {
        int e = tid + u * kThreads;
        if (e < kBK * d) {
            int jj = e / d, dd = e % d;
            if (jj < nk) {
                int64_t off = ((krow0 + jj) * m.hkv + g) * d + dd;
                dk[off] = adk[u];
                dv[off] = adv[u];
            }
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_self_kernel(Meta m, const T* __restrict__ q,
                                                            const T* __restrict__ kb, const T* __restrict__ vb,
                                                            const T* __restrict__ dout, const float* __restrict__ lse,
                                                            const float* __restrict__ dvec, float* __restrict__ dq,
                                                            float* __restrict__ dkb, float* __restrict__ dvb,
                                                            const int32_t* __restrict__ status) {
    extern __shared__ float smem[];
    if (status_bad(status)) return;
    const int d = m.d, dp = d + 1, BL = m.block;
    float* Ks = smem;
    float* Vs = Ks + kBK * dp;
    float* Qc = Vs + kBK * dp;
    float* dOc = Qc + kBR * dp;
    float* Ps = dOc + kBR * dp;
    float* dSs = Ps + kBR * (kBK + 1);
    float* Lc = dSs + kBR * (kBK + 1);
    float* Dc = Lc + kBR;
    const int tid = threadIdx.x;
    const int32_t j = blockIdx.x / m.hkv;
    const int g = blockIdx.x % m.hkv;
    for (int e = tid; e < kBK * d; e += kThreads) {
        int jj = e / d, dd = e % d;
        float kv = 0.f, vv = 0.f;
        if (jj < BL) {
            int64_t off = (((int64_t)BL * j + jj) * m.hkv + g) * d + dd;
            kv = to_f32(kb[off]);
            vv = to_f32(vb[off]);
        }
        Ks[jj * dp + dd] = kv;
        Vs[jj * dp + dd] = vv;
    }
    float adk[kMaxAcc], adv[kMaxAcc];
#pragma unroll
    for (int u = 0; u < kMaxAcc; ++u) adk[u] = adv[u] = 0.f;
    __syncthreads();
    // Context parallelism: the block's own keys belong to rank j % n_ranks (zeros elsewhere).
    if (owns_self(m, j)) tile_rows<T>(m, j, g, BL, Ks, Vs, q, dout, lse, dvec, dq, Qc, dOc, Ps, dSs, Lc, Dc, adk, adv);
#pragma unroll
    for (int u = 0; u < kMaxAcc; ++u) {
        int e = tid + u * kThreads;
        if (e < kBK * d) {
            int jj = e / d, dd = e % d;
            if (jj < BL) {
                int64_t off = (((int64_t)BL * j + jj) * m.hkv + g) * d + dd;
                dkb[off] = adk[u];
                dvb[off] = adv[u];
            }
        }
    }
}

template <typename T>
cudaError_t launch_t(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                     const void* o, const float* lse, const void* dout, const int32_t* anchors, float* dq, float* dk,
                     float* dv, float* dkb, float* dvb, int32_t* status, void* ws, cudaStream_t st) {
    float* dvec = (float*)ws;
    const int64_t rows = m.n_queries * m.hq;
    cudaError_t e = rows > 0 ? cudaMemsetAsync(dq, 0, sizeof(float) * (size_t)rows * m.d, st) : cudaSuccess;
    if (e != cudaSuccess) return e;
    if (rows > 0) {
        dvec_kernel<T><<<(unsigned)((rows * 32 + kThreads - 1) / kThreads), kThreads, 0, st>>>(
            m, (const T*)o, (const T*)dout, dvec);
    }
    TileMap tm;
    tm.tile_base[0] = 0;
    for (int s = 0; s < m.batch; ++s) tm.tile_base[s + 1] = tm.tile_base[s] + (m.seq_len[s] + kBK - 1) / kBK;
    const int d = m.d;
    size_t smem = sizeof(float) * ((size_t)2 * kBK * (d + 1) + 2 * kBR * (d + 1) + 2 * kBR * (kBK + 1) + 2 * kBR);
    e = cudaFuncSetAttribute(bwd_context_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_self_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t ntiles = tm.tile_base[m.batch] * m.hkv;
    if (ntiles > 0)
        bwd_context_kernel<T><<<(unsigned)ntiles, kThreads, smem, st>>>(m, tm, (const T*)q, (const T*)k, (const T*)v,
                                                                       (const T*)dout, lse, dvec, anchors, dq, dk,
                                                                       dv, status);
    const int64_t nself = m.n_blocks * m.hkv;
    if (nself > 0)
        bwd_self_kernel<T><<<(unsigned)nself, kThreads, smem, st>>>(m, (const T*)q, (const T*)kb, (const T*)vb,
                                                                    (const T*)dout, lse, dvec, dq, dkb, dvb, status);
    return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace(const Meta& m) { return align_up(sizeof(float) * (size_t)m.n_queries * m.hq, 256); }

cudaError_t launch_bwd(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                       const void* o, const float* lse, const void* dout, const int32_t* anchors, float* dq,
                       float* dk, float* dv, float* dkb, float* dvb, int32_t* status, void* ws, cudaStream_t st) {
    if (m.dtype == SPLITKV_F32)
        return launch_t<float>(m, q, k, v, kb, vb, o, lse, dout, anchors, dq, dk, dv, dkb, dvb, status, ws, st);
    return launch_t<__nv_bfloat16>(m, q, k, v, kb, vb, o, lse, dout, anchors, dq, dk, dv, dkb, dvb, status, ws, st);
}

}  // namespace splitkv
