// Exact log-sum-exp merge of the chunk partials, fused with the block's own-keys partial
// (Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, Abstract: exact
// attention assembled from chunk-local, query-sized partial results).
//
// One CTA per (global block j, kv head g): its block*G query rows r = i*G + hl. For every row:
//   self partial over the block's own keys: s_t = scale q.kb_t;
//   L = log( sum_t exp(s_t) + sum_{c < ceil(a/C)} exp(LSE_c) )          (max-shifted)
//   O = sum_c exp(LSE_c - L) O_c + sum_t exp(s_t - L) vb_t.
// Memory-bound: every visible partial tile is read once. The per-chunk LSEs are staged in shared
// memory with coalesced loads and turned into weights there; the partial tiles are stored
// [d/4][rows][4], so consecutive threads (consecutive rows) read consecutive 16-byte words, and
// each thread keeps four chunk loads in flight.
#include "common.cuh"
#include "scan.cuh"

namespace splitkv {

namespace {

constexpr int kThreads = 512;

template <typename T>
__global__ void __launch_bounds__(kThreads) merge_kernel(Meta m, int32_t max_nv, const float* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         const T* __restrict__ q, const T* __restrict__ kb,
                                                         const T* __restrict__ vb,
                                                         const int32_t* __restrict__ anchors, T* __restrict__ o,
                                                         float* __restrict__ lse, const int32_t* __restrict__ status) {
    extern __shared__ float smem[];
    if (status_bad(status)) return;
    const int R = m.rows, d = m.d, G = m.group, BL = m.block;
    const int dp = d + 1;
    float* Qs = smem;             // [R][d+1]
    float* Kbs = Qs + R * dp;     // [BL][d+1]
    float* Vbs = Kbs + BL * dp;   // [BL][d]
    float* Ps = Vbs + BL * d;     // [R][BL]   self scores, then self weights
    float* Lr = Ps + R * BL;      // [R]
    float* Wc = Lr + R;           // [max_nv][R] chunk LSEs, then chunk weights
    const int tid = threadIdx.x;
    const int32_t j = blockIdx.x / m.hkv, g = blockIdx.x % m.hkv;
    const int s = sample_of_block(m, j);
    const int32_t b = j - m.anchor_off[s];
    const int32_t nb = m.anchor_off[s + 1] - m.anchor_off[s];
    const int32_t a = anchors[j];
    int32_t nv = (int32_t)(((int64_t)a + m.chunk - 1) / m.chunk);
    if (nv < 0) nv = 0;
    if (nv > m.n_chunk_s[s]) nv = m.n_chunk_s[s];
    if (nv > max_nv) nv = max_nv;
    const int64_t item0 = m.item_base[s] + (int64_t)g * nb + b;  // chunk 0; chunk c adds c*Hkv*nb
    const int64_t cstride = (int64_t)m.hkv * nb;

    for (int e = tid; e < R * d; e += kThreads) {
        int r = e / d, dd = e % d;
        int i = r / G, hl = r % G;
        int64_t row = (int64_t)BL * j + i;
        Qs[r * dp + dd] = to_f32(q[(row * m.hq + (int64_t)g * G + hl) * d + dd]);
    }
    for (int e = tid; e < BL * d; e += kThreads) {
        int t = e / d, dd = e % d;
        int64_t off = (((int64_t)BL * j + t) * m.hkv + g) * d + dd;
        Kbs[t * dp + dd] = to_f32(kb[off]);
        Vbs[t * d + dd] = to_f32(vb[off]);
    }
    for (int e = tid; e < nv * R; e += kThreads) {
        int c = e / R, r = e % R;
        Wc[e] = lse_part[(item0 + c * cstride) * R + r];
    }
    __syncthreads();
    for (int e = tid; e < R * BL; e += kThreads) {
        int r = e / BL, t = e % BL;
        float acc = 0.f;
        for (int dd = 0; dd < d; ++dd) acc = fmaf(Qs[r * dp + dd], Kbs[t * dp + dd], acc);
        Ps[e] = acc * m.scale;
    }
    __syncthreads();
    for (int r = tid; r < R; r += kThreads) {
        float M = -INFINITY;
        for (int t = 0; t < BL; ++t) M = fmaxf(M, Ps[r * BL + t]);
        for (int c = 0; c < nv; ++c) M = fmaxf(M, Wc[c * R + r]);
        float sum = 0.f;
        for (int t = 0; t < BL; ++t) sum += expf(Ps[r * BL + t] - M);
        for (int c = 0; c < nv; ++c) sum += expf(Wc[c * R + r] - M);
        const float L = M + logf(sum);
        Lr[r] = L;
        for (int t = 0; t < BL; ++t) Ps[r * BL + t] = expf(Ps[r * BL + t] - L);
        for (int c = 0; c < nv; ++c) Wc[c * R + r] = expf(Wc[c * R + r] - L);
    }
    __syncthreads();
    const int D4 = d / 4;
    const float4* op = reinterpret_cast<const float4*>(o_part);
    for (int e = tid; e < R * D4; e += kThreads) {
        const int r = e % R, d4 = e / R;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const int64_t base = (int64_t)d4 * R + r;  // float4 index inside an item tile
        int c = 0;
        for (; c + 4 <= nv; c += 4) {
            float4 x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = __ldcs(op + (item0 + (c + u) * cstride) * (int64_t)R * D4 + base);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float wgt = Wc[(c + u) * R + r];
                acc.x = fmaf(wgt, x[u].x, acc.x);
                acc.y = fmaf(wgt, x[u].y, acc.y);
                acc.z = fmaf(wgt, x[u].z, acc.z);
                acc.w = fmaf(wgt, x[u].w, acc.w);
            }
        }
        for (; c < nv; ++c) {
            const float4 x = __ldcs(op + (item0 + c * cstride) * (int64_t)R * D4 + base);
            const float wgt = Wc[c * R + r];
            acc.x = fmaf(wgt, x.x, acc.x);
            acc.y = fmaf(wgt, x.y, acc.y);
            acc.z = fmaf(wgt, x.z, acc.z);
            acc.w = fmaf(wgt, x.w, acc.w);
        }
        for (int t = 0; t < BL; ++t) {
            const float p = Ps[r * BL + t];
            const float* vr = Vbs + t * d + d4 * 4;
            acc.x = fmaf(p, vr[0], acc.x);
            acc.y = fmaf(p, vr[1], acc.y);
            acc.z = fmaf(p, vr[2], acc.z);
            acc.w = fmaf(p, vr[3], acc.w);
        }
        const int i = r / G, hl = r % G;
        const int64_t orow = ((int64_t)BL * j + i) * m.hq + (int64_t)g * G + hl;
        T* dst = o + orow * d + d4 * 4;
        dst[0] = from_f32<T>(acc.x);
        dst[1] = from_f32<T>(acc.y);
        dst[2] = from_f32<T>(acc.z);
        dst[3] = from_f32<T>(acc.w);
        if (d4 == 0) lse[orow] = Lr[r];
    }
}

template <typename T>
cudaError_t launch_t(const Meta& m, const float* o_part, const float* lse_part, const void* q, const void* kb,
                     const void* vb, const int32_t* anchors, void* o, float* lse, int32_t* status, cudaStream_t st) {
    const int R = m.rows, d = m.d, BL = m.block;
    int32_t max_nv = 0;
    for (int s = 0; s < m.batch; ++s) max_nv = m.n_chunk_s[s] > max_nv ? m.n_chunk_s[s] : max_nv;
    size_t smem = sizeof(float) * ((size_t)R * (d + 1) + BL * (d + 1) + BL * d + R * BL + R + (size_t)max_nv * R);
    if (smem > 227 * 1024) return note_error(cudaErrorInvalidConfiguration, "merge: too many chunks per sample");
    cudaError_t e = cudaFuncSetAttribute(merge_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return note_error(e, "cudaFuncSetAttribute(merge_kernel)");
    int64_t grid = m.n_blocks * m.hkv;
    if (grid == 0) return cudaSuccess;
    merge_kernel<T><<<(unsigned)grid, kThreads, smem, st>>>(m, max_nv, o_part, lse_part, (const T*)q, (const T*)kb,
                                                            (const T*)vb, anchors, (T*)o, lse, status);
    return note_error(cudaGetLastError(), "launch merge_kernel");
}

}  // namespace

cudaError_t launch_merge(const Meta& m, const float* o_part, const float* lse_part, const void* q, const void* kb,
                         const void* vb, const int32_t* anchors, void* o, float* lse, int32_t* status,
                         cudaStream_t st) {
    if (m.dtype == SPLITKV_F32)
        return launch_t<float>(m, o_part, lse_part, q, kb, vb, anchors, o, lse, status, st);
    return launch_t<__nv_bfloat16>(m, o_part, lse_part, q, kb, vb, anchors, o, lse, status, st);
}

}  // namespace splitkv
