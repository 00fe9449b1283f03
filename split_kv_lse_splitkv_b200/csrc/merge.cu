// Exact log-sum-exp merge of the partials of one query block (Split-KV: Efficient Context
// Parallelism for Training Diffusion Drafters, Abstract: exact attention assembled from
// chunk-local, query-sized partial results).
//
// Block j (block b of sample s), kv head g has the self partial (its own keys, slot
// n_items + j*Hkv + g, rows 0 ..) and one chunk partial per visible chunk c < ceil(a/C): item
// base_s + (c*Hkv + g)*nt_s + b/P of the query tiles of P blocks, rows (b % P)*block*G ... For each
// of its block*G query rows r:
//   L = log( sum_p exp(LSE_p) ),     O = sum_p exp(LSE_p - L) O_p
// over those partials p, accumulated online (running maximum, rescaled sum) so that the partial
// tiles are read exactly once, in one pass.
//
// Memory-bound. A thread owns one row r and a group of four 16-byte columns (16 floats); a CTA
// owns kThreads consecutive (row, group) units of one (j, g). The partial tiles are stored
// [d/4][rows][4], so a warp's 32 consecutive rows read 512 contiguous bytes per column, and each
// thread keeps four partials' loads in flight. The output row receives 16 contiguous values.
#include "common.cuh"

namespace splitkv {

namespace {

constexpr int kThreads = 256;
constexpr int kCols = 4;    // float4 columns per thread
constexpr int kUnroll = 4;  // partials loaded ahead

struct Online {
    float m, l;
    float4 acc[kCols];
};

__device__ __forceinline__ void online_add(Online& st, float lse_p, const float4 (&x)[kCols]) {
    if (lse_p == -INFINITY) return;  // an empty partial contributes nothing
    const float m_new = fmaxf(st.m, lse_p);
    const float a = __expf(st.m - m_new), w = __expf(lse_p - m_new);
    st.l = fmaf(st.l, a, w);
    st.m = m_new;
#pragma unroll
    for (int u = 0; u < kCols; ++u) {
        st.acc[u].x = fmaf(w, x[u].x, st.acc[u].x * a);
        st.acc[u].y = fmaf(w, x[u].y, st.acc[u].y * a);
        st.acc[u].z = fmaf(w, x[u].z, st.acc[u].z * a);
        st.acc[u].w = fmaf(w, x[u].w, st.acc[u].w * a);
    }
}

// Row `r` of a partial tile of `RT` rows, float4 columns d40 .. d40 + kCols - 1.
__device__ __forceinline__ void load_cols(const float4* __restrict__ tile, int RT, int r, int d40, int D4,
                                          float4 (&x)[kCols]) {
#pragma unroll
    for (int u = 0; u < kCols; ++u)
        x[u] = (d40 + u < D4) ? __ldcs(tile + (int64_t)(d40 + u) * RT + r) : make_float4(0.f, 0.f, 0.f, 0.f);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) merge_kernel(Meta m, int32_t ctas_per_head,
                                                         const float* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         const int32_t* __restrict__ anchors, T* __restrict__ o,
                                                         float* __restrict__ lse, const int32_t* __restrict__ status) {
    if (status_bad(status)) return;
    const int R = m.rows, d = m.d, G = m.group, BL = m.block, D4 = d / 4;
    const int64_t jg = blockIdx.x / ctas_per_head;
    const int32_t j = (int32_t)(jg / m.hkv), g = (int32_t)(jg % m.hkv);
    const int unit = (blockIdx.x % ctas_per_head) * kThreads + threadIdx.x;
    const int groups = (D4 + kCols - 1) / kCols;
    if (unit >= R * groups) return;
    const int r = unit % R, d40 = (unit / R) * kCols;

    const int s = sample_of_block(m, j);
    const int32_t b = j - m.anchor_off[s];
    const int32_t nb = m.anchor_off[s + 1] - m.anchor_off[s];
    const int32_t a = anchors[j];
    int32_t nv = (int32_t)(((int64_t)a + m.chunk - 1) / m.chunk);
    if (nv < 0) nv = 0;
    if (nv > m.n_chunk_s[s]) nv = m.n_chunk_s[s];
    const int32_t nt = (nb + m.pack - 1) / m.pack;  // query tiles of the sample
    const int64_t item0 = m.item_base[s] + (int64_t)g * nt + b / m.pack;  // chunk 0; chunk c adds c*Hkv*nt
    const int64_t cstride = (int64_t)m.hkv * nt;
    const int RT = m.rows_item;                 // rows of a partial tile
    const int rc = (b % m.pack) * R + r;        // this row within its chunk partials
    const int64_t tile4 = (int64_t)RT * D4;     // float4s per partial tile
    const float4* op = reinterpret_cast<const float4*>(o_part);

    Online st;
    st.m = -INFINITY;
    st.l = 0.f;
#pragma unroll
    for (int u = 0; u < kCols; ++u) st.acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    {
        const int64_t self = m.n_items + jg;
        float4 x[kCols];
        load_cols(op + self * tile4, RT, r, d40, D4, x);
        online_add(st, __ldcs(lse_part + self * RT + r), x);
    }
    int32_t c = 0;
    for (; c + kUnroll <= nv; c += kUnroll) {
        float4 x[kUnroll][kCols];
        float lp[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int64_t item = item0 + (int64_t)(c + k) * cstride;
            lp[k] = __ldcs(lse_part + item * RT + rc);
            load_cols(op + item * tile4, RT, rc, d40, D4, x[k]);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) online_add(st, lp[k], x[k]);
    }
    for (; c < nv; ++c) {
        const int64_t item = item0 + (int64_t)c * cstride;
        float4 x[kCols];
        load_cols(op + item * tile4, RT, rc, d40, D4, x);
        online_add(st, __ldcs(lse_part + item * RT + rc), x);
    }

    const float inv = 1.f / st.l;
    const int i = r / G, hl = r % G;
    const int64_t orow = ((int64_t)BL * j + i) * m.hq + (int64_t)g * G + hl;
    T* dst = o + orow * d + d40 * 4;
#pragma unroll
    for (int u = 0; u < kCols; ++u) {
        if (d40 + u < D4) {
            dst[4 * u + 0] = from_f32<T>(st.acc[u].x * inv);
            dst[4 * u + 1] = from_f32<T>(st.acc[u].y * inv);
            dst[4 * u + 2] = from_f32<T>(st.acc[u].z * inv);
            dst[4 * u + 3] = from_f32<T>(st.acc[u].w * inv);
        }
    }
    if (d40 == 0) lse[orow] = st.m + logf(st.l);
}

template <typename T>
cudaError_t launch_t(const Meta& m, const float* o_part, const float* lse_part, const int32_t* anchors, void* o,
                     float* lse, int32_t* status, cudaStream_t st) {
    const int groups = (m.d / 4 + kCols - 1) / kCols;
    const int32_t ctas_per_head = (m.rows * groups + kThreads - 1) / kThreads;
    const int64_t grid = m.n_blocks * m.hkv * ctas_per_head;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffff) return note_error(cudaErrorInvalidConfiguration, "merge: grid too large");
    merge_kernel<T><<<(unsigned)grid, kThreads, 0, st>>>(m, ctas_per_head, o_part, lse_part, anchors, (T*)o, lse,
                                                         status);
    return note_error(cudaGetLastError(), "launch merge_kernel");
}

}  // namespace

cudaError_t launch_merge(const Meta& m, const float* o_part, const float* lse_part, const int32_t* anchors, void* o,
                         float* lse, int32_t* status, cudaStream_t st) {
    if (m.dtype == SPLITKV_F32) return launch_t<float>(m, o_part, lse_part, anchors, o, lse, status, st);
    return launch_t<__nv_bfloat16>(m, o_part, lse_part, anchors, o, lse, status, st);
}

}  // namespace splitkv
