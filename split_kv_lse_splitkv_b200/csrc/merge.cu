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
// tiles are read exactly once, in one pass, in float32.
//
// Memory-bound. The partial tiles are stored [d/E][rows][E] in the problem dtype (E elements per
// 16-byte group: 4 float32 or 8 bf16). A thread owns one row r and 16 consecutive columns (4 or 2
// groups); a CTA owns kThreads consecutive (row, column block) units of one (j, g), so a warp's 32
// consecutive rows read 512 contiguous bytes per group, and each thread keeps two (bf16) or four
// (float32) partials' loads in flight. The output row receives 16 contiguous values, written as
// 16-byte stores: with one element per store, each warp store touched 32 rows' sectors for 64 bytes
// and the stores took as much of the load/store path as the partial loads (drafter_s32k: 62.5 us
// with scalar stores, 36.8 us with 16-byte ones). CTAs start at the last query block: within a sample
// blocks are numbered by anchor, so the last ones merge the most chunks and, launched last, would
// form the tail (36.8 -> 31.7 us).
#include "common.cuh"

namespace splitkv {

namespace {

constexpr int kThreads = 256;
constexpr int kVals = 16;   // columns per thread
// Partials loaded ahead, and CTAs per SM the registers are sized for: bf16 tiles take two partials
// ahead at four CTAs per SM (64 registers), float32 tiles four at the default.
template <typename T>
struct MergeShape {
    static constexpr int kUnroll = 4, kMinBlocks = 1;
};
template <>
struct MergeShape<__nv_bfloat16> {
    static constexpr int kUnroll = 2, kMinBlocks = 4;
};

struct Online {
    float m, l;
    float acc[kVals];
};

__device__ __forceinline__ void online_add(Online& st, float lse_p, const float (&x)[kVals]) {
    if (lse_p == -INFINITY) return;  // an empty partial contributes nothing
    const float m_new = fmaxf(st.m, lse_p);
    const float a = __expf(st.m - m_new), w = __expf(lse_p - m_new);
    st.l = fmaf(st.l, a, w);
    st.m = m_new;
#pragma unroll
    for (int u = 0; u < kVals; ++u) st.acc[u] = fmaf(w, x[u], st.acc[u] * a);
}

__device__ __forceinline__ void unpack16(const uint4& v, float* x, float) {  // 4 float32
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ void unpack16(const uint4& v, float* x, __nv_bfloat16) {  // 8 bf16, low half first
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}

// 16 values x inv to 16-byte aligned `dst`: four float32 or two bf16 16-byte stores.
__device__ __forceinline__ void store_vals(float* dst, const float (&x)[kVals], float inv) {
#pragma unroll
    for (int u = 0; u < kVals; u += 4)
        *reinterpret_cast<float4*>(dst + u) = make_float4(x[u] * inv, x[u + 1] * inv, x[u + 2] * inv, x[u + 3] * inv);
}
__device__ __forceinline__ void store_vals(__nv_bfloat16* dst, const float (&x)[kVals], float inv) {
    uint32_t w[kVals / 2];
#pragma unroll
    for (int e = 0; e < kVals / 2; ++e) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * e] * inv, x[2 * e + 1] * inv);  // low half first
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
#pragma unroll
    for (int u = 0; u < kVals / 8; ++u)
        *reinterpret_cast<uint4*>(dst + 8 * u) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
}

// Row `r` of a partial tile of `RT` rows: 16 columns from 16-byte group g0 on, zero past d.
template <typename T>
__device__ __forceinline__ void load_row(const uint4* __restrict__ tile, int RT, int r, int g0, int ngroups,
                                         float (&x)[kVals]) {
    constexpr int E = 16 / (int)sizeof(T), KG = kVals / E;
    uint4 v[KG];
#pragma unroll
    for (int u = 0; u < KG; ++u)
        v[u] = g0 + u < ngroups ? __ldcs(tile + (int64_t)(g0 + u) * RT + r) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < KG; ++u) unpack16(v[u], x + u * E, T());
}

template <typename T>
__global__ void __launch_bounds__(kThreads, MergeShape<T>::kMinBlocks) merge_kernel(Meta m, int32_t ctas_per_head, const T* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         const int32_t* __restrict__ anchors, T* __restrict__ o,
                                                         float* __restrict__ lse, const int32_t* __restrict__ status) {
    constexpr int E = 16 / (int)sizeof(T);
    constexpr int kUnroll = MergeShape<T>::kUnroll;
    if (status_bad(status)) return;
    const int R = m.rows, d = m.d, G = m.group, BL = m.block, ngroups = d / E;
    const int64_t jg = (int64_t)m.n_blocks * m.hkv - 1 - blockIdx.x / ctas_per_head;  // last blocks (most chunks) first
    const int32_t j = (int32_t)(jg / m.hkv), g = (int32_t)(jg % m.hkv);
    const int unit = (blockIdx.x % ctas_per_head) * kThreads + threadIdx.x;
    const int blocks = (d + kVals - 1) / kVals;  // 16-column blocks per row
    if (unit >= R * blocks) return;
    const int r = unit % R, c0 = (unit / R) * kVals, g0 = c0 / E;

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
    const int RT = m.rows_item;                     // rows of a partial tile
    const int rc = (b % m.pack) * R + r;            // this row within its chunk partials
    const int64_t tile16 = (int64_t)RT * ngroups;   // 16-byte groups per partial tile
    const uint4* op = reinterpret_cast<const uint4*>(o_part);

    Online st;
    st.m = -INFINITY;
    st.l = 0.f;
#pragma unroll
    for (int u = 0; u < kVals; ++u) st.acc[u] = 0.f;
    if (owns_self(m, j)) {
        const int64_t self = m.n_items + jg;
        float x[kVals];
        load_row<T>(op + self * tile16, RT, r, g0, ngroups, x);
        online_add(st, __ldcs(lse_part + self * RT + r), x);
    }
    int32_t c = 0;
    if (m.rank >= 0) {  // context parallelism: only the partials of this rank's chunks
        for (; c < nv; ++c) {
            if (!owns_chunk(m, s, c)) continue;
            const int64_t item = item0 + (int64_t)c * cstride;
            float x[kVals];
            load_row<T>(op + item * tile16, RT, rc, g0, ngroups, x);
            online_add(st, __ldcs(lse_part + item * RT + rc), x);
        }
    }
    for (; c + kUnroll <= nv; c += kUnroll) {
        float x[kUnroll][kVals];
        float lp[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int64_t item = item0 + (int64_t)(c + k) * cstride;
            lp[k] = __ldcs(lse_part + item * RT + rc);
            load_row<T>(op + item * tile16, RT, rc, g0, ngroups, x[k]);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) online_add(st, lp[k], x[k]);
    }
    for (; c < nv; ++c) {
        const int64_t item = item0 + (int64_t)c * cstride;
        float x[kVals];
        load_row<T>(op + item * tile16, RT, rc, g0, ngroups, x);
        online_add(st, __ldcs(lse_part + item * RT + rc), x);
    }

    const float inv = st.l > 0.f ? 1.f / st.l : 0.f;  // nothing merged (a rank without this row's keys): O = 0
    const int i = r / G, hl = r % G;
    const int64_t orow = ((int64_t)BL * j + i) * m.hq + (int64_t)g * G + hl;
    T* dst = o + orow * d + c0;
    if (d % E == 0 && c0 + kVals <= d) {
        // A whole 16-column block: 16-byte stores (rows of d elements keep 16-byte alignment).
        store_vals(dst, st.acc, inv);
    } else {
#pragma unroll
        for (int u = 0; u < kVals; ++u)
            if (c0 + u < d) dst[u] = from_f32<T>(st.acc[u] * inv);
    }
    if (c0 == 0) lse[orow] = st.l > 0.f ? st.m + logf(st.l) : -INFINITY;
}

// Merge across ranks: o_ranks [n_ranks][rows][d] (problem dtype), lse_ranks [n_ranks][rows] float32, rows =
// Nq * Hq; a rank's -inf row holds nothing. One thread per (row, 16 columns).
template <typename T>
__global__ void __launch_bounds__(kThreads) merge_ranks_kernel(int64_t rows, int32_t d, int32_t n_ranks,
                                                              const T* __restrict__ o_ranks,
                                                              const float* __restrict__ lse_ranks,
                                                              T* __restrict__ o, float* __restrict__ lse,
                                                              const int32_t* __restrict__ status) {
    if (status_bad(status)) return;
    const int blocks = (d + kVals - 1) / kVals;
    const int64_t unit = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (unit >= rows * blocks) return;
    const int64_t row = unit / blocks;
    const int c0 = (int)(unit % blocks) * kVals;
    Online st;
    st.m = -INFINITY;
    st.l = 0.f;
#pragma unroll
    for (int u = 0; u < kVals; ++u) st.acc[u] = 0.f;
    for (int32_t r = 0; r < n_ranks; ++r) {
        const float lp = lse_ranks[(int64_t)r * rows + row];
        if (lp == -INFINITY) continue;
        const T* src = o_ranks + ((int64_t)r * rows + row) * d + c0;
        float x[kVals];
#pragma unroll
        for (int u = 0; u < kVals; ++u) x[u] = c0 + u < d ? to_f32(src[u]) : 0.f;
        online_add(st, lp, x);
    }
    const float inv = st.l > 0.f ? 1.f / st.l : 0.f;
    T* dst = o + row * d + c0;
#pragma unroll
    for (int u = 0; u < kVals; ++u)
        if (c0 + u < d) dst[u] = from_f32<T>(st.acc[u] * inv);
    if (c0 == 0) lse[row] = st.l > 0.f ? st.m + logf(st.l) : -INFINITY;
}

template <typename T>
cudaError_t launch_t(const Meta& m, const void* o_part, const float* lse_part, const int32_t* anchors, void* o,
                     float* lse, int32_t* status, cudaStream_t st) {
    const int blocks = (m.d + kVals - 1) / kVals;
    const int32_t ctas_per_head = (m.rows * blocks + kThreads - 1) / kThreads;
    const int64_t grid = m.n_blocks * m.hkv * ctas_per_head;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffff) return note_error(cudaErrorInvalidConfiguration, "merge: grid too large");
    merge_kernel<T><<<(unsigned)grid, kThreads, 0, st>>>(m, ctas_per_head, (const T*)o_part, lse_part, anchors, (T*)o,
                                                         lse, status);
    return note_error(cudaGetLastError(), "launch merge_kernel");
}

}  // namespace

cudaError_t launch_merge_ranks(const Meta& m, int32_t n_ranks, const void* o_ranks, const float* lse_ranks, void* o,
                               float* lse, int32_t* status, cudaStream_t st) {
    const int64_t rows = m.n_queries * m.hq;
    const int64_t units = rows * ((m.d + kVals - 1) / kVals);
    const int64_t grid = (units + kThreads - 1) / kThreads;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffff) return note_error(cudaErrorInvalidConfiguration, "merge_ranks: grid too large");
    if (m.dtype == SPLITKV_F32)
        merge_ranks_kernel<float><<<(unsigned)grid, kThreads, 0, st>>>(rows, m.d, n_ranks, (const float*)o_ranks,
                                                                        lse_ranks, (float*)o, lse, status);
    else
        merge_ranks_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, 0, st>>>(
            rows, m.d, n_ranks, (const __nv_bfloat16*)o_ranks, lse_ranks, (__nv_bfloat16*)o, lse, status);
    return note_error(cudaGetLastError(), "launch merge_ranks_kernel");
}

cudaError_t launch_merge(const Meta& m, const void* o_part, const float* lse_part, const int32_t* anchors, void* o,
                         float* lse, int32_t* status, cudaStream_t st) {
    if (m.dtype == SPLITKV_F32) return launch_t<float>(m, o_part, lse_part, anchors, o, lse, status, st);
    return launch_t<__nv_bfloat16>(m, o_part, lse_part, anchors, o, lse, status, st);
}

}  // namespace splitkv
