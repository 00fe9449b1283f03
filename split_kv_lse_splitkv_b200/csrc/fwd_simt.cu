// Chunk-partial forward on CUDA cores (fp32 FMA), any head_dim <= 128 and any element type.
// It serves the float32 problems and, for bfloat16 problems, an independent cross-check of the
// tensor-core kernel. One persistent CTA per worker walks its LPT queue; per item it runs the
// chunk-local online softmax over key tiles of 32 keys and writes the normalised partial output
// and its natural-log LSE (Split-KV: Efficient Context Parallelism for Training Diffusion
// Drafters, Abstract: exact attention from chunk-local, query-sized partials). After its queue each
// CTA also computes a share of the self partials (block j, kv head g) over the block's own keys,
// stored at slot n_items + j*Hkv + g.
#include "common.cuh"
#include "scan.cuh"

namespace splitkv {

namespace {

constexpr int kThreads = 256;
constexpr int kBK = 32;  // keys per tile (one per lane in the softmax step)

template <typename T>
__global__ void __launch_bounds__(kThreads) fwd_simt_kernel(Meta m, const T* __restrict__ q,
                                                            const T* __restrict__ k, const T* __restrict__ v,
                                                            const T* __restrict__ kb, const T* __restrict__ vb,
                                                            const int32_t* __restrict__ anchors,
                                                            const int32_t* __restrict__ item_id,
                                                            const int32_t* __restrict__ queue_off,
                                                            const int32_t* __restrict__ queue_items,
                                                            T* __restrict__ o_part, float* __restrict__ lse_part,
                                                            int32_t* __restrict__ status) {
    extern __shared__ float smem[];
    if (status_bad(status)) return;
    // Rows of an item's tile, and the rows of one pass over its keys (a tile of more than 128 rows, a
    // 256-row item, takes two passes so that its rows fit in shared memory).
    const int RT = m.rows_item, R = RT > 128 ? 128 : RT, d = m.d, G = m.group;
    const int dp = d + 1;
    float* Qs = smem;                 // [R][d]
    float* Os = Qs + R * d;           // [R][d]
    float* Ks = Os + R * d;           // [kBK][d+1]
    float* Vs = Ks + kBK * dp;        // [kBK][d]
    float* Ss = Vs + kBK * d;         // [R][kBK]
    float* mS = Ss + R * kBK;         // [R]
    float* lS = mS + R;               // [R]
    float* aS = lS + R;               // [R]
    int* vS = reinterpret_cast<int*>(aS + R);  // [R] keys of the chunk each row sees
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int32_t q0 = queue_off[blockIdx.x], q1 = queue_off[blockIdx.x + 1];
    const int64_t n_self = m.n_blocks * m.hkv;
    // Entries: the queue's items, then self items blockIdx.x, blockIdx.x + gridDim.x, ...
    for (int64_t e_idx = q0;; ++e_idx) {
        int64_t id, kbase;
        int32_t nvis;  // keys the tile's last (largest-anchor) block sees: the most of any row
        Item it;
        const T *kp = k, *vp = v;
        if (e_idx < q1) {
            const int32_t kidx = queue_items[e_idx];
            id = item_id[kidx];
            if (id < 0 || id >= m.n_items) { raise_status(status, SPLITKV_DEV_BAD_PLAN); return; }
            it = decode_item(m, id);
            nvis = visible_in_chunk(m, it.s, it.c, anchors[it.j + it.nbt - 1]);
            kbase = m.key_off[it.s] + (int64_t)it.c * m.chunk;
        } else {
            const int64_t sid = blockIdx.x + (e_idx - q1) * (int64_t)gridDim.x;
            if (sid >= n_self) break;
            id = m.n_items + sid;
            it.j = (int32_t)(sid / m.hkv);
            it.g = (int32_t)(sid % m.hkv);
            it.nbt = 1;
            nvis = m.block;
            kbase = (int64_t)m.block * it.j;
            kp = kb;
            vp = vb;
        }

        for (int r0 = 0; r0 < RT; r0 += R) {  // this pass: tile rows r0 .. r0 + R - 1
        for (int e = tid; e < R * d; e += kThreads) {
            int r = e / d, dd = e % d;
            int i = (r0 + r) / G, hl = (r0 + r) % G;
            int64_t row = (int64_t)m.block * it.j + i;  // rows past the tile's blocks are masked below
            Qs[e] = row < m.n_queries ? to_f32(q[(row * m.hq + (int64_t)it.g * G + hl) * d + dd]) : 0.f;
            Os[e] = 0.f;
        }
        for (int r = tid; r < R; r += kThreads) {
            mS[r] = -INFINITY;
            lS[r] = 0.f;
            const int x = (r0 + r) / m.rows;  // block of the tile this row belongs to
            int v = 0;
            if (e_idx >= q1) v = x == 0 ? m.block : 0;  // self item: the block's own keys, its rows only
            else if (x < it.nbt) v = visible_in_chunk(m, it.s, it.c, anchors[it.j + x]);
            vS[r] = v;
        }
        __syncthreads();

        for (int32_t t0 = 0; t0 < nvis; t0 += kBK) {
            const int nk = min(kBK, nvis - t0);
            for (int e = tid; e < kBK * d; e += kThreads) {
                int jj = e / d, dd = e % d;
                float kv = 0.f, vv = 0.f;
                if (jj < nk) {
                    int64_t off = ((kbase + t0 + jj) * m.hkv + it.g) * d + dd;
                    kv = to_f32(kp[off]);
                    vv = to_f32(vp[off]);
                }
                Ks[jj * dp + dd] = kv;
                Vs[jj * d + dd] = vv;
            }
            __syncthreads();
            for (int e = tid; e < R * kBK; e += kThreads) {
                int r = e / kBK, jj = e % kBK;
                float s = -INFINITY;
                if (jj < nk && t0 + jj < vS[r]) {
                    float acc = 0.f;
                    const float* qr = Qs + r * d;
                    const float* kr = Ks + jj * dp;
                    for (int dd = 0; dd < d; ++dd) acc = fmaf(qr[dd], kr[dd], acc);
                    s = acc * m.scale;
                }
                Ss[e] = s;
            }
            __syncthreads();
            for (int r = warp; r < R; r += kThreads / 32) {
                float x = Ss[r * kBK + lane];
                float mx = warp_reduce_max(x);
                float m_old = mS[r];
                float m_new = fmaxf(m_old, mx);
                float p = (x == -INFINITY) ? 0.f : expf(x - m_new);  // (m_new = -inf only if x is too)
                float sum = warp_reduce_sum(p);
                Ss[r * kBK + lane] = p;
                if (lane == 0) {
                    float alpha = (m_old == -INFINITY) ? 0.f : expf(m_old - m_new);
                    aS[r] = alpha;
                    lS[r] = lS[r] * alpha + sum;
                    mS[r] = m_new;
                }
            }
            __syncthreads();
            for (int e = tid; e < R * d; e += kThreads) {
                int r = e / d, dd = e % d;
                float acc = Os[e] * aS[r];
                const float* pr = Ss + r * kBK;
                for (int jj = 0; jj < nk; ++jj) acc = fmaf(pr[jj], Vs[jj * d + dd], acc);
                Os[e] = acc;
            }
            __syncthreads();
        }
        // Normalise and store in the [d/E][R][E] tile layout (E = 16 / sizeof(T) elements per 16-byte
        // group), plus the natural-log LSE.
        constexpr int E = 16 / (int)sizeof(T);
        T* op = o_part + id * (int64_t)RT * d;
        for (int e = tid; e < R * d; e += kThreads) {
            int grp = e / (R * E), rem = e % (R * E);
            int r = rem / E, ce = rem % E;
            // a row that sees no key: O = 0
            op[((int64_t)grp * RT + r0 + r) * E + ce] = from_f32<T>(lS[r] > 0.f ? Os[r * d + grp * E + ce] / lS[r] : 0.f);
        }
        for (int r = tid; r < R; r += kThreads)
            lse_part[id * RT + r0 + r] = lS[r] > 0.f ? mS[r] + logf(lS[r]) : -INFINITY;
        __syncthreads();
        }  // pass
    }
}

template <typename T>
cudaError_t launch_t(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                     const int32_t* anchors, const int32_t* item_id, const int32_t* queue_off,
                     const int32_t* queue_items, int32_t n_workers, void* o_part, float* lse_part, int32_t* status,
                     cudaStream_t st) {
    if (m.n_queries == 0) return cudaSuccess;  // no anchor: no partial to compute
    const int R = m.rows_item > 128 ? 128 : m.rows_item, d = m.d;  // rows of one pass
    size_t smem = sizeof(float) * ((size_t)2 * R * d + kBK * (d + 1) + kBK * d + R * kBK + 4 * R);
    cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fwd_simt_kernel<T><<<n_workers, kThreads, smem, st>>>(m, (const T*)q, (const T*)k, (const T*)v, (const T*)kb,
                                                          (const T*)vb, anchors, item_id, queue_off, queue_items,
                                                          (T*)o_part, lse_part, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(const Meta& m, const void* q, const void* k, const void* v, const void* kb,
                            const void* vb, const int32_t* anchors, const int32_t* item_id, const int32_t* queue_off,
                            const int32_t* queue_items, int32_t n_workers, void* o_part, float* lse_part,
                            int32_t* status, cudaStream_t st) {
    if (m.dtype == SPLITKV_F32)
        return launch_t<float>(m, q, k, v, kb, vb, anchors, item_id, queue_off, queue_items, n_workers, o_part,
                               lse_part, status, st);
    return launch_t<__nv_bfloat16>(m, q, k, v, kb, vb, anchors, item_id, queue_off, queue_items, n_workers, o_part,
                                   lse_part, status, st);
}

}  // namespace splitkv
