// Realized cost pass (Split-KV: Efficient Context Parallelism for Training Diffusion Drafters,
// Abstract: chunks are weighted by the attention work they actually incur).
//
// One thread per item (s, c, g, t) of the chunk-major index space: query tile t holds blocks
// tP .. tP+P-1 of sample s (P = 1: one block), and c is a run of L consecutive chunks (L = 1: one
// chunk; the item's key range is C' = L*C keys). The cost of an item is the number of key tiles of
// its range holding a key one of its rows sees; with a the tile's largest (last) anchor:
//     nvis = clamp(a - c*C', 0, min(C', S - c*C')),  cost = ceil(nvis / Tk).
// Each chunk of C keys gets the item's key tiles that lie inside it (the chunk costs of the cost
// model do not depend on L).
// Three launches: count visible items per CTA (and validate anchors, add chunk costs), scan the
// CTA counts, then write the compacted (item id, cost) list in ascending id order.
#include "common.cuh"
#include "scan.cuh"

namespace splitkv {

namespace {

constexpr int kThreads = 1024;

__device__ inline int32_t item_cost_of(const Meta& m, const int32_t* anchors, int64_t id, Item* out) {
    Item it = decode_item(m, id);
    int32_t a = anchors[it.j + it.nbt - 1];
    int32_t nvis = visible_in_chunk(m, it.s, it.c, a);
    if (out) *out = it;
    return (nvis + m.key_tile - 1) / m.key_tile;
}

__global__ void __launch_bounds__(kThreads) cost_count_kernel(Meta m, const int32_t* __restrict__ anchors,
                                                              int64_t* __restrict__ chunk_cost,
                                                              int32_t* __restrict__ blk_count,
                                                              int32_t* __restrict__ status) {
    __shared__ int32_t sh[33];
    const int64_t id = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    int32_t vis = 0;
    if (id < m.n_items) {
        Item it;
        int32_t cost = item_cost_of(m, anchors, id, &it);
        // Anchor validation, once per block: at its tile's chunk-0 / head-0 item.
        if (it.c == 0 && it.g == 0) {
            for (int32_t x = 0; x < it.nbt; ++x) {
                int32_t a = anchors[it.j + x];
                if (a < m.block || (int64_t)a >= m.seq_len[it.s]) raise_status(status, SPLITKV_DEV_ANCHOR_RANGE);
                if (it.b + x > 0 && anchors[it.j + x - 1] >= a) raise_status(status, SPLITKV_DEV_ANCHOR_ORDER);
            }
        }
        if (cost > 0) {
            vis = owns_chunk(m, it.s, it.c) ? 1 : 0;  // the chunk costs count every rank's items
            // The item's key tiles, added to the cost chunk (cost_chunk keys) that holds each of them.
            const int32_t a = anchors[it.j + it.nbt - 1];
            for (int32_t x = 0; x < m.runs; ++x) {
                const int64_t cc = (int64_t)it.c * m.runs + x;  // cost chunk of the sample
                const int64_t lo = cc * m.cost_chunk;
                if (lo >= m.seq_len[it.s]) break;
                int64_t n = (int64_t)a - lo, width = m.seq_len[it.s] - lo;
                if (width > m.cost_chunk) width = m.cost_chunk;
                n = n < 0 ? 0 : (n > width ? width : n);
                const int64_t tiles = (n + m.key_tile - 1) / m.key_tile;
                if (tiles > 0)
                    atomicAdd((unsigned long long*)&chunk_cost[m.chunk_base[it.s] + cc], (unsigned long long)tiles);
            }
        }
    }
    int32_t total;
    block_exclusive_scan<int32_t>(vis, sh, &total);
    if (threadIdx.x == 0) blk_count[blockIdx.x] = total;
}

// Single CTA: exclusive scan of the per-CTA visible counts.
__global__ void __launch_bounds__(kThreads) cost_scan_kernel(int32_t nblk, int32_t* __restrict__ blk_count,
                                                             int32_t* __restrict__ n_items) {
    __shared__ int32_t sh[33];
    int32_t carry = 0;
    for (int32_t base = 0; base < nblk; base += kThreads) {
        int32_t i = base + threadIdx.x;
        int32_t x = i < nblk ? blk_count[i] : 0;
        int32_t total;
        int32_t ex = block_exclusive_scan<int32_t>(x, sh, &total);
        if (i < nblk) blk_count[i] = carry + ex;
        carry += total;
    }
    if (threadIdx.x == 0) *n_items = carry;
}

__global__ void __launch_bounds__(kThreads) cost_write_kernel(Meta m, const int32_t* __restrict__ anchors,
                                                              const int32_t* __restrict__ blk_off,
                                                              int32_t* __restrict__ item_id,
                                                              int32_t* __restrict__ item_cost) {
    __shared__ int32_t sh[33];
    const int64_t id = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    int32_t cost = 0;
    if (id < m.n_items) {
        Item it;
        cost = item_cost_of(m, anchors, id, &it);
        if (!owns_chunk(m, it.s, it.c)) cost = 0;  // another rank's item
    }
    if (cost > 0) cost += m.item_overhead;  // the per-item constant of the realized cost
    int32_t vis = cost > 0 ? 1 : 0;
    int32_t ex = block_exclusive_scan<int32_t>(vis, sh, nullptr);
    if (vis) {
        int32_t pos = blk_off[blockIdx.x] + ex;
        item_id[pos] = (int32_t)id;
        item_cost[pos] = cost;
    }
}

}  // namespace

size_t cost_workspace(const Meta& m) {
    size_t nblk = (size_t)((m.n_items + kThreads - 1) / kThreads);
    return align_up(nblk * sizeof(int32_t), 256);
}

cudaError_t launch_cost(const Meta& m, const int32_t* anchors, int32_t* item_id, int32_t* item_cost,
                        int64_t* chunk_cost, int32_t* n_items, int32_t* status, void* ws, cudaStream_t st) {
    int32_t nblk = (int32_t)((m.n_items + kThreads - 1) / kThreads);
    int32_t* blk = (int32_t*)ws;
    cudaError_t e = cudaMemsetAsync(chunk_cost, 0, sizeof(int64_t) * (size_t)m.n_chunks, st);
    if (e != cudaSuccess) return e;
    if (nblk == 0) return cudaMemsetAsync(n_items, 0, sizeof(int32_t), st);
    cost_count_kernel<<<nblk, kThreads, 0, st>>>(m, anchors, chunk_cost, blk, status);
    cost_scan_kernel<<<1, kThreads, 0, st>>>(nblk, blk, n_items);
    cost_write_kernel<<<nblk, kThreads, 0, st>>>(m, anchors, blk, item_id, item_cost);
    return cudaGetLastError();
}

}  // namespace splitkv
