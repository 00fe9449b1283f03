// Shared definitions of the Split-KV CUDA library: problem metadata passed by value to every
// kernel, item decoding, status-word helpers and the internal launcher declarations.
#pragma once

#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/splitkv.h"

namespace splitkv {

constexpr int kMaxBatch = SPLITKV_MAX_BATCH;
constexpr int kMaxCost = 64;  // chunk / key_tile upper bound (planner bucket count)

// Everything a kernel needs to decode an item or a query row, by value (no device copy).
struct Meta {
    int32_t batch;
    int32_t hq, hkv, group, d, block, chunk, key_tile, rows;  // rows = block * group (one block)
    // chunk is the key range of one item: a run of `runs` chunks of cost_chunk keys (runs = 1: the
    // chunk itself). Items, partials, the forward, merge and backward work in units of `chunk`;
    // only the per-chunk costs of the cost pass count in cost_chunk.
    int32_t cost_chunk, runs;
    int32_t item_overhead;  // per-item constant of the realized cost (key-tile units): cost = tiles + this
    int32_t pack, rows_item;              // blocks per query tile; rows_item = pack * rows
    float scale;
    int32_t dtype;
    int64_t n_items;                      // all items, visible or not
    int64_t total_keys;
    int64_t n_queries;
    int64_t n_blocks;
    int64_t n_chunks;
    int64_t seq_len[kMaxBatch];
    int64_t key_off[kMaxBatch + 1];       // first context row of each sample
    int64_t item_base[kMaxBatch + 1];     // first item index of each sample
    int64_t chunk_base[kMaxBatch + 1];    // first cost chunk (cost_chunk keys; sample-major) of each sample
    int32_t anchor_off[kMaxBatch + 1];    // first global block of each sample
    int32_t n_chunk_s[kMaxBatch];         // ceil(S_s / chunk): item chunks of each sample
    // Context parallelism (rank >= 0): this rank keeps only the items of the chunks it owns
    // (chunk_rank[chunk] == rank, device int32[n_chunks]) and the self partials of the blocks j with
    // j % n_ranks == rank. rank < 0: everything (one GPU).
    const int32_t* chunk_rank;
    int32_t rank, n_ranks;
};

// This rank's share of the work (always true without context parallelism).
__device__ __forceinline__ bool owns_chunk(const Meta& m, int s, int32_t c) {
    return m.rank < 0 || __ldg(m.chunk_rank + m.chunk_base[s] + c) == m.rank;
}
__device__ __forceinline__ bool owns_self(const Meta& m, int64_t j) { return m.rank < 0 || j % m.n_ranks == m.rank; }

// Decoded work item: query tile t of sample s (blocks b .. b + nbt - 1 of the sample) against chunk c
// at kv head g.
struct Item {
    int32_t s, c, g, b;   // sample, chunk, kv head, first block of the tile within its sample
    int32_t j;            // its global block index = anchor_off[s] + b
    int32_t nbt;          // blocks in the tile: min(pack, blocks of the sample - b)
};

__host__ __device__ inline int sample_of_item(const Meta& m, int64_t id) {
    int s = 0;
    while (s + 1 < m.batch && id >= m.item_base[s + 1]) ++s;
    return s;
}

__host__ __device__ inline Item decode_item(const Meta& m, int64_t id) {
    Item it;
    it.s = sample_of_item(m, id);
    int64_t local = id - m.item_base[it.s];
    int32_t nb = m.anchor_off[it.s + 1] - m.anchor_off[it.s];
    int32_t nt = (nb + m.pack - 1) / m.pack;
    int32_t tile = (int32_t)(local % nt);
    int64_t t = local / nt;
    it.g = (int32_t)(t % m.hkv);
    it.c = (int32_t)(t / m.hkv);
    it.b = tile * m.pack;
    it.j = m.anchor_off[it.s] + it.b;
    it.nbt = nb - it.b < m.pack ? nb - it.b : m.pack;
    return it;
}

__host__ __device__ inline int sample_of_block(const Meta& m, int32_t j) {
    int s = 0;
    while (s + 1 < m.batch && j >= m.anchor_off[s + 1]) ++s;
    return s;
}

// Keys of item chunk c (chunk keys from c * chunk) that a block with anchor a sees (context keys [0, a)).
__host__ __device__ inline int32_t visible_in_chunk(const Meta& m, int s, int c, int32_t a) {
    int64_t lo = (int64_t)c * m.chunk;
    int64_t width = m.seq_len[s] - lo;
    if (width > m.chunk) width = m.chunk;
    int64_t n = (int64_t)a - lo;
    if (n < 0) n = 0;
    if (n > width) n = width;
    return (int32_t)n;
}

__device__ inline void raise_status(int32_t* status, int32_t bits) {
    if (status) atomicOr(status, bits);
}

__device__ inline bool status_bad(const int32_t* status) {
    return status && *((volatile const int32_t*)status) != 0;
}

// Records a failure detail for splitkv_last_error() (thread-local) and passes the error through.
cudaError_t note_error(cudaError_t e, const char* what);
void clear_error();

// ---- internal launchers (defined in the per-kernel .cu files) ----
cudaError_t launch_cost(const Meta& m, const int32_t* anchors, int32_t* item_id, int32_t* item_cost,
                        int64_t* chunk_cost, int32_t* n_items, int32_t* status, void* ws, cudaStream_t st);
size_t cost_workspace(const Meta& m);

cudaError_t launch_plan(const int32_t* item_cost, const int32_t* n_items, int32_t max_items, int32_t max_cost,
                        int32_t n_workers, int32_t* item_worker, int32_t* queue_off, int32_t* queue_items,
                        int64_t* load, int32_t* status, void* ws, cudaStream_t st);
size_t plan_workspace(int32_t max_items, int32_t max_cost, int32_t n_workers);
// Device address of the planner's static scratch array on the current device (looked up once per device).
constexpr size_t kStaticPlanScratchBytes = (size_t)4 << 20;
constexpr int kMaxDevices = 64;
cudaError_t static_plan_scratch(void** out);

cudaError_t launch_fwd_simt(const Meta& m, const void* q, const void* k, const void* v, const void* kb,
                            const void* vb, const int32_t* anchors, const int32_t* item_id, const int32_t* queue_off,
                            const int32_t* queue_items, int32_t n_workers, void* o_part, float* lse_part,
                            int32_t* status, cudaStream_t st);

cudaError_t launch_fwd_tc(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                          const int32_t* anchors, const int32_t* item_id, const int32_t* queue_off,
                          const int32_t* queue_items, int32_t n_workers, void* o_part, float* lse_part,
                          int32_t* status, void* ws, int32_t flags, cudaStream_t st);
bool fwd_tc_supported(const Meta& m);
// Pairs of SMs (two-CTA clusters, cta_group::2 MMAs) for 256-row items: n_workers queues, 2 CTAs each.
cudaError_t launch_fwd_tc2(const Meta& m, const void* q, const void* k, const void* v, const void* kb,
                           const void* vb, const int32_t* anchors, const int32_t* item_id, const int32_t* queue_off,
                           const int32_t* queue_items, int32_t n_workers, void* o_part, float* lse_part,
                           int32_t* status, void* ws, int32_t flags, cudaStream_t st);
bool fwd_tc2_supported(const Meta& m);
cudaError_t fwd_tc2_max_workers(int32_t* out);
constexpr size_t kFwdWorkspaceBytes = 256;  // the tensor-core forward's pool counter

cudaError_t launch_merge(const Meta& m, const void* o_part, const float* lse_part, const int32_t* anchors, void* o,
                         float* lse, int32_t* status, cudaStream_t st);
cudaError_t launch_merge_ranks(const Meta& m, int32_t n_ranks, const void* o_ranks, const float* lse_ranks, void* o,
                               float* lse, int32_t* status, cudaStream_t st);

bool bwd_tc_supported(const Meta& m);
size_t bwd_tc_workspace(const Meta& m);
cudaError_t launch_bwd_tc(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                          const void* o, const float* lse, const void* dout, const int32_t* anchors, float* dq,
                          float* dk, float* dv, float* dkb, float* dvb, int32_t* status, void* ws, cudaStream_t st);

cudaError_t launch_bwd(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb,
                       const void* o, const float* lse, const void* dout, const int32_t* anchors, float* dq,
                       float* dk, float* dv, float* dkb, float* dvb, int32_t* status, void* ws, cudaStream_t st);
size_t bwd_workspace(const Meta& m);

// ---- small device helpers ----
template <typename T> __device__ inline float to_f32(T x);
template <> __device__ inline float to_f32<float>(float x) { return x; }
template <> __device__ inline float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ inline T from_f32(float x);
template <> __device__ inline float from_f32<float>(float x) { return x; }
template <> __device__ inline __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace splitkv
