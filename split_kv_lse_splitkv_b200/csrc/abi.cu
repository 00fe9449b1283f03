// C ABI entry points: host-side validation, problem decoding and kernel launches.
// Every check here runs before anything is enqueued, so a rejected call launches nothing.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#include "common.cuh"

#define SPLITKV_API extern "C" __attribute__((visibility("default")))

namespace splitkv {

static thread_local char g_last_error[256];

cudaError_t note_error(cudaError_t e, const char* what) {
    if (e != cudaSuccess)
        std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", what, cudaGetErrorName(e),
                      cudaGetErrorString(e));
    return e;
}

void clear_error() { g_last_error[0] = 0; }

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Fill `m` from a host problem; returns SPLITKV_OK or a negative code.
int build_meta(const splitkv_problem* p, Meta* m) {
    if (!p || !m) return SPLITKV_EINVAL;
    std::memset(m, 0, sizeof(Meta));
    if (p->batch < 1 || p->batch > kMaxBatch || !p->seq_len || !p->anchor_off) return SPLITKV_EINVAL;
    if (p->n_q_heads < 1 || p->n_kv_heads < 1 || p->n_q_heads % p->n_kv_heads) return SPLITKV_EINVAL;
    if (p->block < 1 || p->chunk < 1 || p->key_tile < 1 || p->head_dim < 1) return SPLITKV_EINVAL;
    const int32_t runs = p->chunks_per_item == 0 ? 1 : p->chunks_per_item;
    if (runs < 1 || p->item_overhead < 0) return SPLITKV_EINVAL;
    if (p->chunk % p->key_tile || (int64_t)p->chunk * runs / p->key_tile + p->item_overhead > kMaxCost)
        return SPLITKV_EUNSUPPORTED;
    if (!(p->scale > 0.f) || p->scale != p->scale) return SPLITKV_EINVAL;
    if (p->dtype != SPLITKV_F32 && p->dtype != SPLITKV_BF16) return SPLITKV_EUNSUPPORTED;
    if (p->head_dim % 4 || p->head_dim > 128 || p->head_dim < 8) return SPLITKV_EUNSUPPORTED;
    if (p->dtype == SPLITKV_BF16 && p->head_dim % 8) return SPLITKV_EUNSUPPORTED;
    if (p->block > 32) return SPLITKV_EUNSUPPORTED;
    m->batch = p->batch;
    m->hq = p->n_q_heads;
    m->hkv = p->n_kv_heads;
    m->group = p->n_q_heads / p->n_kv_heads;
    m->d = p->head_dim;
    m->block = p->block;
    m->chunk = p->chunk * runs;  // an item's key range: a run of `runs` chunks
    m->cost_chunk = p->chunk;
    m->runs = runs;
    m->item_overhead = p->item_overhead;
    m->key_tile = p->key_tile;
    m->rows = p->block * m->group;
    m->pack = p->blocks_per_item == 0 ? 1 : p->blocks_per_item;
    if (m->pack < 1 || m->pack > 64) return SPLITKV_EINVAL;
    m->rows_item = m->pack * m->rows;
    if (m->rows_item > 256) return SPLITKV_EUNSUPPORTED;
    m->scale = p->scale;
    m->dtype = p->dtype;
    if (p->anchor_off[0] != 0) return SPLITKV_EINVAL;
    m->chunk_rank = nullptr;
    m->rank = -1;  // no context parallelism unless a rank entry point sets it
    m->n_ranks = 1;
    int64_t items = 0, keys = 0, chunks = 0;
    for (int s = 0; s < p->batch; ++s) {
        int64_t S = p->seq_len[s];
        int32_t nb = p->anchor_off[s + 1] - p->anchor_off[s];
        if (S < 1 || nb < 0) return SPLITKV_EINVAL;
        int64_t nc = (S + m->chunk - 1) / m->chunk;        // item chunks
        int64_t ncc = (S + p->chunk - 1) / p->chunk;       // cost chunks
        m->seq_len[s] = S;
        m->key_off[s] = keys;
        m->item_base[s] = items;
        m->chunk_base[s] = chunks;
        m->anchor_off[s] = p->anchor_off[s];
        m->n_chunk_s[s] = (int32_t)nc;
        if (nc > INT32_MAX) return SPLITKV_EUNSUPPORTED;
        keys += S;
        chunks += ncc;
        items += nc * m->hkv * ((nb + m->pack - 1) / m->pack);
    }
    m->key_off[p->batch] = keys;
    m->item_base[p->batch] = items;
    m->chunk_base[p->batch] = chunks;
    m->anchor_off[p->batch] = p->anchor_off[p->batch];
    m->n_items = items;
    m->total_keys = keys;
    m->n_chunks = chunks;
    m->n_blocks = p->anchor_off[p->batch];
    m->n_queries = m->n_blocks * p->block;
    if (items >= INT32_MAX || m->n_queries * m->hq >= ((int64_t)1 << 40)) return SPLITKV_EUNSUPPORTED;
    return SPLITKV_OK;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return SPLITKV_OK;
    if (!g_last_error[0]) note_error(e, "kernel launch");
    return SPLITKV_ECUDA;
}

}  // namespace
}  // namespace splitkv

using namespace splitkv;

SPLITKV_API int splitkv_query(const splitkv_problem* problem, splitkv_sizes* out) {
    Meta m;
    int rc = build_meta(problem, &m);
    if (rc) return rc;
    if (!out) return SPLITKV_EINVAL;
    out->n_items_max = m.n_items;
    out->n_chunks = m.n_chunks;
    out->n_queries = m.n_queries;
    out->total_keys = m.total_keys;
    out->n_blocks = m.n_blocks;
    out->o_part_elems = (m.n_items + m.n_blocks * m.hkv) * m.rows_item * m.d;
    out->lse_part_elems = (m.n_items + m.n_blocks * m.hkv) * m.rows_item;
    out->max_cost = m.chunk / m.key_tile + m.item_overhead;
    out->rows_per_item = m.rows_item;
    out->ctas_per_worker = fwd_tc2_supported(m) ? 2 : 1;
    return SPLITKV_OK;
}

SPLITKV_API size_t splitkv_workspace_size(const splitkv_problem* problem, int32_t n_workers) {
    Meta m;
    if (build_meta(problem, &m) || n_workers < 1 || n_workers > 1024) return 0;
    size_t a = cost_workspace(m);
    size_t b = plan_workspace((int32_t)m.n_items, m.chunk / m.key_tile + m.item_overhead, n_workers);
    size_t c = bwd_workspace(m);
    if (kFwdWorkspaceBytes > c) c = kFwdWorkspaceBytes;
    if (bwd_tc_workspace(m) > c) c = bwd_tc_workspace(m);
    size_t r = a > b ? a : b;
    return r > c ? r : c;
}

SPLITKV_API int splitkv_max_workers(const splitkv_problem* problem, int32_t* n_workers) {
    clear_error();
    Meta m;
    int rc = build_meta(problem, &m);
    if (rc) return rc;
    if (!n_workers) return SPLITKV_EINVAL;
    if (fwd_tc2_supported(m)) return cuda_status(fwd_tc2_max_workers(n_workers));
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_status(note_error(e, "cudaDeviceGetAttribute(multiprocessor count)"));
    *n_workers = sms;
    return SPLITKV_OK;
}

SPLITKV_API const char* splitkv_last_error(void) { return g_last_error; }

// The build script passes the sha256 of the library's sources; other builds say "unknown".
#ifndef SPLITKV_SOURCE_SHA
#define SPLITKV_SOURCE_SHA "unknown"
#endif
SPLITKV_API const char* splitkv_build_id(void) { return SPLITKV_SOURCE_SHA; }

SPLITKV_API const char* splitkv_strerror(int code) {
    switch (code) {
        case SPLITKV_OK: return "ok";
        case SPLITKV_EINVAL: return "invalid argument";
        case SPLITKV_EUNSUPPORTED: return "unsupported problem";
        case SPLITKV_ECUDA: return "CUDA call failed";
        case SPLITKV_ENOSPACE: return "workspace too small";
        default: return "unknown status";
    }
}

SPLITKV_API int splitkv_cost(const splitkv_problem* problem, const int32_t* anchors_d, int32_t* item_id_d,
                             int32_t* item_cost_d, int64_t* chunk_cost_d, int32_t* n_items_d, int32_t* status_d,
                             void* workspace_d, size_t workspace_bytes, void* stream) {
    clear_error();
    Meta m;
    int rc = build_meta(problem, &m);
    if (rc) return rc;
    if ((m.n_blocks && !anchors_d) || !item_id_d || !item_cost_d || !chunk_cost_d || !n_items_d || !status_d)
        return SPLITKV_EINVAL;
    if (!workspace_d || workspace_bytes < cost_workspace(m)) return SPLITKV_ENOSPACE;
    return cuda_status(launch_cost(m, anchors_d, item_id_d, item_cost_d, chunk_cost_d, n_items_d, status_d,
                                   workspace_d, (cudaStream_t)stream));
}

// ---------------------------------------------------------------- context parallelism across ranks
SPLITKV_API int splitkv_cp_plan(const int64_t* chunk_cost_h, int64_t n_chunks, int32_t n_ranks, int32_t* chunk_rank_h,
                                int64_t* rank_load_h) {
    clear_error();
    if (n_chunks < 0 || n_ranks < 1 || (n_chunks > 0 && (!chunk_cost_h || !chunk_rank_h)) || !rank_load_h)
        return SPLITKV_EINVAL;
    for (int64_t c = 0; c < n_chunks; ++c)
        if (chunk_cost_h[c] < 0) return SPLITKV_EINVAL;
    // LPT: chunks by (cost descending, index ascending), each to the least (load, rank).
    std::vector<int64_t> order((size_t)n_chunks);
    for (int64_t c = 0; c < n_chunks; ++c) order[(size_t)c] = c;
    std::stable_sort(order.begin(), order.end(),
                     [&](int64_t a, int64_t b) { return chunk_cost_h[a] > chunk_cost_h[b]; });
    using Entry = std::pair<int64_t, int32_t>;  // (load, rank): the smallest on top
    std::priority_queue<Entry, std::vector<Entry>, std::greater<Entry>> heap;
    for (int32_t r = 0; r < n_ranks; ++r) {
        heap.push({0, r});
        rank_load_h[r] = 0;
    }
    for (int64_t c : order) {
        Entry e = heap.top();
        heap.pop();
        chunk_rank_h[c] = e.second;
        e.first += chunk_cost_h[c];
        rank_load_h[e.second] = e.first;
        heap.push(e);
    }
    return SPLITKV_OK;
}

namespace {
int rank_meta(const splitkv_problem* problem, const int32_t* chunk_rank_d, int32_t rank, int32_t n_ranks, Meta* m) {
    int rc = build_meta(problem, m);
    if (rc) return rc;
    if (m->runs != 1) return SPLITKV_EUNSUPPORTED;  // ranks own chunks: an item must lie in one chunk
    if (n_ranks < 1 || rank < 0 || rank >= n_ranks || (m->n_chunks > 0 && !chunk_rank_d)) return SPLITKV_EINVAL;
    m->chunk_rank = chunk_rank_d;
    m->rank = rank;
    m->n_ranks = n_ranks;
    return SPLITKV_OK;
}
}  // namespace

SPLITKV_API int splitkv_cost_rank(const splitkv_problem* problem, const int32_t* anchors_d, const int32_t* chunk_rank_d,
                                  int32_t rank, int32_t n_ranks, int32_t* item_id_d, int32_t* item_cost_d,
                                  int64_t* chunk_cost_d, int32_t* n_items_d, int32_t* status_d, void* workspace_d,
                                  size_t workspace_bytes, void* stream) {
    clear_error();
    Meta m;
    int rc = rank_meta(problem, chunk_rank_d, rank, n_ranks, &m);
    if (rc) return rc;
    if ((m.n_blocks && !anchors_d) || !item_id_d || !item_cost_d || !chunk_cost_d || !n_items_d || !status_d)
        return SPLITKV_EINVAL;
    if (!workspace_d || workspace_bytes < cost_workspace(m)) return SPLITKV_ENOSPACE;
    return cuda_status(launch_cost(m, anchors_d, item_id_d, item_cost_d, chunk_cost_d, n_items_d, status_d,
                                   workspace_d, (cudaStream_t)stream));
}

SPLITKV_API int splitkv_lse_merge_rank(const splitkv_problem* problem, const void* o_part, const float* lse_part,
                                       const int32_t* anchors_d, const int32_t* chunk_rank_d, int32_t rank,
                                       int32_t n_ranks, void* o_r, float* lse_r, int32_t* status_d, void* stream) {
    clear_error();
    Meta m;
    int rc = rank_meta(problem, chunk_rank_d, rank, n_ranks, &m);
    if (rc) return rc;
    if (!o_part || !lse_part || (m.n_queries > 0 && (!o_r || !lse_r)) || !status_d) return SPLITKV_EINVAL;
    if (m.n_blocks && !anchors_d) return SPLITKV_EINVAL;
    if (!aligned16(o_part) || !aligned16(lse_part) || !aligned16(o_r)) return SPLITKV_EINVAL;
    return cuda_status(launch_merge(m, o_part, lse_part, anchors_d, o_r, lse_r, status_d, (cudaStream_t)stream));
}

SPLITKV_API int splitkv_lse_merge_ranks(const splitkv_problem* problem, int32_t n_ranks, const void* o_ranks,
                                        const float* lse_ranks, void* o, float* lse, int32_t* status_d, void* stream) {
    clear_error();
    Meta m;
    int rc = build_meta(problem, &m);
    if (rc) return rc;
    if (n_ranks < 1 || !status_d || (m.n_queries > 0 && (!o_ranks || !lse_ranks || !o || !lse))) return SPLITKV_EINVAL;
    return cuda_status(launch_merge_ranks(m, n_ranks, o_ranks, lse_ranks, o, lse, status_d, (cudaStream_t)stream));
}

SPLITKV_API int splitkv_plan_lpt(const int32_t* item_cost_d, const int32_t* n_items_d, int32_t max_items,
                                 int32_t max_cost, int32_t n_workers, int32_t* item_worker_d, int32_t* queue_off_d,
                                 int32_t* queue_items_d, int64_t* load_d, int32_t* status_d, void* workspace_d,
                                 size_t workspace_bytes, void* stream) {
    clear_error();
    if (max_items < 0 || max_cost < 1 || max_cost > kMaxCost || n_workers < 1 || n_workers > 1024)
        return SPLITKV_EINVAL;
    if (!item_cost_d || !n_items_d || !item_worker_d || !queue_off_d || !queue_items_d || !load_d || !status_d)
        return SPLITKV_EINVAL;
    if (!workspace_d || workspace_bytes < plan_workspace(max_items, max_cost, n_workers)) return SPLITKV_ENOSPACE;
    return cuda_status(launch_plan(item_cost_d, n_items_d, max_items, max_cost, n_workers, item_worker_d,
                                   queue_off_d, queue_items_d, load_d, status_d, workspace_d, (cudaStream_t)stream));
}

SPLITKV_API int splitkv_plan_lpt_noalloc(const int32_t* item_cost_d, const int32_t* n_items_d, int32_t max_items,
                                         int32_t max_cost, int32_t n_workers, int32_t* item_worker_d,
                                         int32_t* queue_off_d, int32_t* queue_items_d, int64_t* load_d,
                                         int32_t* status_d, void* stream) {
    clear_error();
    if (max_items < 0 || max_cost < 1 || max_cost > kMaxCost || n_workers < 1 || n_workers > 1024)
        return SPLITKV_EINVAL;
    if (!item_cost_d || !n_items_d || !item_worker_d || !queue_off_d || !queue_items_d || !load_d || !status_d)
        return SPLITKV_EINVAL;
    const size_t need = plan_workspace(max_items, max_cost, n_workers);
    if (need > kStaticPlanScratchBytes) {
        std::snprintf(g_last_error, sizeof(g_last_error),
                      "splitkv_plan_lpt_noalloc: needs %zu bytes of scratch, the static array holds %zu", need,
                      kStaticPlanScratchBytes);
        return SPLITKV_ENOSPACE;
    }
    void* ws = nullptr;
    if (static_plan_scratch(&ws) != cudaSuccess) return SPLITKV_ECUDA;
    return cuda_status(launch_plan(item_cost_d, n_items_d, max_items, max_cost, n_workers, item_worker_d,
                                   queue_off_d, queue_items_d, load_d, status_d, ws, (cudaStream_t)stream));
}

SPLITKV_API int splitkv_attn_fwd(const splitkv_problem* problem, const void* q, const void* k, const void* v,
                                 const void* kb, const void* vb, const int32_t* anchors_d, const int32_t* item_id_d,
                                 const int32_t* queue_off_d,
                                 const int32_t* queue_items_d, int32_t n_workers, void* o_part, float* lse_part,
                                 int32_t* status_d, int32_t flags, void* workspace_d, size_t workspace_bytes,
                                 void* stream) {
    clear_error();
    Meta m;
    int rc = build_meta(problem, &m);
    if (rc) return rc;
    if (n_workers < 1 || n_workers > 65535 || (flags & ~(SPLITKV_FWD_SIMT | SPLITKV_FWD_TEST_STARVE)))
        return SPLITKV_EINVAL;
    // Query-side buffers are empty (possibly NULL) when the problem has no anchor at all.
    const bool queries = m.n_queries > 0;
    if ((queries && (!q || !kb || !vb)) || !k || !v || !item_id_d || !queue_off_d || !queue_items_d || !o_part ||
        !lse_part || !status_d)
        return SPLITKV_EINVAL;
    if (m.n_blocks && !anchors_d) return SPLITKV_EINVAL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kb) || !aligned16(vb) || !aligned16(o_part))
        return SPLITKV_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    if (!(flags & SPLITKV_FWD_SIMT) && fwd_tc2_supported(m)) {
        if (!workspace_d || workspace_bytes < kFwdWorkspaceBytes) return SPLITKV_ENOSPACE;
        if (!aligned16(workspace_d)) return SPLITKV_EINVAL;
        if (n_workers > 32767) return SPLITKV_EINVAL;  // two CTAs per worker
        return cuda_status(launch_fwd_tc2(m, q, k, v, kb, vb, anchors_d, item_id_d, queue_off_d, queue_items_d,
                                          n_workers, o_part, lse_part, status_d, workspace_d, flags, st));
    }
    if (!(flags & SPLITKV_FWD_SIMT) && fwd_tc_supported(m)) {
        if (!workspace_d || workspace_bytes < kFwdWorkspaceBytes) return SPLITKV_ENOSPACE;
        if (!aligned16(workspace_d)) return SPLITKV_EINVAL;
        return cuda_status(launch_fwd_tc(m, q, k, v, kb, vb, anchors_d, item_id_d, queue_off_d, queue_items_d,
                                         n_workers, o_part, lse_part, status_d, workspace_d, flags, st));
    }
    if (flags & SPLITKV_FWD_TEST_STARVE) return SPLITKV_EUNSUPPORTED;  // a tensor-core path test
    return cuda_status(launch_fwd_simt(m, q, k, v, kb, vb, anchors_d, item_id_d, queue_off_d, queue_items_d,
                                       n_workers, o_part, lse_part, status_d, st));
}

SPLITKV_API int splitkv_lse_merge(const splitkv_problem* problem, const void* o_part, const float* lse_part,
                                  const int32_t* anchors_d, void* o, float* lse, int32_t* status_d, void* stream) {
    clear_error();
    Meta m;
    int rc = build_meta(problem, &m);
    if (rc) return rc;
    if (!o_part || !lse_part || (m.n_queries > 0 && (!o || !lse)) || !status_d) return SPLITKV_EINVAL;
    if (m.n_blocks && !anchors_d) return SPLITKV_EINVAL;
    if (!aligned16(o_part) || !aligned16(lse_part) || !aligned16(o)) return SPLITKV_EINVAL;
    return cuda_status(launch_merge(m, o_part, lse_part, anchors_d, o, lse, status_d, (cudaStream_t)stream));
}

namespace {
int attn_bwd(const Meta& m, const void* q, const void* k, const void* v, const void* kb, const void* vb, const void* o,
             const float* lse, const void* dout, const int32_t* anchors_d, float* dq, float* dk, float* dv, float* dkb,
             float* dvb, int32_t* status_d, void* workspace_d, size_t workspace_bytes, void* stream) {
    const bool queries = m.n_queries > 0;  // without any anchor the query-side buffers are empty
    if ((queries && (!q || !kb || !vb || !o || !lse || !dout || !dq || !dkb || !dvb)) || !k || !v || !dk || !dv ||
        !status_d)
        return SPLITKV_EINVAL;
    if (m.n_blocks && !anchors_d) return SPLITKV_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    if (bwd_tc_supported(m)) {
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kb) || !aligned16(vb) || !aligned16(dout) ||
            !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dkb) || !aligned16(dvb))
            return SPLITKV_EINVAL;
        if (!workspace_d || workspace_bytes < bwd_tc_workspace(m)) return SPLITKV_ENOSPACE;
        return cuda_status(
            launch_bwd_tc(m, q, k, v, kb, vb, o, lse, dout, anchors_d, dq, dk, dv, dkb, dvb, status_d, workspace_d, st));
    }
    if (!workspace_d || workspace_bytes < bwd_workspace(m)) return SPLITKV_ENOSPACE;
    return cuda_status(launch_bwd(m, q, k, v, kb, vb, o, lse, dout, anchors_d, dq, dk, dv, dkb, dvb, status_d,
                                  workspace_d, st));
}
}  // namespace

SPLITKV_API int splitkv_attn_bwd(const splitkv_problem* problem, const void* q, const void* k, const void* v,
                                 const void* kb, const void* vb, const void* o, const float* lse, const void* dout,
                                 const int32_t* anchors_d, float* dq, float* dk, float* dv, float* dkb, float* dvb,
                                 int32_t* status_d, void* workspace_d, size_t workspace_bytes, void* stream) {
    clear_error();
    Meta m;
    int rc = build_meta(problem, &m);
    if (rc) return rc;
    return attn_bwd(m, q, k, v, kb, vb, o, lse, dout, anchors_d, dq, dk, dv, dkb, dvb, status_d, workspace_d,
                    workspace_bytes, stream);
}

SPLITKV_API int splitkv_attn_bwd_rank(const splitkv_problem* problem, const void* q, const void* k, const void* v,
                                      const void* kb, const void* vb, const void* o, const float* lse,
                                      const void* dout, const int32_t* anchors_d, const int32_t* chunk_rank_d,
                                      int32_t rank, int32_t n_ranks, float* dq, float* dk, float* dv, float* dkb,
                                      float* dvb, int32_t* status_d, void* workspace_d, size_t workspace_bytes,
                                      void* stream) {
    clear_error();
    Meta m;
    int rc = rank_meta(problem, chunk_rank_d, rank, n_ranks, &m);
    if (rc) return rc;
    return attn_bwd(m, q, k, v, kb, vb, o, lse, dout, anchors_d, dq, dk, dv, dkb, dvb, status_d, workspace_d,
                    workspace_bytes, stream);
}
