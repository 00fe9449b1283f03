/*
 * splitkv.h — C ABI of the Split-KV hot path on one GPU (sm_100a).
 *
 * Operation (Split-KV: Efficient Context Parallelism for Training Diffusion Drafters, Abstract):
 * the exact block-sparse cross-attention of a short set of anchor-sampled draft queries over a
 * long context. Each anchor a opens a draft block of `block` queries; every query of that block
 * attends bidirectionally to the context keys [0, a) of its sample plus the block's own `block`
 * keys (Kb/Vb). The context K/V is cut into chunks of `chunk` keys; each chunk yields a
 * query-sized partial output O_c plus a per-row log-sum-exp LSE_c, and the partials are merged
 * exactly: L = log sum_c exp(LSE_c), O = sum_c exp(LSE_c - L) O_c. A cost-aware
 * longest-processing-time-first (LPT) planner assigns the (chunk, kv head, block) work items,
 * weighted by their realized cost (visible key tiles), to per-worker queues — here the workers
 * are the SMs of one GPU.
 *
 * Conventions for every entry point
 *   - The caller owns every buffer. The library never allocates device or host memory and never
 *     synchronizes the host with the device. All work is enqueued on `stream` (a cudaStream_t
 *     passed as void*; NULL = legacy default stream).
 *   - Pointers named *_d and the tensor arguments are DEVICE pointers; `problem` and the arrays it
 *     points to are HOST memory, read only during the call.
 *   - Tensors are dense, row-major, innermost dimension last, 16-byte aligned.
 *       q, o, dout          [Nq, Hq, d]      Nq = block * total anchors; rows block*j .. block*j+block-1
 *                                            belong to global block j (the j-th anchor over all samples)
 *       k, v, dk, dv        [sum S, Hkv, d]  samples packed one after another
 *       kb, vb, dkb, dvb    [Nq, Hkv, d]     each block's own keys / values
 *       lse                 [Nq, Hq]         float32, natural log
 *     Query head h reads kv head h / (Hq/Hkv).
 *     A problem without any anchor (Nq = 0) has nothing to compute: its query-side tensors (q, o,
 *     dout, kb, vb, lse, dq, dkb, dvb) and anchors_d are empty and may be NULL; the calls then
 *     write only what has keys (chunk_cost = 0, n_items = 0, an empty plan, dK = dV = 0).
 *   - Return value: SPLITKV_OK, or a negative code detected on the host BEFORE anything is
 *     enqueued (nothing was launched), or SPLITKV_ECUDA if a launch failed. Errors that only the
 *     device can see (bad anchors, costs out of range, an in-kernel wait that ran out) are ORed into
 *     the device status word `status_d` (int32, caller zeroes it once); every kernel reads it first
 *     and skips its work if it is already non-zero. Nothing traps.
 */
#ifndef SPLITKV_H
#define SPLITKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host-side return codes. */
#define SPLITKV_OK 0
#define SPLITKV_EINVAL (-1)       /* null pointer, bad size, misaligned tensor, bad problem    */
#define SPLITKV_EUNSUPPORTED (-2) /* well-formed but not supported (dtype / head_dim / shape)  */
#define SPLITKV_ECUDA (-3)        /* a CUDA runtime or driver call failed                      */
#define SPLITKV_ENOSPACE (-4)     /* workspace smaller than splitkv_workspace_size()           */

/* Bits of the device status word. */
#define SPLITKV_DEV_ANCHOR_ORDER 0x1 /* anchors of a sample not strictly ascending                 */
#define SPLITKV_DEV_ANCHOR_RANGE 0x2 /* an anchor outside [block, S)                               */
#define SPLITKV_DEV_BAD_COST 0x4     /* planner input: a cost outside [1, max_cost] or too many items */
#define SPLITKV_DEV_BAD_PLAN 0x8     /* a queue entry or item id out of range                      */
#define SPLITKV_DEV_TIMEOUT 0x10     /* an in-kernel wait passed its time limit; the kernel returned */
#define SPLITKV_DEV_SMEM_ALIGN 0x20  /* dynamic shared memory not 1024-byte aligned; the backward returned */

/* Element types of q, k, v, kb, vb, o, dout. Accumulation is always float32. */
#define SPLITKV_F32 0
#define SPLITKV_BF16 1

/* Largest batch (number of samples) one problem may hold. */
#define SPLITKV_MAX_BATCH 64

/* Flags of splitkv_attn_fwd. */
#define SPLITKV_FWD_DEFAULT 0 /* bf16 with head_dim 128: tcgen05/TMEM/TMA kernel; else SIMT fp32 */
#define SPLITKV_FWD_SIMT 1    /* force the CUDA-core kernel (any dtype): an independent GPU cross-check */
/* Test of the in-kernel wait limit (tensor-core path only; EUNSUPPORTED elsewhere): the first CTA
 * (cluster) is given no item and its waits a 20 us limit instead of 2 s, so it gives up before issuing
 * any copy or MMA and the call ends with SPLITKV_DEV_TIMEOUT in status_d; the other CTAs run their
 * queues. The partials of the first queue are not written. The next call on the same device, with
 * status_d cleared, computes normally. */
#define SPLITKV_FWD_TEST_STARVE 0x100

/* Problem description (host memory). */
typedef struct {
    int32_t batch;              /* samples B, 1..SPLITKV_MAX_BATCH                                */
    const int64_t *seq_len;     /* host [B]: context length S_s >= 1                               */
    const int32_t *anchor_off;  /* host [B+1]: sample s owns anchors[anchor_off[s] .. anchor_off[s+1]) */
    int32_t n_q_heads;          /* Hq                                                               */
    int32_t n_kv_heads;         /* Hkv, divides Hq                                                  */
    int32_t head_dim;           /* d: 128 for bf16; 8..128 (multiple of 4) for f32                  */
    int32_t block;              /* queries per draft block (16)                                     */
    int32_t chunk;              /* context chunk C, a multiple of key_tile                          */
    int32_t key_tile;           /* Tk, the key tile of the cost model (a divisor of chunk): it sets
                                   the unit of the costs and the plan, not the kernels' tiling      */
    float scale;                /* score scale, normally 1/sqrt(d)                                  */
    int32_t dtype;              /* SPLITKV_F32 or SPLITKV_BF16                                      */
    int32_t blocks_per_item;    /* P: consecutive blocks of a sample sharing one query tile (0 = 1);
                                   an item is then (sample, chunk, kv head, tile of P blocks). The
                                   tensor-core forward runs P * block * G <= 128 on one SM per
                                   worker and P * block * G = 256 (P even, P * block <= 128) on a
                                   pair of SMs per worker                                            */
    int32_t chunks_per_item;    /* L: consecutive chunks one item covers (0 = 1). An item is then
                                   (sample, run of L chunks, kv head, query tile): its worker carries
                                   the softmax across the run and leaves one partial per run (L times
                                   fewer partials to write and merge). chunk_cost_d stays per chunk.
                                   L * chunk / key_tile + item_overhead <= 64                         */
    int32_t item_overhead;      /* kappa >= 0: per-item constant of the realized cost, in key tiles (0 by
                                   default): a visible item costs tiles + kappa in the plan, for the work
                                   every item carries (its query tile, its partial). Chunk costs count
                                   key tiles only                                                    */
} splitkv_problem;

/* Derived sizes of a problem. */
typedef struct {
    int64_t n_items_max;    /* every (sample, run of chunks, kv head, query tile) item, visible or not */
    int64_t n_chunks;       /* sum_s ceil(S_s / chunk): length of chunk_cost_d                       */
    int64_t n_queries;      /* Nq                                                                     */
    int64_t total_keys;     /* sum_s S_s                                                              */
    int64_t n_blocks;       /* total anchors                                                          */
    int64_t o_part_elems;   /* elements of o_part, in the problem dtype (bf16 or float32):
                               (n_items_max + n_blocks*Hkv) * rows * d                               */
    int64_t lse_part_elems; /* float32 elements of lse_part: (n_items_max + n_blocks*Hkv) * rows       */
    int32_t max_cost;       /* L * chunk / key_tile + item_overhead: the largest item cost            */
    int32_t rows_per_item;  /* rows = P * block * G: query rows of one item (its query tile)          */
    int32_t ctas_per_worker;/* SMs that run one worker's queue in splitkv_attn_fwd's default path: 2
                               for 256-row items (a pair of SMs), else 1. Plan onto (SM count) /
                               ctas_per_worker workers for one queue per SM or pair.               */
} splitkv_sizes;

/* Fill `out` for `problem`. Returns SPLITKV_EINVAL / SPLITKV_EUNSUPPORTED for a bad problem. */
int splitkv_query(const splitkv_problem *problem, splitkv_sizes *out);

/* Bytes of scratch that splitkv_cost, splitkv_plan_lpt and splitkv_attn_bwd need for this problem
 * with `n_workers` queues (0 on a bad problem). One buffer of this size serves every call. */
size_t splitkv_workspace_size(const splitkv_problem *problem, int32_t n_workers);

/* Largest worker count whose queues all run at once on the current device in splitkv_attn_fwd's
 * default path: the SM count for one-SM workers, the number of two-CTA clusters the device holds at
 * once for pair workers (sizes.ctas_per_worker = 2; a GPC with an odd number of usable SMs leaves
 * one SM unpaired). The plan should use at most this many workers: more queues than fit run in a
 * second wave. Returns SPLITKV_ECUDA without a usable device. */
int splitkv_max_workers(const splitkv_problem *problem, int32_t *n_workers);

/* Human-readable text of a host return code (static storage). */
const char *splitkv_strerror(int code);

/* Detail of the most recent failure in this thread (the failing CUDA call and its error name), or ""
 * if the last call succeeded. Valid until the next call from the same thread. */
const char *splitkv_last_error(void);

/* Build id: the sha256 (hex) of the sources the library was compiled from (every file under csrc/ and
 * this header, by name and content), or "unknown" for a build that did not supply it. The Python binding
 * compares it with the sources beside the library and warns when they differ (a stale build). Static
 * storage; no failure. */
const char *splitkv_build_id(void);

/*
 * Realized cost pass (Split-KV paper, Abstract: chunks are weighted by the attention work they
 * actually incur). Validates the anchors (strictly ascending per sample, each in [block, S)) and, for every
 * item (s, c, g, b) — sample, context chunk, kv head, block — counts the key tiles of chunk c that
 * hold at least one key the block sees: cost = ceil(clamp(a_b - c*C, 0, min(C, S - c*C)) / Tk).
 * Items of cost 0 are dropped; the others are written in ascending item index
 *   id = base_s + (c*Hkv + g)*n_blocks_s + b     (base_s = items of earlier samples)
 * to item_id_d[0..n) and item_cost_d[0..n), with n stored to *n_items_d (device int32).
 * chunk_cost_d[n_chunks] (int64, sample-major) receives the summed cost of each chunk's items.
 * Buffers: anchors_d int32[n_blocks]; item_id_d, item_cost_d int32[n_items_max].
 */
int splitkv_cost(const splitkv_problem *problem, const int32_t *anchors_d, int32_t *item_id_d,
                 int32_t *item_cost_d, int64_t *chunk_cost_d, int32_t *n_items_d, int32_t *status_d,
                 void *workspace_d, size_t workspace_bytes, void *stream);

/*
 * Cost-aware LPT planner (Split-KV paper, Abstract, and its table of
 * context-parallel methods, load-balancing column). Items 0..n-1 (n = *n_items_d <= max_items) with costs
 * item_cost_d[] in [1, max_cost] are taken in order of (cost descending, index ascending) and each
 * is given to the worker with the least (load, worker index); loads start at 0. Outputs:
 *   item_worker_d int32[max_items]   worker of each item
 *   queue_off_d   int32[n_workers+1] CSR offsets; queue_items_d int32[max_items] lists each
 *                                    worker's items in assignment order
 *   load_d        int64[n_workers]   summed cost per worker
 * The result equals the sequential greedy bit for bit; it is computed one equal-cost run at a time.
 */
int splitkv_plan_lpt(const int32_t *item_cost_d, const int32_t *n_items_d, int32_t max_items,
                     int32_t max_cost, int32_t n_workers, int32_t *item_worker_d, int32_t *queue_off_d,
                     int32_t *queue_items_d, int64_t *load_d, int32_t *status_d, void *workspace_d,
                     size_t workspace_bytes, void *stream);

/*
 * Allocation-free variant of splitkv_plan_lpt (the Split-KV paper has no counterpart: this is a
 * deployment convenience). Same arguments, same result, no workspace argument: its scratch is a
 * fixed 4 MiB array inside the library's own device memory, which every GPU that loads the library
 * holds until the process exits. It is meant for callers that cannot call cudaMalloc: code running
 * while a CUDA graph is being captured, or inside a framework whose caching allocator owns all
 * device memory and forbids side allocations, or a latency-critical path that cannot afford the
 * synchronisation an allocation may imply.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current and caches it; make that first call before any stream capture.
 *   - Returns SPLITKV_ENOSPACE (with splitkv_last_error() stating both sizes) when the plan would
 *     need more scratch than the array holds. The scratch grows with max_items (16 bytes per 1024
 *     items and cost bucket), max_cost and n_workers; every max_cost <= 64 with n_workers <= 1024
 *     fits, and the item count sets the limit: at max_cost 64, up to 14.7 million items on 148
 *     workers and 4.3 million on 1024; at max_cost 16, 61 million on 148.
 *   - The cached address belongs to the device's current CUDA context. cudaDeviceReset destroys that
 *     context (the array is re-created, possibly elsewhere, in the next one), so do not call this
 *     entry point after a cudaDeviceReset in the same process.
 *   - It allocates nothing and frees nothing. Every call shares the one array and leaves its
 *     contents behind (the planner rewrites all it reads before reading it), so calls whose GPU
 *     work overlaps — on two streams, or from two host threads — race and corrupt each other's
 *     plans; order them on one stream.
 */
int splitkv_plan_lpt_noalloc(const int32_t *item_cost_d, const int32_t *n_items_d, int32_t max_items,
                             int32_t max_cost, int32_t n_workers, int32_t *item_worker_d, int32_t *queue_off_d,
                             int32_t *queue_items_d, int64_t *load_d, int32_t *status_d, void *stream);

/*
 * Partial forward (Split-KV paper, Abstract: the method is exact and exchanges only tensors the
 * size of the query set). One persistent CTA per worker walks its queue; for each item
 * (s, c, g, t) it computes, over the keys of chunk c that each row's block sees, the chunk-local
 * softmax of s = scale * q.k for the tile's rows (row x*block*G + i*G + hl: query i of its x-th
 * block, query head g*G + hl). Then the self partials: for global block j and kv head g, the
 * softmax over the block's own `block` keys, kb/vb rows block*j .. block*j + block - 1
 * ([Nq, Hkv, d], problem dtype), stored at slot n_items_max + j*Hkv + g (rows 0 .. block*G - 1).
 * Both kinds write, with rows = sizes.rows_per_item and E = 16 / sizeof(problem dtype) elements
 * per 16-byte group (4 for float32, 8 for bf16):
 *   o_part  [slot][d/E][rows][E]  problem dtype: O_p = sum softmax * v, normalised
 *   lse_part[slot][rows]          float32: LSE_p = log sum exp(s), natural log (-inf: no key)
 * Entries of items that are not visible are not written.
 * item_id_d, queue_off_d and queue_items_d come from splitkv_cost and splitkv_plan_lpt.
 * On the tensor-core path each worker runs its queue, then claims self items from a shared counter
 * as it runs out of work (which SM computes a self partial varies from run to run; its value does
 * not). When k and v together exceed the device's L2 cache, a one-SM worker runs the items of its
 * queue in ascending item id rather than in queue order (the same items, so the same load; all
 * workers then walk the context together and share its K/V in L2); queues of more than 512 items
 * keep queue order. With 256-row items (sizes.ctas_per_worker = 2) each worker is a pair of SMs, a two-CTA
 * cluster that issues M = 256 tensor-core instructions over both SMs (2 * n_workers CTAs, n_workers
 * <= 32767); its self items are (query tile of P blocks, kv head), whose rows of block x see key
 * columns block*x .. block*x + block - 1 of one key tile of kb/vb, and each block's self partial
 * still goes to slot n_items_max + j*Hkv + g. workspace_d: splitkv_workspace_size() bytes, 16-byte
 * aligned (the claim counter, reset by this call); the CUDA-core path, which deals self items
 * round-robin, ignores it (may be NULL).
 * q, k, v, kb, vb and o_part must be 16-byte aligned. flags: SPLITKV_FWD_DEFAULT or
 * SPLITKV_FWD_SIMT.
 */
int splitkv_attn_fwd(const splitkv_problem *problem, const void *q, const void *k, const void *v,
                     const void *kb, const void *vb, const int32_t *anchors_d, const int32_t *item_id_d,
                     const int32_t *queue_off_d, const int32_t *queue_items_d, int32_t n_workers,
                     void *o_part, float *lse_part, int32_t *status_d, int32_t flags, void *workspace_d,
                     size_t workspace_bytes, void *stream);

/*
 * Exact log-sum-exp merge (Split-KV paper, Abstract: exactness with query-sized exchange). For each
 * block j, kv head g and row r it combines the self partial (slot n_items_max + j*Hkv + g) with the
 * visible chunk partials c < ceil(a_j / C):
 *   L = log sum_p exp(LSE_p),  O = sum_p exp(LSE_p - L) O_p
 * and writes o [Nq, Hq, d] (problem dtype) and lse [Nq, Hq] (float32, natural log). o_part,
 * lse_part and o must be 16-byte aligned. Reads only what splitkv_attn_fwd wrote.
 */
int splitkv_lse_merge(const splitkv_problem *problem, const void *o_part, const float *lse_part,
                      const int32_t *anchors_d, void *o, float *lse, int32_t *status_d, void *stream);

/*
 * Backward of the same attention (Split-KV paper, title and Abstract: the method trains diffusion
 * drafters). Recomputes P = exp(s - LSE) from the stored lse, with D = rowsum(dout * o):
 *   dV_j += P dO,  dS = P (dO.v_j - D),  dQ += scale dS k_j,  dK_j += scale dS q
 * for the context keys and the block's own keys. Outputs are float32 and are overwritten:
 *   dq [Nq, Hq, d], dk, dv [sum S, Hkv, d], dkb, dvb [Nq, Hkv, d].
 * bf16 with head_dim 128 runs on the tensor cores in one pass over 128-key tiles: dK/dV of a tile
 * accumulate on its SM and dQ is added into dq with float32 reductions (the summation order of dq
 * varies from run to run; dk, dv, dkb, dvb do not). Every other problem runs on CUDA cores. All tensor
 * pointers must be 16-byte aligned on the tensor-core path. Needs no plan; needs
 * splitkv_workspace_size() bytes of workspace.
 */
int splitkv_attn_bwd(const splitkv_problem *problem, const void *q, const void *k, const void *v,
                     const void *kb, const void *vb, const void *o, const float *lse, const void *dout,
                     const int32_t *anchors_d, float *dq, float *dk, float *dv, float *dkb, float *dvb,
                     int32_t *status_d, void *workspace_d, size_t workspace_bytes, void *stream);

/*
 * Context parallelism across ranks (Split-KV paper, Abstract, and its table of context-parallel
 * methods: every rank sees all draft queries, context chunks are placed on ranks by the cost-aware
 * LPT on their realized cost, K/V stay on the rank that owns them, and only query-sized tensors are
 * exchanged). One step on rank r of n ranks:
 *   1. splitkv_cost (any rank; the same anchors give the same chunk costs everywhere), chunk costs
 *      copied to the host, splitkv_cp_plan -> chunk_rank (identical on every rank, no exchange);
 *   2. splitkv_cost_rank (this rank's items), splitkv_plan_lpt onto this GPU's SMs, splitkv_attn_fwd
 *      (its chunks' partials; k/v need to hold only this rank's chunks, at their global rows);
 *   3. splitkv_lse_merge_rank -> this rank's query-sized (O_r, LSE_r);
 *   4. an all-gather of (O_r, LSE_r) over the ranks (NCCL, by the caller);
 *   5. splitkv_lse_merge_ranks -> O, LSE: exactly the single-GPU result.
 * Backward on rank r: splitkv_attn_bwd_rank with the full O, LSE and dout, then a sum (all-reduce) of
 * dq, dkb and dvb over the ranks; dk and dv of this rank's chunks are final as computed (K/V never
 * leave their rank).
 * Items must lie in one chunk (chunks_per_item = 1; EUNSUPPORTED otherwise).
 */

/* LPT of chunks onto ranks, on the host: chunks in order of (cost descending, index ascending), each to
 * the rank with the least (load, rank index); loads start at 0. chunk_cost_h: host int64[n_chunks]
 * (splitkv_cost's chunk_cost_d, sample-major), costs >= 0. Outputs (host): chunk_rank_h int32[n_chunks],
 * rank_load_h int64[n_ranks]. SPLITKV_EINVAL on a negative cost or bad sizes. */
int splitkv_cp_plan(const int64_t *chunk_cost_h, int64_t n_chunks, int32_t n_ranks, int32_t *chunk_rank_h,
                    int64_t *rank_load_h);

/* splitkv_cost for rank `rank` of n_ranks: items of the chunks with chunk_rank_d[c] == rank only
 * (chunk_rank_d: device int32[n_chunks] from splitkv_cp_plan); chunk_cost_d still counts every chunk. */
int splitkv_cost_rank(const splitkv_problem *problem, const int32_t *anchors_d, const int32_t *chunk_rank_d,
                      int32_t rank, int32_t n_ranks, int32_t *item_id_d, int32_t *item_cost_d,
                      int64_t *chunk_cost_d, int32_t *n_items_d, int32_t *status_d, void *workspace_d,
                      size_t workspace_bytes, void *stream);

/* splitkv_lse_merge for rank `rank`: merges the partials of this rank's visible chunks and, for the
 * blocks j with j % n_ranks == rank, the self partial (every rank computes all self partials; each is
 * merged on one rank). Writes o_r [Nq, Hq, d] (problem dtype) and lse_r [Nq, Hq] (float32); a row
 * with nothing on this rank gets O = 0, LSE = -inf. */
int splitkv_lse_merge_rank(const splitkv_problem *problem, const void *o_part, const float *lse_part,
                           const int32_t *anchors_d, const int32_t *chunk_rank_d, int32_t rank, int32_t n_ranks,
                           void *o_r, float *lse_r, int32_t *status_d, void *stream);

/* Exact merge of the ranks' results: o_ranks [n_ranks][Nq, Hq, d] (problem dtype), lse_ranks
 * [n_ranks][Nq, Hq] (float32, -inf: nothing) -> o [Nq, Hq, d], lse [Nq, Hq], with
 * L = log sum_r exp(LSE_r), O = sum_r exp(LSE_r - L) O_r. */
int splitkv_lse_merge_ranks(const splitkv_problem *problem, int32_t n_ranks, const void *o_ranks,
                            const float *lse_ranks, void *o, float *lse, int32_t *status_d, void *stream);

/* This rank's share of splitkv_attn_bwd (same arguments, plus the chunk placement of splitkv_cp_plan):
 * the key tiles of the chunks with chunk_rank_d[c] == rank and the own keys of the blocks j with
 * j % n_ranks == rank. Outputs are overwritten: dk, dv hold the gradients of this rank's chunks' key
 * rows (zero on the other rows); dq is this rank's partial sum (over its keys); dkb, dvb hold its
 * blocks' rows (zero on the others). Summed over the ranks, dq, dk, dv, dkb and dvb equal
 * splitkv_attn_bwd's. o and lse are the merged forward outputs (splitkv_lse_merge_ranks). */
int splitkv_attn_bwd_rank(const splitkv_problem *problem, const void *q, const void *k, const void *v,
                          const void *kb, const void *vb, const void *o, const float *lse, const void *dout,
                          const int32_t *anchors_d, const int32_t *chunk_rank_d, int32_t rank, int32_t n_ranks,
                          float *dq, float *dk, float *dv, float *dkb, float *dvb, int32_t *status_d,
                          void *workspace_d, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SPLITKV_H */
