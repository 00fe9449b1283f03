// Cost-aware LPT planner on the device (Split-KV: Efficient Context Parallelism for Training
// Diffusion Drafters, Abstract, and its table of context-parallel methods: load balancing by
// longest-processing-time-first on the realized cost).
//
// Definition: items taken in order (cost desc, index asc); each goes to the worker with the
// least (load, worker index). Computing that greedy one item at a time is a long serial chain, so
// it is evaluated one equal-cost run at a time, exactly:
//
//   Within a run of n items of equal cost w, worker i can absorb items at loads L_i, L_i + w,
//   L_i + 2w, ...; the greedy always takes the smallest (load, worker) pair still offered, so the
//   run's picks are the n smallest elements of { (L_i + k*w, i) } in (value, worker) order.
//   Cut the value axis into windows [V0 + r*w, V0 + (r+1)*w) with V0 = min L. Worker i offers
//   exactly one element in every window r >= r_i = (L_i - V0) / w, at offset o_i = (L_i - V0) % w,
//   so inside a window the order is by (o_i, i) — the same order q_i in every window. Windows
//   below R = max r_i ("catch-up") miss the workers with r_i > r; from window R on, every window
//   lists all m workers in q order. Hence rank(i, k) = P(r) + pos_i(r) with r = r_i + k, where
//   P(r) counts the elements of earlier windows and pos_i(r) the workers of window r ahead of i.
//
// Launches: (1) per-CTA cost histograms, (2) one CTA walks the runs (cost W..1) and builds, per
// run, the catch-up element list, the q order and each worker's pick count, then the final loads
// and queue offsets, (3) one thread per item places it. Every quantity is an integer, so the plan
// equals the sequential greedy bit for bit.
#include <mutex>

#include "common.cuh"
#include "scan.cuh"

namespace splitkv {

// Scratch for splitkv_plan_lpt_noalloc: a fixed array in the library's own device memory, so that
// entry point needs no allocation. Every device that loads the library holds it until exit, and
// all calls share it.
static __device__ __align__(256) unsigned char g_plan_scratch[kStaticPlanScratchBytes];

namespace {

constexpr int kThreads = 1024;

struct PlanWs {
    int32_t* hist;     // [nblk][W+1]: per-CTA counts, then per-CTA start positions in sorted order
    int32_t* run_n;    // [W+1]
    int32_t* run_start;
    int32_t* run_ncatch;
    int32_t* run_rmax;
    int32_t* run_qinv;   // [W+1][m]: worker at q position
    int32_t* run_r;      // [W+1][m]: first window of each worker
    int32_t* run_qbase;  // [W+1][m]: items the worker got in earlier runs
    int32_t* run_cbase;  // [W+1]: start of run w's catch-up list in run_catch
    int2* run_catch;     // run w: m * floor(W / w) entries (worker, k), one per catch-up rank
};

// Catch-up entries run w can produce. Every load stays within W (the largest cost) of the smallest
// (each item goes to a least-loaded worker), so a worker's first window is r_i <= floor(W / w) and the
// catch-up windows r < R = max r_i hold at most m * floor(W / w) elements.
__host__ __device__ inline int64_t catch_cap(int32_t W, int32_t m, int32_t w) { return (int64_t)m * (W / w); }

__host__ __device__ inline PlanWs carve(void* ws, int32_t max_items, int32_t W, int32_t m, size_t* bytes) {
    char* p = (char*)ws;
    size_t off = 0;
    auto take = [&](size_t n) { char* r = p + off; off = align_up(off + n, 256); return r; };
    PlanWs w;
    int32_t nblk = (max_items + kThreads - 1) / kThreads;
    w.hist = (int32_t*)take(sizeof(int32_t) * (size_t)(nblk > 0 ? nblk : 1) * (W + 1));
    w.run_n = (int32_t*)take(sizeof(int32_t) * (W + 1));
    w.run_start = (int32_t*)take(sizeof(int32_t) * (W + 1));
    w.run_ncatch = (int32_t*)take(sizeof(int32_t) * (W + 1));
    w.run_rmax = (int32_t*)take(sizeof(int32_t) * (W + 1));
    w.run_qinv = (int32_t*)take(sizeof(int32_t) * (size_t)(W + 1) * m);
    w.run_r = (int32_t*)take(sizeof(int32_t) * (size_t)(W + 1) * m);
    w.run_qbase = (int32_t*)take(sizeof(int32_t) * (size_t)(W + 1) * m);
    w.run_cbase = (int32_t*)take(sizeof(int32_t) * (W + 1));
    int64_t ncatch = 0;
    for (int32_t v = 1; v <= W; ++v) ncatch += catch_cap(W, m, v);
    w.run_catch = (int2*)take(sizeof(int2) * (size_t)(ncatch > 0 ? ncatch : 1));
    if (bytes) *bytes = off;
    return w;
}

__global__ void __launch_bounds__(kThreads) plan_hist_kernel(const int32_t* __restrict__ cost,
                                                             const int32_t* __restrict__ n_items_d,
                                                             int32_t max_items, int32_t W, PlanWs ws,
                                                             int32_t* __restrict__ status) {
    __shared__ int32_t h[kMaxCost + 1];
    if (status_bad(status)) return;
    int32_t n = *n_items_d;
    if (n < 0 || n > max_items) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(status, SPLITKV_DEV_BAD_COST);
        return;
    }
    for (int i = threadIdx.x; i <= W; i += kThreads) h[i] = 0;
    __syncthreads();
    int32_t k = blockIdx.x * kThreads + threadIdx.x;
    if (k < n) {
        int32_t w = cost[k];
        if (w < 1 || w > W) raise_status(status, SPLITKV_DEV_BAD_COST);
        else atomicAdd(&h[w], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i <= W; i += kThreads) ws.hist[(size_t)blockIdx.x * (W + 1) + i] = h[i];
}

// (The explicit one-block minimum keeps ptxas from holding this kernel to 32 registers with spills.)
__global__ void __launch_bounds__(kThreads, 1) plan_runs_kernel(const int32_t* __restrict__ n_items_d,
                                                             int32_t max_items, int32_t W, int32_t m, PlanWs ws,
                                                             int32_t* __restrict__ queue_off,
                                                             int64_t* __restrict__ load_out,
                                                             int32_t* __restrict__ status) {
    __shared__ int64_t L[kThreads];
    __shared__ int32_t qcount[kThreads];
    __shared__ int32_t rr[kThreads];       // first window of each worker
    __shared__ int32_t by_q[kThreads];     // worker at each (offset, worker) position
    __shared__ int32_t cnt_w[32][kMaxCost + 1];
    __shared__ int32_t start_o[kMaxCost + 1];
    __shared__ int32_t total[kMaxCost + 1];
    __shared__ int32_t start[kMaxCost + 1];
    __shared__ int32_t cnt_r[kMaxCost + 2];
    __shared__ int32_t P[kMaxCost + 2];
    __shared__ int32_t cbase[kMaxCost + 1];
    __shared__ int64_t red64[32];
    __shared__ int32_t red32[33];
    __shared__ int32_t scan_sh[33];
    __shared__ int32_t bad;

    if (status_bad(status)) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = (int)(blockDim.x >> 5);
    const int32_t n = *n_items_d;
    const int32_t nblk = (n + kThreads - 1) / kThreads;  // CTAs of plan_hist_kernel

    // Bucket totals, per-CTA offsets within each bucket, bucket starts (cost descending).
    for (int w = tid; w <= W; w += blockDim.x) {
        int32_t acc = 0;
        for (int32_t b = 0; b < nblk; ++b) {
            int32_t c = ws.hist[(size_t)b * (W + 1) + w];
            ws.hist[(size_t)b * (W + 1) + w] = acc;
            acc += c;
        }
        total[w] = acc;
    }
    if (tid == 0) bad = 0;
    __syncthreads();
    if (tid == 0) {
        int32_t s = 0;
        for (int w = W; w >= 1; --w) { start[w] = s; s += total[w]; }
        start[0] = s;
        int32_t cb = 0;
        for (int w = 1; w <= W; ++w) { cbase[w] = cb; ws.run_cbase[w] = cb; cb += (int32_t)catch_cap(W, m, w); }
    }
    __syncthreads();
    for (int w = tid; w <= W; w += blockDim.x)
        for (int32_t b = 0; b < nblk; ++b) ws.hist[(size_t)b * (W + 1) + w] += start[w];

    if (tid < m) { L[tid] = 0; qcount[tid] = 0; }
    __syncthreads();

    for (int w = W; w >= 1; --w) {
        const int32_t nw = total[w];
        if (tid == 0) { ws.run_n[w] = nw; ws.run_start[w] = start[w]; }
        if (nw == 0) continue;  // uniform across the block

        // V0 = min load.
        const int64_t li = tid < m ? L[tid] : INT64_MAX;
        int64_t v = warp_reduce_min(li);
        if (lane == 0) red64[warp] = v;
        for (int i = tid; i < 32 * (kMaxCost + 1); i += blockDim.x) (&cnt_w[0][0])[i] = 0;
        for (int i = tid; i <= W + 1; i += blockDim.x) cnt_r[i] = 0;
        __syncthreads();
        if (tid < 32) {
            int64_t x = tid < nwarps ? red64[tid] : INT64_MAX;  // one entry per warp of the block
            x = warp_reduce_min(x);
            if (tid == 0) red64[0] = x;
        }
        __syncthreads();
        const int64_t V0 = red64[0];
        int32_t ri = 0, oi = w;  // threads without a worker sort into an unused bucket
        if (tid < m) {
            // Window and offset in 32 bits (a 64-bit division is a long dependent sequence on this
            // latency-bound path): a valid plan keeps loads within W of the minimum (r_i <= W / w),
            // and a difference that does not fit in 32 bits is a window past that all the same.
            const uint64_t dlt = (uint64_t)(li - V0);
            if (dlt > 0xffffffffull) {
                ri = W + 1;
                oi = 0;
            } else {
                ri = (int32_t)((uint32_t)dlt / (uint32_t)w);
                oi = (int32_t)((uint32_t)dlt % (uint32_t)w);
            }
            rr[tid] = ri;
            if (ri > W / w) atomicOr(&bad, 1);
            else atomicAdd(&cnt_r[ri], 1);
        }
        // q_i: stable position of worker i in (offset, worker) order, by counting sort.
        const unsigned same = __match_any_sync(0xffffffffu, oi);
        const int rank_warp = __popc(same & ((1u << lane) - 1u));
        if (tid < m && rank_warp == 0) cnt_w[warp][oi] = __popc(same);
        int32_t rmax = warp_reduce_max(tid < m ? ri : 0);
        if (lane == 0) red32[warp] = rmax;
        __syncthreads();
        if (warp == 0) {  // per-offset totals and their exclusive prefix (offsets < w <= 64: two per lane)
            int32_t c0 = 0, c1 = 0;
            for (int x = 0; x < nwarps; ++x) {
                if (lane < w) c0 += cnt_w[x][lane];
                if (lane + 32 < w) c1 += cnt_w[x][lane + 32];
            }
            const int32_t i0 = warp_inclusive_scan(c0);
            const int32_t i1 = warp_inclusive_scan(c1) + __shfl_sync(0xffffffffu, i0, 31);
            if (lane < w) start_o[lane] = i0 - c0;
            if (lane + 32 < w) start_o[lane + 32] = i1 - c1;
        }
        if (tid == 32) {
            int32_t x = 0;
            for (int y = 0; y < nwarps; ++y) x = red32[y] > x ? red32[y] : x;
            red32[32] = x;
        }
        __syncthreads();
        if (bad) break;
        const int32_t R = red32[32];  // <= W / w
        int32_t qi = 0;
        if (tid < m) {
            qi = start_o[oi] + rank_warp;
            for (int x = 0; x < warp; ++x) qi += cnt_w[x][oi];
            by_q[qi] = tid;
        }
        if (tid == 0) {
            // P[r] = sum_{r' < r} #{i : r_i <= r'}
            int32_t le = 0, acc = 0;
            for (int r = 0; r <= R; ++r) {
                P[r] = acc;
                le += cnt_r[r];
                acc += le;
            }
            ws.run_ncatch[w] = P[R] < nw ? P[R] : nw;
            ws.run_rmax[w] = R;
        }
        __syncthreads();
        int32_t picks = 0;  // of worker `tid`
        if (tid < m) {
            ws.run_qinv[(size_t)w * m + qi] = tid;
            ws.run_r[(size_t)w * m + tid] = ri;
        }
        // Catch-up windows r < R: participants (r_i <= r) in q order get ranks P[r] + position.
        // Thread x handles the worker at q position x. A participant's position is the participants
        // before it in its warp (a ballot) plus those of the earlier warps: per-warp counts for every
        // window (cnt_w[warp][r]: the offset counts are consumed), then their prefix over warps.
        const int32_t wx = tid < m ? by_q[tid] : -1;
        const int32_t rx = wx >= 0 ? rr[wx] : 0;
        const unsigned below = (1u << lane) - 1u;
        int32_t picks_x = 0;
        for (int r = 0; r < R; ++r) {
            const unsigned b = __ballot_sync(0xffffffffu, wx >= 0 && rx <= r);
            if (lane == 0) cnt_w[warp][r] = __popc(b);
        }
        __syncthreads();
        if (tid < R) {
            int32_t acc = 0;
            for (int y = 0; y < nwarps; ++y) { const int32_t c = cnt_w[y][tid]; cnt_w[y][tid] = acc; acc += c; }
        }
        __syncthreads();
        for (int r = 0; r < R; ++r) {
            const unsigned b = __ballot_sync(0xffffffffu, wx >= 0 && rx <= r);
            if (wx >= 0 && rx <= r) {
                const int32_t rank = P[r] + cnt_w[warp][r] + __popc(b & below);
                if (rank < nw) {
                    ws.run_catch[cbase[w] + rank] = make_int2(wx, r - rx);
                    ++picks_x;
                }
            }
        }
        __syncthreads();
        // Hand the catch-up counts from position-owner to worker-owner through shared memory.
        if (tid < m) rr[wx] = picks_x;  // rr is no longer needed: reuse it
        __syncthreads();
        if (tid < m) {
            picks = rr[tid];
            // Steady windows r >= R: rank = P[R] + (r - R) * m + q_i.
            const int32_t extra = nw - P[R] - qi;
            if (extra > 0) picks += (extra + m - 1) / m;
            ws.run_qbase[(size_t)w * m + tid] = qcount[tid];
            qcount[tid] += picks;
            L[tid] += (int64_t)picks * w;
        }
        __syncthreads();
    }
    if (bad) {
        if (tid == 0) raise_status(status, SPLITKV_DEV_BAD_PLAN);
        return;
    }
    int32_t c = tid < m ? qcount[tid] : 0;
    int32_t tot;
    int32_t ex = block_exclusive_scan<int32_t>(c, scan_sh, &tot);
    if (tid < m) {
        queue_off[tid] = ex;
        load_out[tid] = L[tid];
    }
    if (tid == 0) {
        queue_off[m] = tot;
        if (tot != n) raise_status(status, SPLITKV_DEV_BAD_PLAN);
    }
}

__global__ void __launch_bounds__(kThreads) plan_assign_kernel(const int32_t* __restrict__ cost,
                                                               const int32_t* __restrict__ n_items_d,
                                                               int32_t W, int32_t m, PlanWs ws,
                                                               const int32_t* __restrict__ queue_off,
                                                               int32_t* __restrict__ item_worker,
                                                               int32_t* __restrict__ queue_items,
                                                               int32_t* __restrict__ status) {
    __shared__ int32_t cnt[32][kMaxCost + 1];
    if (status_bad(status)) return;
    const int32_t n = *n_items_d;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < 32 * (kMaxCost + 1); i += kThreads) (&cnt[0][0])[i] = 0;
    __syncthreads();
    const int32_t k = blockIdx.x * kThreads + tid;
    const bool valid = k < n;
    const int32_t w = valid ? cost[k] : 0;
    const unsigned same = __match_any_sync(0xffffffffu, w);
    const int rank_warp = __popc(same & ((1u << lane) - 1u));
    if (valid && rank_warp == 0) cnt[warp][w] = __popc(same);
    __syncthreads();
    if (!valid || w < 1 || w > W) return;
    int32_t before = 0;
    for (int x = 0; x < warp; ++x) before += cnt[x][w];
    const int32_t j = ws.hist[(size_t)blockIdx.x * (W + 1) + w] - ws.run_start[w] + before + rank_warp;
    int32_t worker, kk;
    const int32_t ncatch = ws.run_ncatch[w];
    if (j < ncatch) {
        int2 e = ws.run_catch[ws.run_cbase[w] + j];
        worker = e.x;
        kk = e.y;
    } else {
        int32_t jj = j - ncatch;
        int32_t window = ws.run_rmax[w] + jj / m;
        worker = ws.run_qinv[(size_t)w * m + (jj % m)];
        kk = window - ws.run_r[(size_t)w * m + worker];
    }
    const int32_t pos = queue_off[worker] + ws.run_qbase[(size_t)w * m + worker] + kk;
    if (worker < 0 || worker >= m || kk < 0 || pos < queue_off[worker] || pos >= queue_off[worker + 1]) {
        raise_status(status, SPLITKV_DEV_BAD_PLAN);
        return;
    }
    item_worker[k] = worker;
    queue_items[pos] = k;
}

}  // namespace

cudaError_t static_plan_scratch(void** out) {
    // The array's device address differs per device; look it up once per device, with that device
    // current (cudaGetSymbolAddress), and keep it. Host code must not use the symbol itself.
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return note_error(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return note_error(cudaErrorInvalidDevice, "plan scratch: device index");
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_plan_scratch);
        if (e != cudaSuccess) return note_error(e, "cudaGetSymbolAddress(plan scratch)");
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

size_t plan_workspace(int32_t max_items, int32_t max_cost, int32_t n_workers) {
    size_t bytes = 0;
    carve(nullptr, max_items, max_cost, n_workers, &bytes);
    return bytes;
}

cudaError_t launch_plan(const int32_t* item_cost, const int32_t* n_items, int32_t max_items, int32_t max_cost,
                        int32_t n_workers, int32_t* item_worker, int32_t* queue_off, int32_t* queue_items,
                        int64_t* load, int32_t* status, void* ws, cudaStream_t st) {
    PlanWs w = carve(ws, max_items, max_cost, n_workers, nullptr);
    int32_t nblk = (max_items + kThreads - 1) / kThreads;
    if (nblk < 1) nblk = 1;
    plan_hist_kernel<<<nblk, kThreads, 0, st>>>(item_cost, n_items, max_items, max_cost, w, status);
    // One CTA with a thread per worker (at least 4 warps: offsets up to max_cost <= 64 get a thread
    // each): the run loop is bound by its barriers, which cost less with fewer warps.
    int32_t runs_threads = ((n_workers + 31) / 32) * 32;
    if (runs_threads < 128) runs_threads = 128;
    plan_runs_kernel<<<1, runs_threads, 0, st>>>(n_items, max_items, max_cost, n_workers, w, queue_off, load, status);
    plan_assign_kernel<<<nblk, kThreads, 0, st>>>(item_cost, n_items, max_cost, n_workers, w, queue_off,
                                                  item_worker, queue_items, status);
    return cudaGetLastError();
}

}  // namespace splitkv
