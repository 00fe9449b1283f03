// Block-wide scans and reductions built from warp shuffles (blockDim.x a multiple of 32, <= 1024).
#pragma once

#include <cstdint>

namespace splitkv {

template <typename T>
__device__ inline T warp_inclusive_scan(T x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Exclusive scan over the block; returns this thread's prefix and writes the block total.
// `sh` must hold 33 elements of T. All threads of the block must call it.
template <typename T>
__device__ inline T block_exclusive_scan(T x, T* sh, T* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
    T inc = warp_inclusive_scan(x);
    if (lane == 31) sh[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        T w = lane < nwarps ? sh[lane] : T(0);
        T wi = warp_inclusive_scan(w);
        if (lane < nwarps) sh[lane] = wi - w;
        if (lane == nwarps - 1) sh[32] = wi;
    }
    __syncthreads();
    T res = sh[warp] + inc - x;
    if (total) *total = sh[32];
    __syncthreads();
    return res;
}

template <typename T>
__device__ inline T warp_reduce_min(T x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        T y = __shfl_xor_sync(0xffffffffu, x, o);
        x = y < x ? y : x;
    }
    return x;
}

template <typename T>
__device__ inline T warp_reduce_max(T x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        T y = __shfl_xor_sync(0xffffffffu, x, o);
        x = y > x ? y : x;
    }
    return x;
}

template <typename T>
__device__ inline T warp_reduce_sum(T x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace splitkv
