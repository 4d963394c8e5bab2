// block_scan.cuh -- deterministic block-wide exclusive prefix sum of one int per thread.
#pragma once

namespace lsa {

// Exclusive scan of v over the NT threads of the block (NT a multiple of 32,
// at most 1024).  `warp_tot` is shared scratch of NT/32 ints.  Returns the
// exclusive prefix and writes the block total to *total (all threads).
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_tot[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        int t = lane < NT / 32 ? warp_tot[lane] : 0;
        int ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += n;
        }
        if (lane < NT / 32) warp_tot[lane] = ti - t;  // exclusive warp offsets
        if (lane == NT / 32 - 1) warp_tot[NT / 32] = ti;
    }
    __syncthreads();
    int res = warp_tot[wid] + inc - v;
    *total = warp_tot[NT / 32];
    __syncthreads();
    return res;
}

}  // namespace lsa
