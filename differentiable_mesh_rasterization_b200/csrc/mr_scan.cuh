// Three-launch exclusive scan of int counts (internal header), shared by the mesh and
// the point binning passes.
#pragma once

#include "mr_common.cuh"

namespace mr {
namespace {

// Exclusive scan of nb counts in three launches: 4096-entry tiles scanned by 1024-thread
// CTAs (coalesced, warp shuffles), the tile totals scanned by one CTA, then the tile
// prefixes added; offsets[nb] = total.
constexpr int kScanTile = 4096;

__device__ __forceinline__ long long block_exclusive_scan(long long x, long long* wsum, long long& total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    long long inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[w] = inc;
    __syncthreads();
    if (w == 0) {
        long long y = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += z;
        }
        wsum[lane] = y;
    }
    __syncthreads();
    total = wsum[(blockDim.x >> 5) - 1];
    const long long ex = (w ? wsum[w - 1] : 0) + inc - x;
    __syncthreads();
    return ex;
}

__global__ void __launch_bounds__(1024) k_scan_tiles(const int* __restrict__ counts, int nb, int* __restrict__ offsets,
                                                     long long* __restrict__ tile_sum) {
    __shared__ long long wsum[32];
    const int base = blockIdx.x * kScanTile + threadIdx.x * 4;
    int v[4];
    long long sum = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        v[u] = base + u < nb ? counts[base + u] : 0;
        sum += v[u];
    }
    long long total;
    long long run = block_exclusive_scan(sum, wsum, total);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (base + u < nb) offsets[base + u] = (int)run;
        run += v[u];
    }
    if (threadIdx.x == 0) tile_sum[blockIdx.x] = total;
}

__global__ void __launch_bounds__(1024) k_scan_tops(long long* __restrict__ tile_sum, int ntiles,
                                                    long long* __restrict__ total_out) {
    __shared__ long long wsum[32];
    long long carry = 0;
    for (int base = 0; base < ntiles; base += 1024) {
        const int i = base + threadIdx.x;
        const long long x = i < ntiles ? tile_sum[i] : 0;
        long long total;
        const long long ex = block_exclusive_scan(x, wsum, total);
        if (i < ntiles) tile_sum[i] = carry + ex;
        carry += total;
    }
    if (threadIdx.x == 0) *total_out = carry;
}

__global__ void k_scan_add(int* __restrict__ offsets, int nb, const long long* __restrict__ tile_pre,
                           const long long* __restrict__ total) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= nb; i += gridDim.x * blockDim.x) {
        if (i == nb) offsets[nb] = (int)*total;
        else offsets[i] += (int)tile_pre[i / kScanTile];
    }
}

}  // namespace
}  // namespace mr
