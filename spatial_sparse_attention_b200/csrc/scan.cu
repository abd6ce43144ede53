// Device-wide exclusive prefix sum of int32 values: three passes (tile sums, scan of the tile
// sums in one CTA, rescan of each tile with its offset). Used by the plan (block, neighbour and
// window offsets) and the allocation-free block offsets.
#include "common.cuh"

namespace ssa {

namespace {

constexpr int kThreads = 256;
constexpr int kItems = 8;
constexpr int kTile = kThreads * kItems;

// Exclusive scan of one value per thread across the CTA; returns this thread's offset and the
// CTA total through `total`.
__device__ int block_exclusive_scan(int v, int* total) {
    __shared__ int warp_sums[kThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kThreads / 32) warp_sums[lane] = w;
    }
    __syncthreads();
    int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
    *total = warp_sums[kThreads / 32 - 1];
    __syncthreads();
    return before;
}

__global__ void k_tile_sums(const int32_t* __restrict__ in, int64_t n, int32_t* __restrict__ sums) {
    int64_t base = (int64_t)blockIdx.x * kTile + (int64_t)threadIdx.x * kItems;
    int s = 0;
#pragma unroll
    for (int t = 0; t < kItems; ++t)
        if (base + t < n) s += in[base + t];
    int total;
    block_exclusive_scan(s, &total);
    if (threadIdx.x == 0) sums[blockIdx.x] = total;
}

// One CTA scans `m` tile sums in place (exclusive) and stores the grand total at sums[m].
__global__ void k_scan_sums(int32_t* __restrict__ sums, int64_t m) {
    int carry = 0;
    for (int64_t base = 0; base < m; base += kTile) {
        int v[kItems];
        int s = 0;
#pragma unroll
        for (int t = 0; t < kItems; ++t) {
            int64_t i = base + (int64_t)threadIdx.x * kItems + t;
            v[t] = i < m ? sums[i] : 0;
            s += v[t];
        }
        int total;
        int off = block_exclusive_scan(s, &total) + carry;
#pragma unroll
        for (int t = 0; t < kItems; ++t) {
            int64_t i = base + (int64_t)threadIdx.x * kItems + t;
            if (i < m) sums[i] = off;
            off += v[t];
        }
        carry += total;
    }
    if (threadIdx.x == 0) sums[m] = carry;
}

__global__ void k_apply(const int32_t* in, int64_t n, const int32_t* __restrict__ sums,
                        int64_t m, int32_t* out) {
    int64_t base = (int64_t)blockIdx.x * kTile + (int64_t)threadIdx.x * kItems;
    int v[kItems];
    int s = 0;
#pragma unroll
    for (int t = 0; t < kItems; ++t) {
        v[t] = base + t < n ? in[base + t] : 0;
        s += v[t];
    }
    int total;
    int off = block_exclusive_scan(s, &total) + sums[blockIdx.x];
#pragma unroll
    for (int t = 0; t < kItems; ++t) {
        if (base + t < n) out[base + t] = off;
        off += v[t];
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) out[n] = sums[m];
}

}  // namespace

int64_t scan_tmp_len(int64_t n) { return cdiv(n > 0 ? n : 1, kTile) + 1; }

void scan_exclusive(const int32_t* in, int32_t* out, int64_t n, int32_t* tmp, cudaStream_t s) {
    int64_t m = cdiv(n > 0 ? n : 1, kTile);
    k_tile_sums<<<(unsigned)m, kThreads, 0, s>>>(in, n, tmp);
    k_scan_sums<<<1, kThreads, 0, s>>>(tmp, m);
    k_apply<<<(unsigned)m, kThreads, 0, s>>>(in, n, tmp, m, out);
    note_launch(3);
}

}  // namespace ssa
