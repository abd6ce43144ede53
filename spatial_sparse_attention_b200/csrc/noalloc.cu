// Block offsets of one sequence without any device allocation: the counting part of the plan's
// block partition (token counts per 8^3 block, exclusive scans, CSR offsets of the occupied blocks
// in block-key order) with its scratch in one file-scope device array instead of allocator
// memory. The method has no counterpart of this entry point; it serves callers that must not
// allocate (declared in include/ssa.h, ssa_block_offsets_noalloc).
//
// Scratch: a fixed 16.8 MB array, taken with cudaGetSymbolAddress once per device. Every call
// clears the counters it uses before counting, so nothing has to be zeroed by the caller. Calls
// that overlap in time (different streams, or different host threads without ordering) share the
// array and race; serialise them. The first call on a device performs the symbol lookup.
#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace ssa {

namespace {

constexpr int64_t kNAMaxBlocks = (int64_t)1 << 21;   // grid up to 1024^3 cells
constexpr int64_t kNAScanTmp = 2048;                  // >= scan_tmp_len(kNAMaxBlocks + 1)
// layout (int32): counts [kNAMaxBlocks + 1], block index [kNAMaxBlocks + 1], flag, scan scratch
constexpr int64_t kNAInts = 2 * (kNAMaxBlocks + 1) + 64 + kNAScanTmp;

static __device__ __align__(256) int32_t g_noalloc_scratch[kNAInts];

constexpr int kNAThreads = 256;

__global__ void k_na_clear(int32_t* __restrict__ counts, int32_t* __restrict__ flag, int64_t G) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k <= G) counts[k] = 0;
    if (k == 0) *flag = 0;
}

__global__ void k_na_count(const int32_t* __restrict__ coords, int64_t n, int gx, int gy, int gz,
                           int gby, int gbz, int32_t* __restrict__ counts, int32_t* __restrict__ flag) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int32_t x = coords[3 * i], y = coords[3 * i + 1], z = coords[3 * i + 2];
    if (x < 0 || y < 0 || z < 0 || x >= gx || y >= gy || z >= gz) {
        atomicOr(flag, 1);
        return;
    }
    const int64_t key = ((int64_t)(x / kBlockEdge) * gby + (y / kBlockEdge)) * gbz + (z / kBlockEdge);
    atomicAdd(&counts[key], 1);
}

__global__ void k_na_occupied(const int32_t* __restrict__ counts, int32_t* __restrict__ occ, int64_t G) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k < G) occ[k] = counts[k] > 0 ? 1 : 0;
}

// offs: exclusive token offsets per block key; idx: exclusive block index per key
__global__ void k_na_fill(const int32_t* __restrict__ offs, const int32_t* __restrict__ idx, int64_t G,
                          const int32_t* __restrict__ flag, int32_t* __restrict__ blk_off,
                          int64_t cap, int32_t* __restrict__ n_blocks) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k < G && idx[k + 1] > idx[k] && idx[k] < cap) blk_off[idx[k]] = offs[k];
    if (k == 0) {
        if (idx[G] < cap) blk_off[idx[G]] = offs[G];
        *n_blocks = *flag ? -1 : idx[G];
    }
}

int32_t* scratch_of_device() {
    static std::mutex mu;
    static int32_t* ptrs[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        ptrs[dev] = static_cast<int32_t*>(p);
    }
    return ptrs[dev];
}

}  // namespace

}  // namespace ssa

using namespace ssa;

extern "C" SSA_API ssa_status_t ssa_block_offsets_noalloc(const int32_t* coords, int64_t n,
                                                          const int32_t* grid, int32_t* blk_off,
                                                          int64_t blk_off_capacity,
                                                          int32_t* n_blocks, void* stream) {
    if (!coords || !grid || !blk_off || !n_blocks || n < 1) return SSA_ERR_INVALID_ARG;
    for (int a = 0; a < 3; ++a)
        if (grid[a] < 1 || grid[a] > 65535) return SSA_ERR_INVALID_ARG;
    const int gbx = (grid[0] + kBlockEdge - 1) / kBlockEdge;
    const int gby = (grid[1] + kBlockEdge - 1) / kBlockEdge;
    const int gbz = (grid[2] + kBlockEdge - 1) / kBlockEdge;
    const int64_t G = (int64_t)gbx * gby * gbz;
    if (G > kNAMaxBlocks) return SSA_ERR_UNSUPPORTED;   // the scratch holds 2^21 block counters
    if (blk_off_capacity < std::min<int64_t>(n, G) + 1) return SSA_ERR_INVALID_ARG;
    int32_t* base = scratch_of_device();
    if (!base) return SSA_ERR_CUDA;
    int32_t* counts = base;
    int32_t* occ = base + (kNAMaxBlocks + 1);
    int32_t* flag = occ + (kNAMaxBlocks + 1);
    int32_t* tmp = flag + 64;
    cudaStream_t st = (cudaStream_t)stream;
    const unsigned gk = (unsigned)cdiv(G + 1, kNAThreads);
    k_na_clear<<<gk, kNAThreads, 0, st>>>(counts, flag, G);
    k_na_count<<<(unsigned)cdiv(n, kNAThreads), kNAThreads, 0, st>>>(coords, n, grid[0], grid[1], grid[2],
                                                                     gby, gbz, counts, flag);
    k_na_occupied<<<gk, kNAThreads, 0, st>>>(counts, occ, G);
    note_launch(3);
    scan_exclusive(occ, occ, G, tmp, st);
    scan_exclusive(counts, counts, G, tmp, st);
    k_na_fill<<<gk, kNAThreads, 0, st>>>(counts, occ, G, flag, blk_off, blk_off_capacity, n_blocks);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}
