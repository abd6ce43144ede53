// Compression by sparse 3D convolution over the block grid, and gates predicted from the
// queries for the fp32 path (Direct3D-S2 summary page, "Technical principles of Direct3D-S2", SSA
// item: blocks become block-level tokens by sparse 3D convolution and pooling; the branches are
// aggregated with predicted gating scores).
//
// The form implemented: the block means (pooling kernel) go through one 3x3x3 sparse convolution
// over the occupied blocks of each sequence, stride 1, outputs at the occupied blocks only, an
// absent neighbour contributing nothing:
//   Kc_b = sum over offsets o with block b+o occupied of mean(K_{b+o}) . W_o,
// W_o (D x D) shared by K, V and all heads; offset (dx, dy, dz) is W[9(dx+1) + 3(dy+1) + (dz+1)].
// Every head of a block has the same neighbours, so one CTA computes a block for a chunk of heads
// (K and V rows together) as a small fp32 product per present neighbour, staged in shared memory.
#include <algorithm>

#include "common.cuh"

namespace ssa {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxRows = 64;   // K and V rows of one head chunk (2 x heads)

// blk_nbr[b * 27 + o]: the block at offset o of block b inside b's sequence, -1 if unoccupied.
// Blocks of a sequence are in lexicographic (bx, by, bz) order: a binary search finds them.
__global__ void k_block_neighbours(const int32_t* __restrict__ blk_coord, const int32_t* __restrict__ blk_seq,
                                   const int32_t* __restrict__ seq_blk, int64_t Mb,
                                   int32_t* __restrict__ blk_nbr) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= Mb * 27) return;
    const int64_t b = e / 27;
    const int o = (int)(e % 27);
    const int32_t x = blk_coord[3 * b] + o / 9 - 1, y = blk_coord[3 * b + 1] + (o / 3) % 3 - 1,
                  z = blk_coord[3 * b + 2] + o % 3 - 1;
    const int32_t s = blk_seq[b];
    int32_t lo = seq_blk[s], hi = seq_blk[s + 1];
    while (lo < hi) {
        const int32_t mid = lo + (hi - lo) / 2;
        const int32_t* c = blk_coord + 3 * mid;
        const bool less = c[0] < x || (c[0] == x && (c[1] < y || (c[1] == y && c[2] < z)));
        if (less) lo = mid + 1; else hi = mid;
    }
    const bool found = lo < seq_blk[s + 1] && blk_coord[3 * lo] == x && blk_coord[3 * lo + 1] == y &&
                       blk_coord[3 * lo + 2] == z;
    blk_nbr[e] = found ? lo : -1;
}

// One CTA per block. Thread (row group rg = t / 32, lane) accumulates rows rg, rg + 8, ... (K rows
// of the chunk's heads, then V rows) and columns lane, lane + 32, ...
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) k_conv_compress(const float* __restrict__ means,
                                                            const float* __restrict__ W,
                                                            const int32_t* __restrict__ blk_nbr,
                                                            int64_t Mb, int H, int64_t Mb8,
                                                            T* __restrict__ kc, T* __restrict__ vc,
                                                            T* __restrict__ kcg, T* __restrict__ vcg) {
    constexpr int kCT = D / 32, kRT = kMaxRows / 8;
    extern __shared__ float sm[];
    float* A = sm;                        // [kMaxRows][D] neighbour means of the chunk
    float* Ws = sm + kMaxRows * D;        // [D][D] one offset's matrix
    const int64_t b = blockIdx.x;
    const int tid = threadIdx.x, rg = tid >> 5, lane = tid & 31;
    const int hc_max = kMaxRows / 2;
    for (int h0 = 0; h0 < H; h0 += hc_max) {
        const int hc = min(hc_max, H - h0);
        float acc[kRT][kCT];
#pragma unroll
        for (int i = 0; i < kRT; ++i)
#pragma unroll
            for (int c = 0; c < kCT; ++c) acc[i][c] = 0.0f;
        for (int o = 0; o < 27; ++o) {
            const int32_t nb = blk_nbr[b * 27 + o];
            if (nb < 0) continue;   // the same for every thread of the CTA
            __syncthreads();        // the previous offset's tiles are no longer read
            for (int e = tid; e < 2 * hc * D; e += kThreads) {
                const int r = e / D, d = e % D;
                const int which = r / hc, h = h0 + r % hc;
                A[r * D + d] = means[(((int64_t)which * H + h) * Mb + nb) * D + d];
            }
            for (int e = tid; e < D * D; e += kThreads) Ws[e] = W[(int64_t)o * D * D + e];
            __syncthreads();
#pragma unroll 4
            for (int d = 0; d < D; ++d) {
                float w[kCT];
#pragma unroll
                for (int c = 0; c < kCT; ++c) w[c] = Ws[d * D + lane + 32 * c];
#pragma unroll
                for (int i = 0; i < kRT; ++i) {
                    const int r = rg + 8 * i;
                    if (r < 2 * hc) {
                        const float a = A[r * D + d];
#pragma unroll
                        for (int c = 0; c < kCT; ++c) acc[i][c] = fmaf(a, w[c], acc[i][c]);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kRT; ++i) {
            const int r = rg + 8 * i;
            if (r >= 2 * hc) continue;
            const int which = r / hc, h = h0 + r % hc;
            T* dst = which == 0 ? kc : vc;
            T* gdst = which == 0 ? kcg : vcg;
#pragma unroll
            for (int c = 0; c < kCT; ++c) {
                const int e = lane + 32 * c;
                const T val = Elem<T>::from_f(acc[i][c]);
                dst[((int64_t)h * Mb + b) * D + e] = val;
                if (gdst) {
                    const int64_t gd = (int64_t)h * Mb8 * D * (int64_t)sizeof(T) + grouped_off(b, e & ~7, D) +
                                       (e & 7) * (int64_t)sizeof(T);
                    *reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(gdst) + gd) = val;
                }
            }
        }
        __syncthreads();
    }
}

template <typename T, int D>
void run_conv(const Plan* p, const Workspace& w, const float* means, const float* wconv, cudaStream_t st) {
    const size_t smem = sizeof(float) * (kMaxRows * D + D * D);
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(k_conv_compress<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        configured = true;
    }
    k_conv_compress<T, D><<<(unsigned)p->Mb, kThreads, smem, st>>>(
        means, wconv, p->blk_nbr, p->Mb, w.H, w.Mb8, (T*)w.kc, (T*)w.vc,
        w.dtype == SSA_F32 ? nullptr : (T*)w.kcg, w.dtype == SSA_F32 ? nullptr : (T*)w.vcg);
    note_launch();
}

template <typename T>
void run_conv_d(const Plan* p, const Workspace& w, const float* means, const float* wconv, cudaStream_t st) {
    switch (w.D) {
    case 32: run_conv<T, 32>(p, w, means, wconv, st); break;
    case 64: run_conv<T, 64>(p, w, means, wconv, st); break;
    case 96: run_conv<T, 96>(p, w, means, wconv, st); break;
    default: run_conv<T, 128>(p, w, means, wconv, st); break;
    }
}

// gates[(i * H + h) * 3 + c] = sigmoid(bg[c] + sum_d q[i][h][d] * wg[d][c]); one warp per row
__global__ void k_gates_f32(const float* __restrict__ q, const float* __restrict__ wg,
                            const float* __restrict__ bg, int64_t rows, int D, float* __restrict__ gates) {
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    float t[3] = {0.0f, 0.0f, 0.0f};
    for (int d = lane; d < D; d += 32) {
        const float x = q[r * D + d];
#pragma unroll
        for (int c = 0; c < 3; ++c) t[c] = fmaf(x, wg[d * 3 + c], t[c]);
    }
#pragma unroll
    for (int c = 0; c < 3; ++c)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t[c] += __shfl_xor_sync(0xffffffffu, t[c], o);
    if (lane < 3) gates[r * 3 + lane] = 1.0f / (1.0f + __expf(-(t[lane] + bg[lane])));
}

}  // namespace

ssa_status_t ensure_block_neighbours(Plan* p, cudaStream_t st) {
    if (p->blk_nbr) return SSA_OK;
    p->blk_nbr = (int32_t*)plan_alloc(p, sizeof(int32_t) * (size_t)std::max<int64_t>(p->Mb * 27, 1));
    if (!p->blk_nbr) return SSA_ERR_ALLOC;
    k_block_neighbours<<<(unsigned)cdiv(p->Mb * 27, 256), 256, 0, st>>>(p->blk_coord, p->blk_seq, p->seq_blk_d,
                                                                     p->Mb, p->blk_nbr);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

void launch_conv_compress(const Plan* p, const Workspace& w, const float* means, const float* wconv,
                          cudaStream_t st) {
    switch (w.dtype) {
    case SSA_F32: run_conv_d<float>(p, w, means, wconv, st); break;
    case SSA_BF16: run_conv_d<__nv_bfloat16>(p, w, means, wconv, st); break;
    default: run_conv_d<__half>(p, w, means, wconv, st); break;
    }
}

void launch_gates_f32(const Plan* p, const float* q, const float* wg, const float* bg, int H, int D,
                      float* gates, cudaStream_t st) {
    const int64_t rows = p->N * H;
    k_gates_f32<<<(unsigned)cdiv(rows * 32, 256), 256, 0, st>>>(q, wg, bg, rows, D, gates);
    note_launch();
}

}  // namespace ssa
