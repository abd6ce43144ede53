// Backward of Spatial Sparse Attention (Direct3D-S2 model page, "What is Direct3D-S2?":
// the method has a backward pass, reported ~9.6x faster than baseline sparse attention).
// Gradients of L = sum(dO * out) with respect to Q, K, V, with the block selection held at the
// forward's choice and the rounding of the compressed tokens treated as identity.
//
// Correctness-grade CUDA-core kernels, fp32 accumulation:
//   k_bwd_rows:     one warp per (token, head); for each branch (compressed, selected, window)
//                   three passes over its keys: softmax statistics, sum_j P_j dP_j, then
//                   dq += s dz_j k_j with dk_j += s dz_j q and dv_j += g P_j dO scattered by
//                   fp32 atomics (compressed keys scatter into dKc / dVc);
//   k_bwd_compress: dK_j += (1/n_b) dKc_b Wc^T for every token of block b (same for V);
//   k_bwd_cast:     fp32 accumulators to the input type.
#include "common.cuh"

namespace ssa {

namespace {

constexpr int kWarps = 8;

struct BwdParams {
    const void* q;
    const void* k;
    const void* v;
    const void* dout;
    const void* kc;
    const void* vc;
    const float* gates;
    const float* wc;
    const int32_t* perm;
    const int32_t* tok_blk;
    const int32_t* tok_pos;
    const int32_t* blk_off;
    const int32_t* seq_blk;
    const SeqInfo* seqs;
    const int32_t* nbr_off;
    const int32_t* nbr_idx;
    const int32_t* sel;
    void* dq;
    float* dk32;
    float* dv32;
    float* dkc;
    float* dvc;
    int64_t N, Mb;
    int H, D, topk, B;
    float scale;
};

template <typename T>
__device__ __forceinline__ float ld(const void* base, int64_t i) {
    return Elem<T>::to_f(reinterpret_cast<const T*>(base)[i]);
}

template <typename T>
__device__ __forceinline__ float wdot(const float (&a)[4], const void* base, int64_t row, int D, int lane) {
    float s = 0.0f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int d = lane + 32 * t;
        if (d < D) s = fmaf(a[t], ld<T>(base, row + d), s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
    return __shfl_sync(0xffffffffu, s, 0);
}

// One branch: keys/values at rows key_row(j) of kb/vb (element offsets of a D-vector), gradient
// targets at rows of dkt/dvt (fp32).
template <typename T, class Rows>
__device__ void branch_backward(const BwdParams& P, int n, Rows rows, const void* kb, const void* vb,
                                float* dkt, float* dvt, float g, const float (&q)[4],
                                const float (&go)[4], float (&dq)[4], int lane) {
    const int D = P.D;
    float m = -INFINITY, l = 0.0f;
    for (int j = 0; j < n; ++j) {
        const float z = P.scale * wdot<T>(q, kb, rows(j), D, lane);
        if (z > m) {
            l = (m == -INFINITY) ? 0.0f : l * expf(m - z);
            m = z;
        }
        l += expf(z - m);
    }
    float pdp = 0.0f;
    for (int j = 0; j < n; ++j) {
        const int64_t r = rows(j);
        const float p = expf(P.scale * wdot<T>(q, kb, r, D, lane) - m) / l;
        pdp += p * g * wdot<T>(go, vb, r, D, lane);
    }
    for (int j = 0; j < n; ++j) {
        const int64_t r = rows(j);
        const float p = expf(P.scale * wdot<T>(q, kb, r, D, lane) - m) / l;
        const float dp = g * wdot<T>(go, vb, r, D, lane);
        const float dz = p * (dp - pdp);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int d = lane + 32 * t;
            if (d < D) {
                dq[t] = fmaf(P.scale * dz, ld<T>(kb, r + d), dq[t]);
                atomicAdd(dkt + r + d, P.scale * dz * q[t]);
                atomicAdd(dvt + r + d, g * p * go[t]);
            }
        }
    }
}

template <typename T, int KM>
__global__ void __launch_bounds__(kWarps * 32) k_bwd_rows(const BwdParams P) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= P.N * P.H) return;
    const int64_t i = w / P.H;
    const int h = (int)(w % P.H);
    const int H = P.H, D = P.D;
    const int s = find_seq(P.seqs, P.B, i);
    const int32_t bl = P.seq_blk[s], bh = P.seq_blk[s + 1];
    float q[4], go[4], dq[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int d = lane + 32 * t;
        q[t] = d < D ? ld<T>(P.q, (i * H + h) * D + d) : 0.0f;
        go[t] = d < D ? ld<T>(P.dout, (i * H + h) * D + d) : 0.0f;
    }
    const float* g = P.gates + (i * H + h) * 3;
    // compressed branch: keys Kc[h][b]
    branch_backward<T>(P, bh - bl, [&](int j) { return ((int64_t)h * P.Mb + bl + j) * D; }, P.kc,
                       P.vc, P.dkc, P.dvc, g[0], q, go, dq, lane);
    // selected branch: tokens of the selected blocks, in slot order
    const int32_t* srow = P.sel + ((int64_t)P.tok_pos[i] * H + h) * P.topk;
    int32_t counts[KM + 1];
    int n_sel = 0;
#pragma unroll
    for (int t = 0; t <= KM; ++t) {
        const int32_t b = t < P.topk ? srow[t] : -1;
        counts[t] = b >= 0 ? P.blk_off[b + 1] - P.blk_off[b] : 0;
        n_sel += counts[t];
    }
    branch_backward<T>(
        P, n_sel,
        [&](int j) {
            int t = 0;
            while (j >= counts[t]) {   // slot t holds tokens [sum counts[<t], sum counts[<=t])
                j -= counts[t];
                ++t;
            }
            const int64_t tok = P.perm[P.blk_off[srow[t]] + j];
            return (tok * H + h) * D;
        },
        P.k, P.v, P.dk32, P.dv32, g[1], q, go, dq, lane);
    // window branch
    const int32_t w0 = P.nbr_off[i];
    branch_backward<T>(P, P.nbr_off[i + 1] - w0,
                       [&](int j) { return ((int64_t)P.nbr_idx[w0 + j] * H + h) * D; }, P.k, P.v,
                       P.dk32, P.dv32, g[2], q, go, dq, lane);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int d = lane + 32 * t;
        if (d < D) reinterpret_cast<T*>(P.dq)[(i * H + h) * D + d] = Elem<T>::from_f(dq[t]);
    }
}

// dK_j += (1/n_b) * sum_e dKc_b[e] * Wc[d][e] for every token j of block b; same for V.
__global__ void k_bwd_compress(const BwdParams P) {
    const int64_t b = blockIdx.x;
    const int h = blockIdx.y;
    const int D = P.D, H = P.H;
    const int32_t lo = P.blk_off[b], n = P.blk_off[b + 1] - lo;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        float uk = 0.0f, uv = 0.0f;
        for (int e = 0; e < D; ++e) {
            const float w = P.wc[d * D + e];
            uk = fmaf(P.dkc[((int64_t)h * P.Mb + b) * D + e], w, uk);
            uv = fmaf(P.dvc[((int64_t)h * P.Mb + b) * D + e], w, uv);
        }
        uk /= (float)n;
        uv /= (float)n;
        for (int t = 0; t < n; ++t) {
            const int64_t tok = P.perm[lo + t];
            P.dk32[(tok * H + h) * D + d] += uk;
            P.dv32[(tok * H + h) * D + d] += uv;
        }
    }
}

template <typename T>
__global__ void k_bwd_cast(const float* __restrict__ a, const float* __restrict__ b, int64_t n,
                           T* __restrict__ oa, T* __restrict__ ob) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    oa[i] = Elem<T>::from_f(a[i]);
    ob[i] = Elem<T>::from_f(b[i]);
}

template <typename T>
ssa_status_t run(Plan* p, const Workspace& w, BwdParams P, void* dk, void* dv, cudaStream_t st) {
    const unsigned grid = (unsigned)cdiv(p->N * w.H, kWarps);
    if (w.k - 1 <= 8) k_bwd_rows<T, 8><<<grid, kWarps * 32, 0, st>>>(P);
    else if (w.k - 1 <= 16) k_bwd_rows<T, 16><<<grid, kWarps * 32, 0, st>>>(P);
    else k_bwd_rows<T, 32><<<grid, kWarps * 32, 0, st>>>(P);
    k_bwd_compress<<<dim3((unsigned)p->Mb, (unsigned)w.H), 128, 0, st>>>(P);
    const int64_t n = p->N * w.H * w.D;
    k_bwd_cast<T><<<(unsigned)cdiv(n, 256), 256, 0, st>>>(P.dk32, P.dv32, n, (T*)dk, (T*)dv);
    note_launch(3);
    return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

}  // namespace

ssa_status_t launch_backward(Plan* p, const Workspace& w, const void* q, const void* k,
                             const void* v, const float* gates, const float* wc, const void* dout,
                             void* dq, void* dk, void* dv, cudaStream_t st) {
    const int64_t nd = p->N * w.H * w.D, cd = (int64_t)w.H * p->Mb * w.D;
    float* acc = (float*)p->alloc(sizeof(float) * (2 * nd + 2 * cd), st, p->alloc_ctx);
    if (!acc) return SSA_ERR_ALLOC;
    if (cudaMemsetAsync(acc, 0, sizeof(float) * (2 * nd + 2 * cd), st)) return SSA_ERR_CUDA;
    BwdParams P;
    P.q = q;
    P.k = k;
    P.v = v;
    P.dout = dout;
    P.kc = w.kc;
    P.vc = w.vc;
    P.gates = gates;
    P.wc = wc;
    P.perm = p->perm;
    P.tok_blk = p->tok_blk;
    P.tok_pos = p->tok_pos;
    P.blk_off = p->blk_off;
    P.seq_blk = p->seq_blk_d;
    P.seqs = p->d_seqs;
    P.nbr_off = p->nbr_off32;
    P.nbr_idx = p->nbr_idx;
    P.sel = w.sel;
    P.dq = dq;
    P.dk32 = acc;
    P.dv32 = acc + nd;
    P.dkc = acc + 2 * nd;
    P.dvc = acc + 2 * nd + cd;
    P.N = p->N;
    P.Mb = p->Mb;
    P.H = w.H;
    P.D = w.D;
    P.topk = w.k;
    P.B = p->B;
    P.scale = (float)(1.0 / sqrt((double)w.D));
    ssa_status_t rc;
    switch (w.dtype) {
    case SSA_F32: rc = run<float>(p, w, P, dk, dv, st); break;
    case SSA_BF16: rc = run<__nv_bfloat16>(p, w, P, dk, dv, st); break;
    default: rc = run<__half>(p, w, P, dk, dv, st); break;
    }
    p->release(acc, st, p->alloc_ctx);
    return rc;
}

}  // namespace ssa
