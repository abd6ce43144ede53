// Backward of Spatial Sparse Attention (Direct3D-S2 model page, "What is Direct3D-S2?":
// the method has a backward pass, reported ~9.6x faster than baseline sparse attention).
// Gradients of L = sum(dO * out) with respect to Q, K, V, with the block selection held at the
// forward's choice and the rounding of the compressed tokens treated as identity.
//
// For one branch with weights P = softmax(s q.k_j) over its keys, output o = sum_j P_j v_j and gate
// g: dz_j = g P_j (dO.v_j - dO.o), dq = s sum_j dz_j k_j, dk_j = s sum_i dz_ij q_i and
// dv_j = sum_i g_i P_ij dO_i. The branches are computed where their structure is dense:
//   compressed (every query of a sequence against every block): five strided-batched GEMMs per
//     sequence and batch of heads (cuBLAS; TF32 tensor cores for 16-bit inputs, whose values
//     TF32 holds exactly, fp32 for fp32 inputs): S = Q Kc^T and dP = dO Vc^T, a row kernel for
//     the softmax and dZ, then dQ += dZ Kc, dKc = dZ^T Q, dVc = (g P)^T dO;
//   selected and window, query side (k_bwd_rows): one warp per (token, head) walks the row's keys
//     three times (statistics, sum_j P_j dP_j, dq) and keeps each branch's log-sum-exp and that
//     sum for the key side;
//   selected and window, key side (k_bwd_keys): one warp per (token, head) walks the queries that
//     selected the token's block (an inverted selection list) and the token's window neighbours
//     (the window relation is symmetric) and accumulates dk_j, dv_j in registers: no atomics;
//   k_bwd_compress: dK_j += (1/n_b) dKc_b Wc^T for every token of block b (same for V);
//   casts of the fp32 accumulators to the input type.
#include <cublas_v2.h>

#include "common.cuh"

namespace ssa {

namespace {

constexpr int kWarps = 8;

struct BwdParams {
    const void* q;
    const void* k;
    const void* v;
    const void* dout;
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
    const int32_t* inv_off;    // [H * Mb + 1] queries that selected each (head, block): CSR
    const int32_t* inv_tok;    // tokens
    float* stats;              // [N, H, 4]: selected lse, sum P dP; window lse, sum P dP
    float* dq32;
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

__device__ __forceinline__ float warp_sum(float s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Lane L holds elements [4L, 4L + 4) of a D-vector (D <= 128, a multiple of 32): one 8-byte
// (16-bit types) or 16-byte (fp32) load per row.
template <typename T>
__device__ __forceinline__ void load4(const T* base, int64_t row, int D, int lane, float (&x)[4]) {
    if (4 * lane >= D) {
        x[0] = x[1] = x[2] = x[3] = 0.0f;
        return;
    }
    if constexpr (std::is_same<T, float>::value) {
        const float4 v = *reinterpret_cast<const float4*>(base + row + 4 * lane);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
        const uint2 v = *reinterpret_cast<const uint2*>(base + row + 4 * lane);
        const T* e = reinterpret_cast<const T*>(&v);
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = Elem<T>::to_f(e[c]);
    }
}

template <typename T>
__device__ __forceinline__ void load_row(const void* base, int64_t row, int D, int lane, float (&x)[4]) {
    load4<T>(reinterpret_cast<const T*>(base), row, D, lane, x);
}

// Keys are visited four at a time (independent loads and reductions in flight). A visitor gets
// the element offsets of up to four key rows.
struct Rows4 {
    int64_t r[4];
    int n;
};

// The selected blocks' tokens (slot order), then nothing else: calls f(batch) for batches of 4.
template <class F>
__device__ __forceinline__ void visit_selected(const int32_t* srow, int topk, const int32_t* blk_off,
                                               const int32_t* perm, int H, int h, int D, F&& f) {
    Rows4 bt;
    bt.n = 0;
    for (int t = 0; t < topk; ++t) {
        const int32_t b = srow[t];
        if (b < 0) continue;
        for (int32_t e = blk_off[b]; e < blk_off[b + 1]; ++e) {
            bt.r[bt.n++] = ((int64_t)perm[e] * H + h) * D;
            if (bt.n == 4) {
                f(bt);
                bt.n = 0;
            }
        }
    }
    if (bt.n) f(bt);
}

template <class F>
__device__ __forceinline__ void visit_list(const int32_t* idx, int32_t n, int H, int h, int D, F&& f) {
    Rows4 bt;
    for (int32_t e = 0; e < n; e += 4) {
        bt.n = min(4, n - e);
#pragma unroll
        for (int u = 0; u < 4; ++u) bt.r[u] = u < bt.n ? ((int64_t)idx[e + u] * H + h) * D : 0;
        f(bt);
    }
}

// Warp sums of eight values (a[0..3], b[0..3]), returned to every lane: a reduce-scatter that
// halves the values each step (lanes that differ in bit 4, then 3, then 2 exchange the half the
// other keeps), sums over bits 1 and 0, then a gather from the lane holding each total (17
// shuffles instead of 40).
__device__ __forceinline__ void warp_sum8(float (&a)[4], float (&b)[4]) {
    const int lane = threadIdx.x & 31;
    const bool h4 = lane & 16, h3 = lane & 8, h2 = lane & 4;
    float w4[4], w2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = h4 ? a[i] : b[i];
        const float keep = h4 ? b[i] : a[i];
        w4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = h3 ? w4[i] : w4[2 + i];
        const float keep = h3 ? w4[2 + i] : w4[i];
        w2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float w1 = (h2 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, h2 ? w2[0] : w2[1], 4);
    w1 += __shfl_xor_sync(0xffffffffu, w1, 2);
    w1 += __shfl_xor_sync(0xffffffffu, w1, 1);
    // the total of value k = 4 (bit 4) + 2 (bit 3) + (bit 2) is in lanes 4k .. 4k + 3
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        a[i] = __shfl_sync(0xffffffffu, w1, 4 * i);
        b[i] = __shfl_sync(0xffffffffu, w1, 16 + 4 * i);
    }
}

// Query side of one branch over the keys a visitor yields: two passes. Pass 1 keeps the running
// maximum m, l = sum e^(z - m) and t = sum e^(z - m) dP (dP = g dO.v), so that the branch's
// log-sum-exp is m + log l and sum_j P_j dP_j = t / l; pass 2 adds s sum_j dz_j k_j to dq.
template <typename T, class Visit>
__device__ void branch_rows(const BwdParams& P, Visit visit, float g, const float (&q)[4], const float (&go)[4],
                            float (&dq)[4], int lane, float& lse, float& pdp) {
    const int D = P.D;
    const T* K = reinterpret_cast<const T*>(P.k);
    const T* V = reinterpret_cast<const T*>(P.v);
    float m = -INFINITY, l = 0.0f, tsum = 0.0f;
    visit([&](const Rows4& bt) {
        float zq[4], zv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            zq[u] = zv[u] = 0.0f;
            if (u < bt.n) {
                float kx[4], vx[4];
                load4<T>(K, bt.r[u], D, lane, kx);
                load4<T>(V, bt.r[u], D, lane, vx);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    zq[u] = fmaf(q[c], kx[c], zq[u]);
                    zv[u] = fmaf(go[c], vx[c], zv[u]);
                }
            }
        }
        warp_sum8(zq, zv);
        float bm = -INFINITY;
#pragma unroll
        for (int u = 0; u < 4; ++u) if (u < bt.n) bm = fmaxf(bm, P.scale * zq[u]);
        if (bm > m) {
            const float f = (m == -INFINITY) ? 0.0f : expf(m - bm);
            l *= f;
            tsum *= f;
            m = bm;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u < bt.n) {
                const float e = expf(P.scale * zq[u] - m);
                l += e;
                tsum = fmaf(e, g * zv[u], tsum);
            }
        }
    });
    lse = l > 0.0f ? m + logf(l) : 0.0f;
    pdp = l > 0.0f ? tsum / l : 0.0f;
    const float ls = lse, pd = pdp;
    visit([&](const Rows4& bt) {
        float zq[4], zv[4], kv[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            zq[u] = zv[u] = 0.0f;
            float vx[4];
            if (u < bt.n) {
                load4<T>(K, bt.r[u], D, lane, kv[u]);
                load4<T>(V, bt.r[u], D, lane, vx);
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) kv[u][c] = vx[c] = 0.0f;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                zq[u] = fmaf(q[c], kv[u][c], zq[u]);
                zv[u] = fmaf(go[c], vx[c], zv[u]);
            }
        }
        warp_sum8(zq, zv);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u < bt.n) {
                const float p = expf(P.scale * zq[u] - ls);
                const float dz = P.scale * p * (g * zv[u] - pd);
#pragma unroll
                for (int t = 0; t < 4; ++t) dq[t] = fmaf(dz, kv[u][t], dq[t]);
            }
        }
    });
}

// Query side of the selected and window branches: one warp per (token, head).
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) k_bwd_rows(const BwdParams P) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= P.N * P.H) return;
    // heads outermost, tokens in block order: the warps in flight share one head's keys in L2
    const int h = (int)(w / P.N);
    const int64_t i = P.perm[w % P.N];
    const int H = P.H, D = P.D;
    float q[4], go[4], dq[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    load_row<T>(P.q, (i * H + h) * D, D, lane, q);
    load_row<T>(P.dout, (i * H + h) * D, D, lane, go);
    const float* g = P.gates + (i * H + h) * 3;
    const int32_t* srow = P.sel + ((int64_t)P.tok_pos[i] * H + h) * P.topk;
    float lse_s, pdp_s, lse_w, pdp_w;
    branch_rows<T>(
        P, [&](auto&& f) { visit_selected(srow, P.topk, P.blk_off, P.perm, H, h, D, f); }, g[1], q, go, dq, lane,
        lse_s, pdp_s);
    const int32_t w0 = P.nbr_off[i];
    branch_rows<T>(
        P, [&](auto&& f) { visit_list(P.nbr_idx + w0, P.nbr_off[i + 1] - w0, H, h, D, f); }, g[2], q, go, dq,
        lane, lse_w, pdp_w);
    if (4 * lane < D)
        *reinterpret_cast<float4*>(P.dq32 + (i * H + h) * D + 4 * lane) = make_float4(dq[0], dq[1], dq[2], dq[3]);
    if (lane == 0) *reinterpret_cast<float4*>(P.stats + (i * H + h) * 4) = make_float4(lse_s, pdp_s, lse_w, pdp_w);
}

// Key side of the selected and window branches: one warp per (token j, head h). Writes dk_j and
// dv_j of these two branches (the compressed branch is added by k_bwd_compress). Queries are
// taken four at a time.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) k_bwd_keys(const BwdParams P) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= P.N * P.H) return;
    // heads outermost, tokens in block order: the warps in flight share one head's queries in L2
    const int h = (int)(w / P.N);
    const int64_t j = P.perm[w % P.N];
    const int H = P.H, D = P.D;
    const T* Q = reinterpret_cast<const T*>(P.q);
    const T* dO = reinterpret_cast<const T*>(P.dout);
    float kj[4], vj[4], dk[4] = {0.0f, 0.0f, 0.0f, 0.0f}, dv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    load_row<T>(P.k, (j * H + h) * D, D, lane, kj);
    load_row<T>(P.v, (j * H + h) * D, D, lane, vj);
    // up to four queries (tokens tk[0..n)) of a branch with gate index gi and statistics at si
    auto quad = [&](const int32_t* tk, int n, int gi, int si) {
        float qi[4][4], goi[4][4], zq[4], zv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            zq[u] = zv[u] = 0.0f;
            if (u < n) {
                const int64_t r = ((int64_t)tk[u] * H + h) * D;
                load4<T>(Q, r, D, lane, qi[u]);
                load4<T>(dO, r, D, lane, goi[u]);
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) qi[u][c] = goi[u][c] = 0.0f;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                zq[u] = fmaf(qi[u][c], kj[c], zq[u]);
                zv[u] = fmaf(goi[u][c], vj[c], zv[u]);
            }
        }
        warp_sum8(zq, zv);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u < n) {
                const int64_t ih = (int64_t)tk[u] * H + h;
                const float2 st = *reinterpret_cast<const float2*>(P.stats + ih * 4 + si);
                const float g = P.gates[ih * 3 + gi];
                const float p = expf(P.scale * zq[u] - st.x);
                const float dz = P.scale * p * (g * zv[u] - st.y);
                const float gp = g * p;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    dk[t] = fmaf(dz, qi[u][t], dk[t]);
                    dv[t] = fmaf(gp, goi[u][t], dv[t]);
                }
            }
        }
    };
    // selected: the queries whose selection holds this token's block
    const int64_t lb = (int64_t)h * P.Mb + P.tok_blk[j];
    const int32_t s0 = P.inv_off[lb], s1 = P.inv_off[lb + 1];
    for (int32_t e = s0; e < s1; e += 4) quad(P.inv_tok + e, min(4, s1 - e), 1, 0);
    // window: the token's neighbours (j is in i's window exactly when i is in j's)
    const int32_t w0 = P.nbr_off[j], w1 = P.nbr_off[j + 1];
    for (int32_t e = w0; e < w1; e += 4) quad(P.nbr_idx + e, min(4, w1 - e), 2, 2);
    if (4 * lane < D) {
        *reinterpret_cast<float4*>(P.dk32 + (j * H + h) * D + 4 * lane) = make_float4(dk[0], dk[1], dk[2], dk[3]);
        *reinterpret_cast<float4*>(P.dv32 + (j * H + h) * D + 4 * lane) = make_float4(dv[0], dv[1], dv[2], dv[3]);
    }
}

// Inverted selection: count, then fill, the tokens that selected each (head, block).
__global__ void k_inv_count(const int32_t* __restrict__ sel, int64_t N, int H, int k, int64_t Mb,
                            int32_t* __restrict__ cnt) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= N * H * k) return;
    const int32_t b = sel[e];
    const int h = (int)((e / k) % H);
    if (b >= 0) atomicAdd(&cnt[(int64_t)h * Mb + b], 1);
}
__global__ void k_inv_fill(const int32_t* __restrict__ sel, const int32_t* __restrict__ perm, int64_t N,
                           int H, int k, int64_t Mb, const int32_t* __restrict__ off, int32_t* __restrict__ cur,
                           int32_t* __restrict__ tok) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= N * H * k) return;
    const int32_t b = sel[e];
    if (b < 0) return;
    const int64_t pos = e / ((int64_t)H * k);
    const int h = (int)((e / k) % H);
    const int64_t c = (int64_t)h * Mb + b;
    tok[off[c] + atomicAdd(&cur[c], 1)] = perm[pos];
}

// Compressed branch, rows of one sequence and batch of heads: S (scores q.Kc) and dP (dO.Vc)
// rows of Mb_s entries become dZ = s g0 P (dP - sum P dP) and G = g0 P, in place.
__global__ void k_bwd_softmax_c(float* __restrict__ S, float* __restrict__ dP, int64_t Ns, int32_t Mbs,
                                int64_t lo, int H, int h0, int hb, const float* __restrict__ gates, float scale) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= Ns * hb) return;
    const int hh = (int)(w / Ns);
    const int64_t n = w % Ns;
    float* srow = S + w * Mbs;   // [hb][Ns][Mbs]
    float* prow = dP + w * Mbs;
    float m = -INFINITY, l = 0.0f, t = 0.0f;   // t = sum e^(z - m) dP
    for (int b = lane; b < Mbs; b += 32) {
        const float z = scale * srow[b];
        if (z > m) {
            const float f = (m == -INFINITY) ? 0.0f : expf(m - z);
            l *= f;
            t *= f;
            m = z;
        }
        const float e = expf(z - m);
        l += e;
        t = fmaf(e, prow[b], t);
    }
    // combine the lanes
    float M = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = (m == -INFINITY) ? 0.0f : expf(m - M);
    const float L = warp_sum(l * f), Tt = warp_sum(t * f);
    const float delta = Tt / L;
    const float g0 = gates[((lo + n) * H + h0 + hh) * 3];
    for (int b = lane; b < Mbs; b += 32) {
        const float p = expf(scale * srow[b] - M) / L;
        srow[b] = scale * g0 * p * (prow[b] - delta);
        prow[b] = g0 * p;
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
__global__ void k_to_f32(const T* __restrict__ a, int64_t n, float* __restrict__ o) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) o[i] = Elem<T>::to_f(a[i]);
}
template <typename T>
__global__ void k_from_f32(const float* __restrict__ a, int64_t n, T* __restrict__ o) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) o[i] = Elem<T>::from_f(a[i]);
}

// fp32 view of a T tensor (a conversion into `buf` unless T is float)
template <typename T>
const float* as_f32(const void* a, int64_t n, float* buf, cudaStream_t st) {
    if (std::is_same<T, float>::value) return static_cast<const float*>(a);
    if (n > 0) {
        k_to_f32<T><<<(unsigned)cdiv(n, 256), 256, 0, st>>>(static_cast<const T*>(a), n, buf);
        note_launch();
    }
    return buf;
}

// fp32 strided-batched GEMM (column-major, as cuBLAS); tf32: TF32 tensor cores, fp32 accumulate
bool sgemm(cublasHandle_t hd, bool tf32, cublasOperation_t ta, cublasOperation_t tb, int m, int n, int k,
           const float* A, int lda, long long sa, const float* B, int ldb, long long sb, float beta,
           float* C, int ldc, long long sc, int batch) {
    const float alpha = 1.0f;
    return cublasGemmStridedBatchedEx(hd, ta, tb, m, n, k, &alpha, A, CUDA_R_32F, lda, sa, B, CUDA_R_32F, ldb, sb,
                                      &beta, C, CUDA_R_32F, ldc, sc, batch,
                                      tf32 ? CUBLAS_COMPUTE_32F_FAST_TF32 : CUBLAS_COMPUTE_32F,
                                      CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS;
}

template <typename T>
ssa_status_t run(Plan* p, const Workspace& w, BwdParams P, const void* q, const void* dout, void* dq,
                 void* dk, void* dv, cudaStream_t st) {
    const int H = w.H, D = w.D;
    const int64_t N = p->N, Mb = p->Mb, nd = N * H * D, cd = (int64_t)H * Mb * D;
    std::vector<void*> tmp;
    auto A = [&](size_t bytes) -> float* {
        void* ptr = p->alloc(std::max<size_t>(bytes, 16), st, p->alloc_ctx);
        if (ptr) tmp.push_back(ptr);
        return static_cast<float*>(ptr);
    };
    auto release = [&]() {
        for (void* ptr : tmp) p->release(ptr, st, p->alloc_ctx);
    };
    ssa_status_t rc = SSA_OK;
    // ---- selected and window branches, query side -------------------------------------------
    const unsigned grid = (unsigned)cdiv(N * H, kWarps);
    if (N > 0) {
        ProfScope ps("bwd_rows", st);
        k_bwd_rows<T><<<grid, kWarps * 32, 0, st>>>(P);
        note_launch();
    }
    // ---- compressed branch: GEMMs per sequence and batch of heads ----------------------------
    if (!p->cublas) {
        cublasHandle_t hd;
        if (cublasCreate(&hd) != CUBLAS_STATUS_SUCCESS) return SSA_ERR_CUDA;
        p->cublas = hd;
    }
    cublasHandle_t hd = static_cast<cublasHandle_t>(p->cublas);
    if (cublasSetStream(hd, st) != CUBLAS_STATUS_SUCCESS ||
        cublasSetMathMode(hd, std::is_same<T, float>::value ? CUBLAS_DEFAULT_MATH : CUBLAS_TF32_TENSOR_OP_MATH) !=
            CUBLAS_STATUS_SUCCESS)
        return SSA_ERR_CUDA;
    const bool f32 = std::is_same<T, float>::value;
    float* q32b = f32 ? nullptr : A(sizeof(float) * nd);
    float* do32b = f32 ? nullptr : A(sizeof(float) * nd);
    float* kc32b = f32 ? nullptr : A(sizeof(float) * cd);
    float* vc32b = f32 ? nullptr : A(sizeof(float) * cd);
    if (!f32 && (!q32b || !do32b || !kc32b || !vc32b)) {
        release();
        return SSA_ERR_ALLOC;
    }
    const float* q32 = as_f32<T>(q, nd, q32b, st);
    const float* do32 = as_f32<T>(dout, nd, do32b, st);
    const float* kc32 = as_f32<T>(w.kc, cd, kc32b, st);
    const float* vc32 = as_f32<T>(w.vc, cd, vc32b, st);
    int64_t most = 1;   // largest rows x blocks of a sequence
    for (int s = 0; s < p->B; ++s)
        most = std::max<int64_t>(most, (p->seqs[s].hi - p->seqs[s].lo) * (p->seq_blk[s + 1] - p->seq_blk[s]));
    // heads per batch: each of the two [heads, rows, blocks] fp32 buffers within 16 GB (all 22
    // heads of a 110k-token sequence at once: the skinny dKc / dVc products get more parallelism)
    const int hb = (int)std::max<int64_t>(1, std::min<int64_t>(H, ((int64_t)1 << 32) / most));
    float* SB = A(sizeof(float) * (size_t)hb * most);
    float* PB = A(sizeof(float) * (size_t)hb * most);
    if (!SB || !PB) {
        release();
        return SSA_ERR_ALLOC;
    }
    const cublasOperation_t NN = CUBLAS_OP_N, TT = CUBLAS_OP_T;
    for (int s = 0; s < p->B && rc == SSA_OK; ++s) {
        ProfScope ps_c("bwd_compressed", st);
        const int64_t lo = p->seqs[s].lo, Ns = p->seqs[s].hi - lo;
        const int64_t bl = p->seq_blk[s], Mbs = p->seq_blk[s + 1] - bl;
        if (Ns == 0 || Mbs == 0) continue;
        for (int h0 = 0; h0 < H && rc == SSA_OK; h0 += hb) {
            const int nb = std::min(hb, H - h0);
            const long long sNM = (long long)Ns * Mbs, sC = (long long)Mb * D;
            const float* qh = q32 + lo * H * D + (int64_t)h0 * D;
            const float* doh = do32 + lo * H * D + (int64_t)h0 * D;
            const float* kch = kc32 + ((int64_t)h0 * Mb + bl) * D;
            const float* vch = vc32 + ((int64_t)h0 * Mb + bl) * D;
            // S = Q Kc^T, dP = dO Vc^T  ([nb][Ns][Mbs] row-major)
            if (!sgemm(hd, !f32, TT, NN, (int)Mbs, (int)Ns, D, kch, D, sC, qh, H * D, D, 0.0f, SB, (int)Mbs, sNM, nb) ||
                !sgemm(hd, !f32, TT, NN, (int)Mbs, (int)Ns, D, vch, D, sC, doh, H * D, D, 0.0f, PB, (int)Mbs, sNM, nb)) {
                rc = SSA_ERR_CUDA;
                break;
            }
            k_bwd_softmax_c<<<(unsigned)cdiv(Ns * nb, kWarps), kWarps * 32, 0, st>>>(
                SB, PB, Ns, (int32_t)Mbs, lo, H, h0, nb, P.gates, P.scale);
            note_launch();
            // dQ += dZ Kc; dKc = dZ^T Q; dVc = G^T dO
            if (!sgemm(hd, !f32, NN, NN, D, (int)Ns, (int)Mbs, kch, D, sC, SB, (int)Mbs, sNM, 1.0f,
                       P.dq32 + lo * H * D + (int64_t)h0 * D, H * D, D, nb) ||
                !sgemm(hd, !f32, NN, TT, D, (int)Mbs, (int)Ns, qh, H * D, D, SB, (int)Mbs, sNM, 0.0f,
                       P.dkc + ((int64_t)h0 * Mb + bl) * D, D, sC, nb) ||
                !sgemm(hd, !f32, NN, TT, D, (int)Mbs, (int)Ns, doh, H * D, D, PB, (int)Mbs, sNM, 0.0f,
                       P.dvc + ((int64_t)h0 * Mb + bl) * D, D, sC, nb))
                rc = SSA_ERR_CUDA;
        }
    }
    if (rc != SSA_OK) {
        release();
        return rc;
    }
    // ---- selected and window branches, key side ---------------------------------------------
    const int64_t nsel = N * H * w.k, ncb = (int64_t)H * Mb;
    int32_t* cnt = reinterpret_cast<int32_t*>(A(sizeof(int32_t) * (ncb + 1)));
    int32_t* off = reinterpret_cast<int32_t*>(A(sizeof(int32_t) * (ncb + 1)));
    int32_t* cur = reinterpret_cast<int32_t*>(A(sizeof(int32_t) * (ncb + 1)));
    int32_t* stmp = reinterpret_cast<int32_t*>(A(sizeof(int32_t) * scan_tmp_len(ncb + 1)));
    int32_t* itok = reinterpret_cast<int32_t*>(A(sizeof(int32_t) * std::max<int64_t>(nsel, 1)));
    if (!cnt || !off || !cur || !stmp || !itok) {
        release();
        return SSA_ERR_ALLOC;
    }
    if (cudaMemsetAsync(cnt, 0, sizeof(int32_t) * (ncb + 1), st) ||
        cudaMemsetAsync(cur, 0, sizeof(int32_t) * (ncb + 1), st)) {
        release();
        return SSA_ERR_CUDA;
    }
    if (nsel > 0) {
        k_inv_count<<<(unsigned)cdiv(nsel, 256), 256, 0, st>>>(w.sel, N, H, w.k, Mb, cnt);
        note_launch();
    }
    scan_exclusive(cnt, off, ncb, stmp, st);
    if (nsel > 0) {
        k_inv_fill<<<(unsigned)cdiv(nsel, 256), 256, 0, st>>>(w.sel, p->perm, N, H, w.k, Mb, off, cur, itok);
        note_launch();
    }
    P.inv_off = off;
    P.inv_tok = itok;
    if (N > 0) {
        ProfScope ps("bwd_keys", st);
        k_bwd_keys<T><<<grid, kWarps * 32, 0, st>>>(P);
        note_launch();
    }
    // ---- compressed branch into dK, dV; results in the input type ------------------------------
    if (Mb > 0) {
        k_bwd_compress<<<dim3((unsigned)Mb, (unsigned)H), 128, 0, st>>>(P);
        note_launch();
    }
    if (nd > 0) {
        k_from_f32<T><<<(unsigned)cdiv(nd, 256), 256, 0, st>>>(P.dq32, nd, (T*)dq);
        k_from_f32<T><<<(unsigned)cdiv(nd, 256), 256, 0, st>>>(P.dk32, nd, (T*)dk);
        k_from_f32<T><<<(unsigned)cdiv(nd, 256), 256, 0, st>>>(P.dv32, nd, (T*)dv);
        note_launch(3);
    }
    rc = cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
    release();
    return rc;
}

}  // namespace

void destroy_blas(Plan* p) {
    if (p->cublas) cublasDestroy(static_cast<cublasHandle_t>(p->cublas));
    p->cublas = nullptr;
}

ssa_status_t launch_backward(Plan* p, const Workspace& w, const void* q, const void* k,
                             const void* v, const float* gates, const float* wc, const void* dout,
                             void* dq, void* dk, void* dv, cudaStream_t st) {
    const int64_t nd = p->N * w.H * w.D, cd = (int64_t)w.H * p->Mb * w.D;
    const size_t bytes = sizeof(float) * (size_t)(3 * nd + 2 * cd + 4 * p->N * w.H);
    float* acc = (float*)p->alloc(std::max<size_t>(bytes, 16), st, p->alloc_ctx);
    if (!acc) return SSA_ERR_ALLOC;
    BwdParams P;
    P.q = q;
    P.k = k;
    P.v = v;
    P.dout = dout;
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
    P.inv_off = nullptr;
    P.inv_tok = nullptr;
    P.dq32 = acc;
    P.dk32 = acc + nd;
    P.dv32 = acc + 2 * nd;
    P.dkc = acc + 3 * nd;
    P.dvc = acc + 3 * nd + cd;
    P.stats = acc + 3 * nd + 2 * cd;
    P.N = p->N;
    P.Mb = p->Mb;
    P.H = w.H;
    P.D = w.D;
    P.topk = w.k;
    P.B = p->B;
    P.scale = (float)(1.0 / sqrt((double)w.D));
    ssa_status_t rc;
    {
        ProfScope ps("backward", st);
        switch (w.dtype) {
        case SSA_F32: rc = run<float>(p, w, P, q, dout, dq, dk, dv, st); break;
        case SSA_BF16: rc = run<__nv_bfloat16>(p, w, P, q, dout, dq, dk, dv, st); break;
        default: rc = run<__half>(p, w, P, q, dout, dq, dk, dv, st); break;
        }
    }
    p->release(acc, st, p->alloc_ctx);
    return rc;
}

}  // namespace ssa
