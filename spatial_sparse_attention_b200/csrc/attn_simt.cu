// fp32 forward of Spatial Sparse Attention on the CUDA cores: the three branches and the gated
// sum for fp32 inputs, where the fp32 tolerance rules out 16-bit tensor-core operands. One warp per (token, head); lanes
// split the head dimension; every branch is an online softmax over its key list:
//   compressed tokens of the sequence (with the running top-(k-1) of the other blocks),
//   the tokens of the selected blocks (own block first), the window neighbour list.
// Direct3D-S2 summary page, "Technical principles", SSA item.
#include "common.cuh"

namespace ssa {

namespace {

constexpr int kWarps = 8;

struct SimtParams {
    const float* q;
    const float* k;
    const float* v;
    const float* kc;   // [H, Mb, D]
    const float* vc;
    const float* gates;
    const int32_t* perm;
    const int32_t* tok_blk;
    const int32_t* tok_pos;
    const int32_t* blk_off;
    const int32_t* seq_blk;
    const SeqInfo* seqs;
    const int32_t* nbr_off;
    const int32_t* nbr_idx;
    int32_t* sel;
    float* out;
    float* bout[3];   // optional per-branch outputs (o_cmp, o_sel, o_win), null when not wanted
    int64_t N, Mb;
    int H, D, topk, B;
    float scale;
};

__device__ __forceinline__ float warp_dot(const float (&q)[4], const float* row, int D, int lane) {
    float s = 0.0f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int d = lane + 32 * t;
        if (d < D) s = fmaf(q[t], row[d], s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
    return __shfl_sync(0xffffffffu, s, 0);   // every lane sees lane 0's sum (identical decisions)
}

struct Online {
    float m = -INFINITY, l = 0.0f, o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    __device__ __forceinline__ void add(float z, const float* vrow, int D, int lane) {
        if (z > m) {
            const float a = m == -INFINITY ? 0.0f : expf(m - z);
            l *= a;
#pragma unroll
            for (int t = 0; t < 4; ++t) o[t] *= a;
            m = z;
        }
        const float p = expf(z - m);
        l += p;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int d = lane + 32 * t;
            if (d < D) o[t] = fmaf(p, vrow[d], o[t]);
        }
    }
};

template <int KM>
__global__ void __launch_bounds__(kWarps * 32) k_forward_simt(const SimtParams P) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= P.N * P.H) return;
    const int64_t i = w / P.H;
    const int h = (int)(w % P.H);
    const int H = P.H, D = P.D;
    const int s = find_seq(P.seqs, P.B, i);
    const int32_t bl = P.seq_blk[s], bh = P.seq_blk[s + 1];
    const int32_t ob = P.tok_blk[i];
    float q[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int d = lane + 32 * t;
        q[t] = d < D ? P.q[(i * H + h) * D + d] : 0.0f;
    }
    // compressed attention + top-(k-1) of the other blocks
    float tv[KM];
    int32_t ti[KM];
#pragma unroll
    for (int t = 0; t < KM; ++t) {
        tv[t] = -INFINITY;
        ti[t] = -1;
    }
    Online cmp;
    for (int32_t b = bl; b < bh; ++b) {
        const float z = warp_dot(q, P.kc + ((int64_t)h * P.Mb + b) * D, D, lane);
        cmp.add(z * P.scale, P.vc + ((int64_t)h * P.Mb + b) * D, D, lane);
        if (b != ob && z > tv[KM - 1]) {
            float cz = z;
            int32_t cb = b;
#pragma unroll
            for (int t = 0; t < KM; ++t) {
                const bool better = cz > tv[t] || (cz == tv[t] && (unsigned)cb < (unsigned)ti[t]);
                const float ov = tv[t];
                const int32_t oi = ti[t];
                tv[t] = better ? cz : ov;
                ti[t] = better ? cb : oi;
                cz = better ? ov : cz;
                cb = better ? oi : cb;
            }
        }
    }
    int32_t* srow = P.sel + ((int64_t)P.tok_pos[i] * H + h) * P.topk;
    if (lane == 0) {
        srow[0] = ob;
#pragma unroll
        for (int t = 0; t < KM; ++t)
            if (t + 1 < P.topk) srow[t + 1] = ti[t];
    }
    // selected blocks: one softmax over all their tokens
    Online sel;
    for (int slot = 0; slot < P.topk; ++slot) {
        int32_t b = ob;
        if (slot > 0) {
            b = -1;
#pragma unroll
            for (int t = 0; t < KM; ++t)
                if (t + 1 == slot) b = ti[t];
        }
        if (b < 0) continue;
        for (int32_t p = P.blk_off[b]; p < P.blk_off[b + 1]; ++p) {
            const int64_t j = P.perm[p];
            const float z = warp_dot(q, P.k + (j * H + h) * D, D, lane);
            sel.add(z * P.scale, P.v + (j * H + h) * D, D, lane);
        }
    }
    // window
    Online win;
    for (int32_t t = P.nbr_off[i]; t < P.nbr_off[i + 1]; ++t) {
        const int64_t j = P.nbr_idx[t];
        const float z = warp_dot(q, P.k + (j * H + h) * D, D, lane);
        win.add(z * P.scale, P.v + (j * H + h) * D, D, lane);
    }
    const float* g = P.gates + (i * H + h) * 3;
    const float a0 = g[0] / cmp.l, a1 = g[1] / sel.l, a2 = g[2] / win.l;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int d = lane + 32 * t;
        if (d < D) P.out[(i * H + h) * D + d] = a0 * cmp.o[t] + a1 * sel.o[t] + a2 * win.o[t];
    }
    const Online* br[3] = {&cmp, &sel, &win};
#pragma unroll
    for (int b = 0; b < 3; ++b) {
        if (!P.bout[b]) continue;
        const float il = 1.0f / br[b]->l;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int d = lane + 32 * t;
            if (d < D) P.bout[b][(i * H + h) * D + d] = br[b]->o[t] * il;
        }
    }
}

}  // namespace

void launch_forward_simt(const Plan* p, const Workspace& w, const void* q, const void* k,
                         const void* v, const float* gates, void* out, const BranchOut& bo,
                         cudaStream_t st) {
    SimtParams P;
    P.q = (const float*)q;
    P.k = (const float*)k;
    P.v = (const float*)v;
    P.kc = (const float*)w.kc;
    P.vc = (const float*)w.vc;
    P.gates = gates;
    P.perm = p->perm;
    P.tok_blk = p->tok_blk;
    P.tok_pos = p->tok_pos;
    P.blk_off = p->blk_off;
    P.seq_blk = p->seq_blk_d;
    P.seqs = p->d_seqs;
    P.nbr_off = p->nbr_off32;
    P.nbr_idx = p->nbr_idx;
    P.sel = w.sel;
    P.out = (float*)out;
    for (int b = 0; b < 3; ++b) P.bout[b] = bo.o[b];
    P.N = p->N;
    P.Mb = p->Mb;
    P.H = w.H;
    P.D = w.D;
    P.topk = w.k;
    P.B = p->B;
    P.scale = (float)(1.0 / sqrt((double)w.D));
    const unsigned grid = (unsigned)cdiv(p->N * w.H, kWarps);
    if (w.k - 1 <= 8) k_forward_simt<8><<<grid, kWarps * 32, 0, st>>>(P);
    else if (w.k - 1 <= 16) k_forward_simt<16><<<grid, kWarps * 32, 0, st>>>(P);
    else k_forward_simt<32><<<grid, kWarps * 32, 0, st>>>(P);
    note_launch();
}

}  // namespace ssa
