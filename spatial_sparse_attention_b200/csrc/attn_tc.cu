// Tensor-core (tcgen05 / TMEM) forward of Spatial Sparse Attention for bf16 and fp16 inputs,
// fp32 accumulation. Rows a4-a8 of the method (Direct3D-S2 summary page, "Technical principles",
// SSA item: compressed block tokens, selection of important blocks from the compression module's
// attention scores, local window, gated aggregation).
//
// Dataflow for one forward:
//   k_qmajor   one CTA per (query tile of 128 sorted tokens, head):
//              (1) attention over the compressed tokens of the sequence, with a running
//                  top-(k-1) of the other blocks per row (the own block is slot 0);
//              (2) window attention over the tile's window key union, Chebyshev mask;
//              (3) attention over the own block (tokens of the tile's blocks, same-block mask).
//              Writes base = g0*o_cmp + g2*o_win (fp32), the own-block partial (slot 0) and the
//              selection.
//   k_inv_*    inverts the selection into per-(head, block) query lists (counting sort).
//   k_kbmajor  persistent CTAs; one work item = (head, block, up to 128 queries that selected
//              it): dense 128 x n_b tiles on the tensor cores; writes one normalised partial
//              output and its log2-sum-exp per (query, head, slot).
//   k_combine  merges the k partials of each (query, head) into o_sel and writes
//              out = base + g1*o_sel in token order.
// Every attention tile: S = Q K^T into TMEM (tcgen05.mma, operands in 64-byte-swizzled shared
// memory), softmax rows by the owning thread (TMEM lane = row), P written to shared memory,
// O += P V into TMEM (V as an MN-major operand). Waits are bounded; a wait that runs out sets
// DEV_TIMEOUT, the CTA frees its TMEM and returns.
#include "attn_common.cuh"


namespace ssa {

namespace {

using namespace attn;

// ---------------------------------------------------------------------------------------------
// ---------------------------------------------------------------------------------------------
// key-block-major kernel: the other selected blocks
// ---------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128) k_kbmajor(const FwdParams P, int64_t HMb) {
    using L = Lay<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* g = align1024(smem_raw);
    Ctx c;
    c.g = g;
    c.sb = tc::smem_u32(g);
    c.bar = reinterpret_cast<uint64_t*>(g + L::kMisc);
    c.phase = 0;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(g + L::kMisc + 8);
    const int tid = threadIdx.x;
    const int H = P.H;

    if (tid < 32) {
        tc::tmem_alloc(tslot, 256);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(c.bar, 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    c.tmem = *tslot;

    const T* Q = reinterpret_cast<const T*>(P.q);
    const int64_t total = P.item_off[HMb];
    bool ok = true;
    for (int64_t item = blockIdx.x; item < total && ok; item += gridDim.x) {
        int64_t lo = 0, hi = HMb - 1;   // last hb with item_off[hb] <= item
        while (lo < hi) {
            int64_t mid = (lo + hi + 1) >> 1;
            if (P.item_off[mid] <= item) lo = mid; else hi = mid - 1;
        }
        const int64_t hb = lo;
        const int h = (int)(hb / P.Mb);
        const int32_t b = (int32_t)(hb % P.Mb);
        const int64_t e0 = P.inv_off[hb] + (item - P.item_off[hb]) * 128;
        const int64_t left = P.inv_off[hb + 1] - e0;
        const int nq = left < 128 ? (int)left : 128;
        const bool row_ok = tid < nq;
        const int32_t entry = P.inv_list[e0 + (row_ok ? tid : 0)];
        const int32_t pos = entry >> 5, slot = entry & 31;

        __syncthreads();   // previous item's tiles fully consumed
        load_rows<T, D>(c, L::kQ, 128, [&](int row) -> const T* {
            return row < nq ? Q + ((int64_t)P.perm[P.inv_list[e0 + row] >> 5] * H + h) * D : nullptr;
        });
        const int32_t r0 = P.blk_poff[b], nb = P.blk_off[b + 1] - P.blk_off[b];
        const int32_t nrow = P.blk_poff[b + 1] - r0;
        const T* KS = reinterpret_cast<const T*>(P.ks) + (int64_t)h * P.Npad * D;
        const T* VS = reinterpret_cast<const T*>(P.vs) + (int64_t)h * P.Npad * D;
        float m = -INFINITY, l = 0.0f;
        for (int j0 = 0; j0 < nrow && ok; j0 += 128) {
            const int width = min(128, nrow - j0);
            if (j0 > 0) __syncthreads();
            load_rows<T, D>(c, L::kK, width, [&](int row) -> const T* { return KS + (int64_t)(r0 + j0 + row) * D; });
            load_rows<T, D>(c, L::kV, width, [&](int row) -> const T* { return VS + (int64_t)(r0 + j0 + row) * D; });
            tiles_ready();
            const int lim = nb - j0;
            ok = run_tile<T, D>(c, width, j0 == 0, m, l, P.sl, P.status,
                                [&](int col) { return col < lim; }, [](int, float) {});
        }
        if (ok) store_partial<T, D>(P, pos, h, slot, row_ok, c, m, l);
    }

    tc::fence_before_sync();
    __syncthreads();
    if (tid < 32) {
        tc::fence_after_sync();
        tc::tmem_dealloc(c.tmem, 256);
    }
}

// ---------------------------------------------------------------------------------------------
// selection inversion and merge
// ---------------------------------------------------------------------------------------------
__global__ void k_inv_count(const int32_t* __restrict__ sel, int64_t NH, int H, int k, int64_t Mb,
                            int32_t* __restrict__ inv_cnt) {
    int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= NH) return;
    const int h = (int)(w % H);
    for (int s = 1; s < k; ++s) {
        int32_t b = sel[w * k + s];
        if (b >= 0 && b < Mb) atomicAdd(&inv_cnt[(int64_t)h * Mb + b], 1);
    }
}

__global__ void k_inv_items(const int32_t* __restrict__ inv_cnt, int64_t HMb, int32_t* __restrict__ item_cnt) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < HMb) item_cnt[i] = (inv_cnt[i] + 127) / 128;
}

__global__ void k_inv_fill(const int32_t* __restrict__ sel, int64_t NH, int H, int k, int64_t Mb,
                           const int32_t* __restrict__ inv_off, int32_t* __restrict__ inv_fill,
                           int32_t* __restrict__ inv_list) {
    int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= NH) return;
    const int h = (int)(w % H);
    const int32_t pos = (int32_t)(w / H);
    for (int s = 1; s < k; ++s) {
        int32_t b = sel[w * k + s];
        if (b < 0 || b >= Mb) continue;
        int64_t hb = (int64_t)h * Mb + b;
        inv_list[inv_off[hb] + atomicAdd(&inv_fill[hb], 1)] = (pos << 5) | s;
    }
}

// One warp per (sorted position, head): merge the k partials by their log2-sum-exp weights.
template <typename T, int D>
__global__ void k_combine(const FwdParams P) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= P.N * P.H) return;
    const int h = (int)(w % P.H);
    const int64_t pos = w / P.H;
    const int k = P.k;
    const int32_t* srow = P.sel + w * k;
    const bool valid = lane < k && (lane == 0 || srow[lane] >= 0);
    const float lse = valid ? P.part_lse[w * k + lane] : -INFINITY;
    float mx = lse;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float wgt = valid ? tc::ex2(lse - mx) : 0.0f;
    float tot = wgt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    const int32_t tok = P.perm[pos];
    const float g1 = P.gates[((int64_t)tok * P.H + h) * 3 + 1] / tot;
    const PartT<T>* po = reinterpret_cast<const PartT<T>*>(P.part_o) + w * k * D;
    T* out = reinterpret_cast<T*>(P.out) + ((int64_t)tok * P.H + h) * D;
    const float* brow = P.base + w * D;
#pragma unroll
    for (int d = lane; d < D; d += 32) {
        float acc = 0.0f;
        for (int s = 0; s < k; ++s) {
            const float ws = __shfl_sync(0xffffffffu, wgt, s);
            if (ws != 0.0f) acc += ws * Elem<PartT<T>>::to_f(po[s * D + d]);
        }
        out[d] = Elem<T>::from_f(brow[d] + g1 * acc);
    }
}

__global__ void k_export_sel(const int32_t* __restrict__ sel, const int32_t* __restrict__ tok_pos,
                             int64_t N, int H, int k, int32_t* __restrict__ out) {
    int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_tok = (int64_t)H * k;
    if (e >= N * per_tok) return;
    const int64_t tok = e / per_tok, rest = e % per_tok;
    out[e] = sel[(int64_t)tok_pos[tok] * per_tok + rest];
}

template <typename T, int D, int KM>
bool run_forward(const Plan* p, const FwdParams& P, cudaStream_t st, int num_sms) {
    using L = Lay<D>;
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(k_kbmajor<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        configured = true;
    }
    const Workspace& w = p->ws;
    const int64_t NH = p->N * P.H;
    const int64_t HMb = (int64_t)P.H * p->Mb;
    {
        ProfScope ps("k_qmajor", st);
        if (!launch_qmajor(p, w, P, st)) return false;
    }
    trace_step("k_qmajor", st);
    {
        ProfScope ps("selection_inversion", st);
        cudaMemsetAsync(w.inv_cnt, 0, sizeof(int32_t) * (HMb + 1), st);
        cudaMemsetAsync(w.inv_fill, 0, sizeof(int32_t) * (HMb + 1), st);
        const unsigned g256 = (unsigned)cdiv(NH, 256);
        k_inv_count<<<g256, 256, 0, st>>>(w.sel, NH, P.H, P.k, p->Mb, w.inv_cnt);
        note_launch(2);
        scan_exclusive(w.inv_cnt, w.inv_off, HMb, w.scan_tmp, st);
        k_inv_items<<<(unsigned)cdiv(HMb, 256), 256, 0, st>>>(w.inv_cnt, HMb, w.item_cnt);
        note_launch();
        scan_exclusive(w.item_cnt, w.item_off, HMb, w.scan_tmp, st);
        k_inv_fill<<<g256, 256, 0, st>>>(w.sel, NH, P.H, P.k, p->Mb, w.inv_off, w.inv_fill, w.inv_list);
    }
    trace_step("selection inversion", st);
    {
        ProfScope ps("k_kbmajor", st);
        k_kbmajor<T, D><<<(unsigned)(2 * num_sms), 128, L::kAlloc, st>>>(P, HMb);
    }
    trace_step("k_kbmajor", st);
    {
        ProfScope ps("k_combine", st);
        k_combine<T, D><<<(unsigned)cdiv(NH * 32, 256), 256, 0, st>>>(P);
    }
    trace_step("k_combine", st);
    note_launch(3);
    return true;
}

template <typename T, int D>
bool dispatch_km(const Plan* p, const FwdParams& P, cudaStream_t st, int sms) {
    if (P.k - 1 <= 8) return run_forward<T, D, 8>(p, P, st, sms);
    if (P.k - 1 <= 16) return run_forward<T, D, 16>(p, P, st, sms);
    return run_forward<T, D, 32>(p, P, st, sms);
}

template <typename T>
bool dispatch_d(const Plan* p, const FwdParams& P, int D, cudaStream_t st, int sms) {
    switch (D) {
    case 32: return dispatch_km<T, 32>(p, P, st, sms);
    case 64: return dispatch_km<T, 64>(p, P, st, sms);
    case 96: return dispatch_km<T, 96>(p, P, st, sms);
    default: return dispatch_km<T, 128>(p, P, st, sms);
    }
}

}  // namespace

bool launch_forward_tc(const Plan* p, const Workspace& w, const void* q, const float* gates,
                       void* out, cudaStream_t st) {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    FwdParams P;
    P.q = q;
    P.ks = w.ks;
    P.vs = w.vs;
    P.kc = w.kc;
    P.vc = w.vc;
    P.gates = gates;
    P.perm = p->perm;
    P.tok_blk = p->tok_blk;
    P.tok_pos = p->tok_pos;
    P.blk_off = p->blk_off;
    P.blk_poff = p->blk_poff;
    P.scoord = p->scoord;
    P.qt_pos = p->qt_pos;
    P.qt_len = p->qt_len;
    P.qt_seq = p->qt_seq;
    P.seq_blk = p->seq_blk_d;
    P.wt_off = p->wt_off;
    P.wt_keys = p->wt_keys;
    P.inv_off = w.inv_off;
    P.inv_list = w.inv_list;
    P.item_off = w.item_off;
    P.sel = w.sel;
    P.base = w.base;
    P.part_o = w.part_o;
    P.part_lse = w.part_lse;
    P.out = out;
    P.status = p->d_status;
    P.N = p->N;
    P.Npad = p->Npad;
    P.Mb = p->Mb;
    P.H = w.H;
    P.k = w.k;
    P.r = p->r;
    P.sl = (float)(1.4426950408889634 / sqrt((double)w.D));
    if (w.dtype == SSA_BF16) return dispatch_d<__nv_bfloat16>(p, P, w.D, st, sms);
    return dispatch_d<__half>(p, P, w.D, st, sms);
}

void launch_export_sel(const Plan* p, const Workspace& w, int32_t* sel_out, cudaStream_t st) {
    const int64_t n = p->N * w.H * w.k;
    k_export_sel<<<(unsigned)cdiv(n, 256), 256, 0, st>>>(w.sel, p->tok_pos, p->N, w.H, w.k, sel_out);
    note_launch();
}

}  // namespace ssa
