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
#include <type_traits>

#include "common.cuh"
#include "tc.cuh"

namespace ssa {

namespace {

constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 2 GHz

template <int D>
struct Lay {
    static constexpr uint32_t kChunks = D / 32;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kChunks * tc::kRegion;
    static constexpr uint32_t kV = kK + kChunks * tc::kRegion;
    static constexpr uint32_t kP = kV + kChunks * tc::kRegion;
    static constexpr uint32_t kMeta = kP + 4 * tc::kRegion;   // int4[128]
    static constexpr uint32_t kMisc = kMeta + 128 * 16;      // mbarrier, TMEM slot, flags
    static constexpr uint32_t kBytes = kMisc + 64;
    // request at least ~100 KB so that at most two CTAs (2 x 256 TMEM columns) share an SM
    static constexpr uint32_t kAlloc = (kBytes + 1024 > 102400u) ? kBytes + 1024 : 102400u;
};

struct FwdParams {
    const void* q;
    const void* ks;
    const void* vs;
    const void* kc;
    const void* vc;
    const float* gates;
    const int32_t* perm;
    const int32_t* tok_blk;
    const int32_t* tok_pos;
    const int32_t* blk_off;
    const int32_t* blk_poff;
    const int4* scoord;
    const int32_t* qt_pos;
    const int32_t* qt_len;
    const int32_t* qt_seq;
    const int32_t* seq_blk;
    const int32_t* wt_off;
    const int32_t* wt_keys;
    const int32_t* inv_off;
    const int32_t* inv_list;
    const int32_t* item_off;
    int32_t* sel;
    float* base;
    void* part_o;
    float* part_lse;
    void* out;
    int32_t* status;
    int64_t N, Npad, Mb;
    int H, k, r;
    float sl;   // softmax scale * log2(e)
};

template <typename T>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    if constexpr (std::is_same<T, __half>::value) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    } else {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
}

template <typename T>
__device__ __forceinline__ float unpack_lo(uint32_t v) {
    if constexpr (std::is_same<T, __half>::value) return __half2float(__ushort_as_half((unsigned short)(v & 0xffffu)));
    else return __uint_as_float(v << 16);
}
template <typename T>
__device__ __forceinline__ float unpack_hi(uint32_t v) {
    if constexpr (std::is_same<T, __half>::value) return __half2float(__ushort_as_half((unsigned short)(v >> 16)));
    else return __uint_as_float(v & 0xffff0000u);
}

struct Ctx {
    uint8_t* g;      // generic pointer to the 1024-aligned shared base
    uint32_t sb;     // shared-space address of the same
    uint32_t tmem;   // TMEM base (lane 0, column 0): S at columns [0,128), O at [128, 128+D)
    uint64_t* bar;
    uint32_t phase;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    uint32_t s = tc::smem_u32(p);
    return p + ((1024u - (s & 1023u)) & 1023u);
}

// One key tile (K at Lay::kK, V at Lay::kV, `width` rows, a multiple of 16 <= 128) against the
// query tile at Lay::kQ. Updates the row's running max `m` (log2 units, lazily: O and l are
// rescaled only when the max grows by more than 8) and sum `l`; O accumulates in TMEM.
// `valid(col)` masks keys; `hook(col, z)` sees every valid raw logit (before scaling).
// Returns false (CTA-uniform) if a bounded wait ran out.
template <typename T, int D, class Valid, class Hook>
__device__ __forceinline__ bool run_tile(Ctx& c, int width, bool first, float& m, float& l,
                                         float sl, int32_t* status, Valid valid, Hook hook) {
    using L = Lay<D>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    const int tid = threadIdx.x;
    const uint32_t lane_base = (uint32_t)((tid >> 5) * 32) << 16;
    const uint32_t s_tm = c.tmem + lane_base;
    const uint32_t o_tm = c.tmem + lane_base + 128;

    if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_f16(kBf16, 128, width, false);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_f16_ss(c.tmem, tc::desc_kmajor(c.sb + L::kQ, kk),
                           tc::desc_kmajor(c.sb + L::kK, kk), idesc, kk > 0 ? 1u : 0u);
        tc::mma_commit(c.bar);
    }
    bool ok = tc::mbar_wait(c.bar, c.phase, kWaitCycles);
    c.phase ^= 1u;
    if (__syncthreads_or(!ok)) {
        if (tid == 0) atomicOr(status, DEV_TIMEOUT);
        return false;
    }
    tc::fence_after_sync();

    // pass 1: tile max over valid keys (+ hook)
    float tmax = -INFINITY;
    for (int c0 = 0; c0 < width; c0 += 16) {
        float s[16];
        tc::tmem_ld16(s_tm + c0, s);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            if (valid(c0 + e)) {
                tmax = fmaxf(tmax, s[e]);
                hook(c0 + e, s[e]);
            }
        }
    }
    const float tm = tmax * sl;
    bool rescale = false;
    float alpha = 1.0f;
    if (tm > m + 8.0f) {
        const bool had = m != -INFINITY;
        alpha = had ? tc::ex2(m - tm) : 0.0f;
        rescale = had && !first;
        l *= alpha;
        m = tm;
    }
    // TMEM loads/stores are warp-collective: the O round trip runs for the whole warp when any
    // of its rows needs it (factor 1 for the others)
    if (__any_sync(0xffffffffu, rescale)) {
        const float f = rescale ? alpha : 1.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
            float o[16];
            tc::tmem_ld16(o_tm + c0, o);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] *= f;
            tc::tmem_st16(o_tm + c0, o);
        }
    }
    // pass 2: P = exp2(z*sl - m) into shared memory (row tid, K-major, swizzled)
    const bool live = m != -INFINITY;
    for (int c0 = 0; c0 < width; c0 += 16) {
        float s[16];
        tc::tmem_ld16(s_tm + c0, s);
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float p0 = (live && valid(c0 + 2 * e)) ? tc::ex2(fmaf(s[2 * e], sl, -m)) : 0.0f;
            float p1 = (live && valid(c0 + 2 * e + 1)) ? tc::ex2(fmaf(s[2 * e + 1], sl, -m)) : 0.0f;
            pk[e] = pack2<T>(p0, p1);
            // the row sum uses the rounded weights the MMA multiplies V with, so that the
            // normalised output is an exact convex combination of the rounded weights
            l += unpack_lo<T>(pk[e]) + unpack_hi<T>(pk[e]);
        }
        uint4* dst0 = reinterpret_cast<uint4*>(c.g + L::kP + tc::tile_off(tid, c0 >> 3));
        uint4* dst1 = reinterpret_cast<uint4*>(c.g + L::kP + tc::tile_off(tid, (c0 >> 3) + 1));
        *dst0 = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *dst1 = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_f16(kBf16, 128, D, true);
        for (int kk = 0; kk < width / 16; ++kk)
            tc::mma_f16_ss(c.tmem + 128, tc::desc_kmajor(c.sb + L::kP, kk),
                           tc::desc_mnmajor(c.sb + L::kV, kk), idesc,
                           (first && kk == 0) ? 0u : 1u);
        tc::mma_commit(c.bar);
    }
    ok = tc::mbar_wait(c.bar, c.phase, kWaitCycles);
    c.phase ^= 1u;
    if (__syncthreads_or(!ok)) {
        if (tid == 0) atomicOr(status, DEV_TIMEOUT);
        return false;
    }
    tc::fence_after_sync();
    return true;
}

// cp.async of `rows` rows of D elements (row r from src_of(r), nullptr = zeros) into a
// swizzled tile at shared offset `off`.
template <typename T, int D, class Src>
__device__ __forceinline__ void load_rows(const Ctx& c, uint32_t off, int rows, Src src_of) {
    constexpr int kU = D / 8;
    for (int e = threadIdx.x; e < rows * kU; e += blockDim.x) {
        const int row = e / kU, c16 = e % kU;
        const T* src = src_of(row);
        tc::cp_async16(c.sb + off + tc::tile_off(row, c16), src ? (const void*)(src + c16 * 8) : (const void*)c.g,
                       src ? 16u : 0u);
    }
}

__device__ __forceinline__ void tiles_ready() {
    tc::cp_async_wait_all();
    tc::fence_proxy_async();
    __syncthreads();
}

template <int KM>
__device__ __forceinline__ void topk_insert(float (&tv)[KM], int32_t (&ti)[KM], float z, int32_t b) {
    float cz = z;
    int32_t cb = b;
#pragma unroll
    for (int t = 0; t < KM; ++t) {
        // order: logit descending, then block index ascending (an entry displaced by a larger
        // logit must still pass equal-logit entries with a higher index)
        const bool better = cz > tv[t] || (cz == tv[t] && (unsigned)cb < (unsigned)ti[t]);
        const float ov = tv[t];
        const int32_t oi = ti[t];
        tv[t] = better ? cz : ov;
        ti[t] = better ? cb : oi;
        cz = better ? ov : cz;
        cb = better ? oi : cb;
    }
}

// Reads this row's O (D columns) scaled by `f` into registers chunk by chunk and hands each
// chunk of 16 values to `sink(d0, v)`. Warp-collective: every thread of the CTA calls it.
template <int D, class Sink>
__device__ __forceinline__ void read_o(const Ctx& c, float f, Sink sink) {
    const uint32_t o_tm = c.tmem + ((uint32_t)((threadIdx.x >> 5) * 32) << 16) + 128;
#pragma unroll 1
    for (int d0 = 0; d0 < D; d0 += 16) {
        float o[16];
        tc::tmem_ld16(o_tm + d0, o);
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] *= f;
        sink(d0, o);
    }
}

// Storage type of the per-(query, head, slot) partial outputs: fp16 for fp16 inputs (a partial is
// a convex combination of V rows, so it cannot overflow fp16, and 2^-11 resolution is kept);
// fp32 for bf16 inputs (bf16's 2^-8 resolution would dominate the error budget).
template <typename T>
using PartT = typename std::conditional<std::is_same<T, __nv_bfloat16>::value, float, __half>::type;

// Normalised partial output and its log2-sum-exp for (pos, h, slot). Called by every thread
// (TMEM reads are warp-collective); only rows with `row_ok` store.
template <typename T, int D>
__device__ __forceinline__ void store_partial(const FwdParams& P, int64_t pos, int h, int slot,
                                              bool row_ok, const Ctx& c, float m, float l) {
    using PT = PartT<T>;
    const float inv = row_ok ? 1.0f / l : 0.0f;
    PT* dst = reinterpret_cast<PT*>(P.part_o) + (((int64_t)pos * P.H + h) * P.k + slot) * D;
    read_o<D>(c, inv, [&](int d0, float (&o)[16]) {
        if (!row_ok) return;
        if constexpr (std::is_same<PT, float>::value) {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4*>(dst + d0 + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        } else {
            uint4 a = make_uint4(pack2<__half>(o[0], o[1]), pack2<__half>(o[2], o[3]),
                                 pack2<__half>(o[4], o[5]), pack2<__half>(o[6], o[7]));
            uint4 b = make_uint4(pack2<__half>(o[8], o[9]), pack2<__half>(o[10], o[11]),
                                 pack2<__half>(o[12], o[13]), pack2<__half>(o[14], o[15]));
            reinterpret_cast<uint4*>(dst + d0)[0] = a;
            reinterpret_cast<uint4*>(dst + d0)[1] = b;
        }
    });
    if (row_ok) P.part_lse[((int64_t)pos * P.H + h) * P.k + slot] = m + __log2f(l);
}

// ---------------------------------------------------------------------------------------------
// query-major kernel: compressed attention + top-k, window, own block
// ---------------------------------------------------------------------------------------------
template <typename T, int D, int KM>
__global__ void __launch_bounds__(128) k_qmajor(const FwdParams P) {
    using L = Lay<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* g = align1024(smem_raw);
    Ctx c;
    c.g = g;
    c.sb = tc::smem_u32(g);
    c.bar = reinterpret_cast<uint64_t*>(g + L::kMisc);
    c.phase = 0;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(g + L::kMisc + 8);
    int4* kmeta = reinterpret_cast<int4*>(g + L::kMeta);
    const int tid = threadIdx.x;
    const int tile = blockIdx.x, h = blockIdx.y;
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

    const int32_t p0 = P.qt_pos[tile], len = P.qt_len[tile], seq = P.qt_seq[tile];
    const bool row_ok = tid < len;
    const int32_t pos = p0 + (row_ok ? tid : len - 1);
    const int32_t tok = P.perm[pos];
    const int32_t ob = P.tok_blk[tok];
    const int4 qc = P.scoord[P.blk_poff[ob] + (pos - P.blk_off[ob])];
    const T* Q = reinterpret_cast<const T*>(P.q);
    load_rows<T, D>(c, L::kQ, 128, [&](int row) -> const T* {
        return row < len ? Q + ((int64_t)P.perm[p0 + row] * H + h) * D : nullptr;
    });

    bool ok = true;
    float m, l;
    float* brow = P.base + ((int64_t)pos * H + h) * D;

    // (1) compressed attention over all blocks of the sequence, running top-(k-1)
    {
        const int32_t bl = P.seq_blk[seq], nkeys = P.seq_blk[seq + 1] - bl;
        const T* KC = reinterpret_cast<const T*>(P.kc) + (int64_t)h * P.Mb * D;
        const T* VC = reinterpret_cast<const T*>(P.vc) + (int64_t)h * P.Mb * D;
        float tv[KM];
        int32_t ti[KM];
#pragma unroll
        for (int t = 0; t < KM; ++t) {
            tv[t] = -INFINITY;
            ti[t] = -1;
        }
        m = -INFINITY;
        l = 0.0f;
        for (int j0 = 0; j0 < nkeys && ok; j0 += 128) {
            const int cnt = min(128, nkeys - j0), width = (int)round_up(cnt, 16);
            load_rows<T, D>(c, L::kK, width, [&](int row) -> const T* {
                return row < cnt ? KC + (int64_t)(bl + j0 + row) * D : nullptr;
            });
            load_rows<T, D>(c, L::kV, width, [&](int row) -> const T* {
                return row < cnt ? VC + (int64_t)(bl + j0 + row) * D : nullptr;
            });
            tiles_ready();
            const int32_t bbase = bl + j0;
            ok = run_tile<T, D>(
                c, width, j0 == 0, m, l, P.sl, P.status, [&](int col) { return col < cnt; },
                [&](int col, float z) {
                    const int32_t b = bbase + col;
                    if (b != ob && z > tv[KM - 1]) topk_insert<KM>(tv, ti, z, b);
                });
        }
        if (ok) {
            const float f = row_ok ? P.gates[((int64_t)tok * H + h) * 3 + 0] / l : 0.0f;
            read_o<D>(c, f, [&](int d0, float (&o)[16]) {
                if (!row_ok) return;
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4*>(brow + d0 + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
            });
            if (row_ok) {
                int32_t* srow = P.sel + ((int64_t)pos * H + h) * P.k;
                srow[0] = ob;
#pragma unroll
                for (int t = 0; t < KM; ++t)
                    if (t + 1 < P.k) srow[t + 1] = ti[t];
            }
        }
    }

    // (2) window attention over the tile's key union, Chebyshev mask
    if (ok) {
        const int32_t w0 = P.wt_off[tile], nw = P.wt_off[tile + 1] - w0;
        const T* KS = reinterpret_cast<const T*>(P.ks) + (int64_t)h * P.Npad * D;
        const T* VS = reinterpret_cast<const T*>(P.vs) + (int64_t)h * P.Npad * D;
        const int r = P.r;
        m = -INFINITY;
        l = 0.0f;
        for (int j0 = 0; j0 < nw && ok; j0 += 128) {
            const int cnt = min(128, nw - j0), width = (int)round_up(cnt, 16);
            __syncthreads();   // kmeta of the previous tile is no longer read
            for (int row = tid; row < width; row += blockDim.x)
                kmeta[row] = row < cnt ? P.scoord[P.wt_keys[w0 + j0 + row]] : make_int4(1 << 28, 1 << 28, 1 << 28, -1);
            load_rows<T, D>(c, L::kK, width, [&](int row) -> const T* {
                return row < cnt ? KS + (int64_t)P.wt_keys[w0 + j0 + row] * D : nullptr;
            });
            load_rows<T, D>(c, L::kV, width, [&](int row) -> const T* {
                return row < cnt ? VS + (int64_t)P.wt_keys[w0 + j0 + row] * D : nullptr;
            });
            tiles_ready();
            ok = run_tile<T, D>(
                c, width, j0 == 0, m, l, P.sl, P.status,
                [&](int col) {
                    const int4 kc = kmeta[col];
                    return max(abs(kc.x - qc.x), max(abs(kc.y - qc.y), abs(kc.z - qc.z))) <= r;
                },
                [](int, float) {});
        }
        if (ok) {
            const float f = row_ok ? P.gates[((int64_t)tok * H + h) * 3 + 2] / l : 0.0f;
            read_o<D>(c, f, [&](int d0, float (&o)[16]) {
                if (!row_ok) return;
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    float4 b = *reinterpret_cast<float4*>(brow + d0 + e);
                    *reinterpret_cast<float4*>(brow + d0 + e) =
                        make_float4(b.x + o[e], b.y + o[e + 1], b.z + o[e + 2], b.w + o[e + 3]);
                }
            });
        }
    }

    // (3) own block: the padded rows of the tile's blocks, same-block mask
    if (ok) {
        const int32_t bfirst = P.tok_blk[P.perm[p0]], blast = P.tok_blk[P.perm[p0 + len - 1]];
        const int32_t r0 = P.blk_poff[bfirst], nrow = P.blk_poff[blast + 1] - r0;
        const T* KS = reinterpret_cast<const T*>(P.ks) + (int64_t)h * P.Npad * D;
        const T* VS = reinterpret_cast<const T*>(P.vs) + (int64_t)h * P.Npad * D;
        m = -INFINITY;
        l = 0.0f;
        for (int j0 = 0; j0 < nrow && ok; j0 += 128) {
            const int width = min(128, nrow - j0);   // padded rows: already a multiple of 16
            __syncthreads();
            for (int row = tid; row < width; row += blockDim.x) kmeta[row] = P.scoord[r0 + j0 + row];
            load_rows<T, D>(c, L::kK, width, [&](int row) -> const T* { return KS + (int64_t)(r0 + j0 + row) * D; });
            load_rows<T, D>(c, L::kV, width, [&](int row) -> const T* { return VS + (int64_t)(r0 + j0 + row) * D; });
            tiles_ready();
            ok = run_tile<T, D>(
                c, width, j0 == 0, m, l, P.sl, P.status, [&](int col) { return kmeta[col].w == ob; },
                [](int, float) {});
        }
        if (ok) store_partial<T, D>(P, pos, h, 0, row_ok, c, m, l);
    }

    tc::fence_before_sync();
    __syncthreads();
    if (tid < 32) {
        tc::fence_after_sync();
        tc::tmem_dealloc(c.tmem, 256);
    }
}

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
        if (b >= 0) atomicAdd(&inv_cnt[(int64_t)h * Mb + b], 1);
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
        if (b < 0) continue;
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
void run_forward(const Plan* p, const FwdParams& P, cudaStream_t st, int num_sms) {
    using L = Lay<D>;
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(k_qmajor<T, D, KM>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        cudaFuncSetAttribute(k_kbmajor<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
        configured = true;
    }
    const Workspace& w = p->ws;
    const int64_t NH = p->N * P.H;
    const int64_t HMb = (int64_t)P.H * p->Mb;
    {
        ProfScope ps("k_qmajor", st);
        k_qmajor<T, D, KM><<<dim3((unsigned)p->n_qtiles, (unsigned)P.H), 128, L::kAlloc, st>>>(P);
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
}

template <typename T, int D>
void dispatch_km(const Plan* p, const FwdParams& P, cudaStream_t st, int sms) {
    if (P.k - 1 <= 8) run_forward<T, D, 8>(p, P, st, sms);
    else if (P.k - 1 <= 16) run_forward<T, D, 16>(p, P, st, sms);
    else run_forward<T, D, 32>(p, P, st, sms);
}

template <typename T>
void dispatch_d(const Plan* p, const FwdParams& P, int D, cudaStream_t st, int sms) {
    switch (D) {
    case 32: dispatch_km<T, 32>(p, P, st, sms); break;
    case 64: dispatch_km<T, 64>(p, P, st, sms); break;
    case 96: dispatch_km<T, 96>(p, P, st, sms); break;
    default: dispatch_km<T, 128>(p, P, st, sms); break;
    }
}

}  // namespace

void launch_forward_tc(const Plan* p, const Workspace& w, const void* q, const float* gates,
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
    if (w.dtype == SSA_BF16) dispatch_d<__nv_bfloat16>(p, P, w.D, st, sms);
    else dispatch_d<__half>(p, P, w.D, st, sms);
}

void launch_export_sel(const Plan* p, const Workspace& w, int32_t* sel_out, cudaStream_t st) {
    const int64_t n = p->N * w.H * w.k;
    k_export_sel<<<(unsigned)cdiv(n, 256), 256, 0, st>>>(w.sel, p->tok_pos, p->N, w.H, w.k, sel_out);
    note_launch();
}

}  // namespace ssa
