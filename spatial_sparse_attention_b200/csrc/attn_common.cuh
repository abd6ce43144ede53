// Shared device pieces of the tensor-core attention kernels: shared-memory tile layout, the
// forward parameter block, 16-bit packing, the serial attention tile step, the register top-k and
// the partial-output store.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "tc.cuh"

namespace ssa {
namespace attn {

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

// Same, reading O from the TMEM address `o_tm` (this thread's lane, first O column).
template <typename T, int D>
__device__ __forceinline__ void store_partial_tm(const FwdParams& P, int64_t pos, int h, int slot,
                                                 bool row_ok, uint32_t o_tm, float m, float l) {
    using PT = PartT<T>;
    const float inv = row_ok ? 1.0f / l : 0.0f;
    PT* dst = reinterpret_cast<PT*>(P.part_o) + (((int64_t)pos * P.H + h) * P.k + slot) * D;
#pragma unroll 1
    for (int d0 = 0; d0 < D; d0 += 16) {
        float o[16];
        tc::tmem_ld16(o_tm + d0, o);
        if (!row_ok) continue;
        if constexpr (std::is_same<PT, float>::value) {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4*>(dst + d0 + e) =
                    make_float4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv);
        } else {
            uint32_t u[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) u[e] = pack2<__half>(o[2 * e] * inv, o[2 * e + 1] * inv);
            reinterpret_cast<uint4*>(dst + d0)[0] = make_uint4(u[0], u[1], u[2], u[3]);
            reinterpret_cast<uint4*>(dst + d0)[1] = make_uint4(u[4], u[5], u[6], u[7]);
        }
    }
    if (row_ok) P.part_lse[((int64_t)pos * P.H + h) * P.k + slot] = m + __log2f(l);
}

// Pipelined query-major kernel (attn_qmajor.cu): compressed attention + top-k, own block and
// window for every query tile. Returns false if the tensor maps could not be encoded.
bool launch_qmajor(const Plan* p, const Workspace& w, const FwdParams& P, cudaStream_t st);

}  // namespace attn
}  // namespace ssa
