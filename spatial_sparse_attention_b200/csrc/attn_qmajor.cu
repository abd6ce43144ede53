// Query-major SSA attention, pipelined on the sm_100a tensor cores.
//
// One CTA per (query tile of 128 sorted tokens, head) computes, for every row of the tile, three
// attentions in one stream of 64-key tiles (Direct3D-S2 summary page, "Technical principles",
// SSA item):
//   phase 0  the compressed tokens of the sequence (block mean . Wc), with a running top-(k-1)
//            of the other blocks by compressed logit -> base = g0 * o_cmp, the selection;
//   phase 1  the tokens of the row's own block (same-block mask) -> partial output of slot 0;
//   phase 2  the tokens within Chebyshev radius r (the tile's window key union, distance mask)
//            -> base += g2 * o_win.
// Warp roles (192 threads):
//   warp 0    producer: K and V tiles into two-stage shared-memory rings, by TMA
//             (cp.async.bulk.tensor, 64-byte swizzle) for the contiguous phases 0 and 1 and by
//             cp.async gathers for the window keys, plus the keys' coordinates;
//   warp 1    MMA issuer (one thread): S = Q K^T into one of two TMEM buffers, O += P V;
//   warps 2-5 softmax: one thread per row (its TMEM lane), online softmax with a lazy rescale
//             (O and the row sum are rescaled only when the row max grows by more than 2^8),
//             P written to shared memory in the MMA's operand layout.
// The tensor core computes S of tile j+1 while the softmax works on tile j. K stages are
// released when S has consumed them, V stages (and the key coordinates) when P V has. Every
// wait is bounded; a wait that runs out records DEV_TIMEOUT and the CTA winds down.
#include <cuda.h>

#include "attn_common.cuh"

namespace ssa {
namespace attn {

namespace {

constexpr int kKT = 64;
constexpr int kThreadsQ = 192;

template <int D>
struct QL {
    static constexpr uint32_t kCh = D / 32;
    static constexpr uint32_t kQReg = 128 * 64;   // 32 columns of the 128-row Q tile
    static constexpr uint32_t kKVReg = kKT * 64;  // 32 columns of a 64-row K or V tile
    static constexpr uint32_t kPReg = 128 * 64;   // 32 keys of the 128-row P tile
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kCh * kQReg;
    static constexpr uint32_t kV = kK + 2 * kCh * kKVReg;
    static constexpr uint32_t kP = kV + 2 * kCh * kKVReg;
    static constexpr uint32_t kMeta = kP + 2 * 2 * kPReg;
    static constexpr uint32_t kBar = kMeta + 2 * kKT * 16;
    static constexpr uint32_t kBytes = kBar + 16 * 8 + 16;
    static constexpr uint32_t kAlloc = (kBytes + 1024 > 102400u) ? kBytes + 1024 : 102400u;
    static constexpr uint32_t kTileBytes = kCh * kKVReg;
};

enum : int {
    KFULL = 0, KEMPTY = 2, VFULL = 4, VEMPTY = 6, SFULL = 8, SFREE = 10, PFULL = 12, NBAR = 14
};

struct Sched {
    int nc, no, nw;
    __device__ int total() const { return nc + no + nw; }
    __device__ int phase(int j) const { return j < nc ? 0 : (j < nc + no ? 1 : 2); }
    __device__ int local(int j) const { return j < nc ? j : (j < nc + no ? j - nc : j - nc - no); }
    __device__ bool first(int j) const { return j == 0 || j == nc || j == nc + no; }
};

// Key mask of phase PH for column `col` of the current tile.
template <int PH>
__device__ __forceinline__ bool key_valid(int col, const int4* km, int lim, int4 qc, int32_t ob, int rr) {
    if (PH == 0) return col < lim;
    const int4 kc = km[col];
    if (PH == 1) return kc.w == ob;
    return col < lim && max(abs(kc.x - qc.x), max(abs(kc.y - qc.y), abs(kc.z - qc.z))) <= rr;
}

// v[e] for a per-thread index e, by a tree of selects (stays in registers)
__device__ __forceinline__ float pick16(const float (&v)[16], int e) {
    float a[8], b[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = (e & 1) ? v[2 * i + 1] : v[2 * i];
#pragma unroll
    for (int i = 0; i < 4; ++i) b[i] = (e & 2) ? a[2 * i + 1] : a[2 * i];
    const float c0 = (e & 4) ? b[1] : b[0];
    const float c1 = (e & 4) ? b[3] : b[2];
    return (e & 8) ? c1 : c0;
}

// Pass 1 over one S tile: the row max of the valid keys; in phase 0 also the running top-(k-1)
// of the other blocks (candidates above the current k-1-th logit are collected as a bit mask per
// 16 columns and inserted one by one).
template <int PH, int KM>
__device__ __forceinline__ float softmax_pass1(uint32_t s_tm, const int4* km, int lim, int4 qc,
                                               int32_t ob, int rr, int32_t bbase, float (&tv)[KM],
                                               int32_t (&ti)[KM]) {
    float tmax = -INFINITY;
#pragma unroll 1
    for (int c0 = 0; c0 < kKT; c0 += 16) {
        float sv[16];
        tc::tmem_ld16(s_tm + c0, sv);
        uint32_t cand = 0;
        const float thr = tv[KM - 1];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const bool v = key_valid<PH>(c0 + e, km, lim, qc, ob, rr);
            tmax = fmaxf(tmax, v ? sv[e] : -INFINITY);
            if (PH == 0) cand |= (uint32_t)(v && sv[e] > thr && bbase + c0 + e != ob) << e;
        }
        if (PH == 0) {
            while (cand) {
                const int e = __ffs(cand) - 1;
                cand &= cand - 1;
                topk_insert<KM>(tv, ti, pick16(sv, e), bbase + c0 + e);
            }
        }
    }
    return tmax;
}

// Pass 2: P = 2^(z*sl - m) rounded to T into this row of the P tile; l accumulates the rounded
// weights.
template <typename T, int PH, uint32_t kPReg>
__device__ __forceinline__ void softmax_pass2(uint32_t s_tm, const int4* km, int lim, int4 qc,
                                              int32_t ob, int rr, float sl, float m, uint8_t* pbuf,
                                              int row, float& l) {
    const bool live = m != -INFINITY;
#pragma unroll 1
    for (int c0 = 0; c0 < kKT; c0 += 16) {
        float sv[16];
        tc::tmem_ld16(s_tm + c0, sv);
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const bool v0 = live && key_valid<PH>(c0 + 2 * e, km, lim, qc, ob, rr);
            const bool v1 = live && key_valid<PH>(c0 + 2 * e + 1, km, lim, qc, ob, rr);
            const float a0 = v0 ? tc::ex2(fmaf(sv[2 * e], sl, -m)) : 0.0f;
            const float a1 = v1 ? tc::ex2(fmaf(sv[2 * e + 1], sl, -m)) : 0.0f;
            pk[e] = pack2<T>(a0, a1);
            l += unpack_lo<T>(pk[e]) + unpack_hi<T>(pk[e]);
        }
        const int c16 = c0 >> 3;
        *reinterpret_cast<uint4*>(pbuf + (c16 >> 2) * kPReg + tc::sw64(row, c16 & 3)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(pbuf + ((c16 + 1) >> 2) * kPReg + tc::sw64(row, (c16 + 1) & 3)) =
            make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
}

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, int32_t* status) {
    if (tc::mbar_wait(bar, parity, kWaitCycles)) return true;
    atomicOr(status, DEV_TIMEOUT);
    return false;
}

template <typename T, int D, int KM>
__global__ void __launch_bounds__(kThreadsQ, 2) k_qmajor(const __grid_constant__ FwdParams P,
                                                      const __grid_constant__ CUtensorMap tm_kc,
                                                      const __grid_constant__ CUtensorMap tm_vc,
                                                      const __grid_constant__ CUtensorMap tm_ks,
                                                      const __grid_constant__ CUtensorMap tm_vs) {
    using L = QL<D>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* g = align1024(smem_raw);
    const uint32_t sb = tc::smem_u32(g);
    uint64_t* bar = reinterpret_cast<uint64_t*>(g + L::kBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(g + L::kBar + NBAR * 8);
    int4* meta = reinterpret_cast<int4*>(g + L::kMeta);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, H = P.H;

    // ---- per-CTA schedule -------------------------------------------------------------------
    const int32_t p0 = P.qt_pos[tile], len = P.qt_len[tile], seq = P.qt_seq[tile];
    const int32_t bl = P.seq_blk[seq], nkeys = P.seq_blk[seq + 1] - bl;
    const int32_t bfirst = P.tok_blk[P.perm[p0]], blast = P.tok_blk[P.perm[p0 + len - 1]];
    const int32_t r0 = P.blk_poff[bfirst], nrow = P.blk_poff[blast + 1] - r0;
    const int32_t w0 = P.wt_off[tile], nwin = P.wt_off[tile + 1] - w0;
    Sched sc;
    sc.nc = (nkeys + kKT - 1) / kKT;
    sc.no = (nrow + kKT - 1) / kKT;
    sc.nw = (nwin + kKT - 1) / kKT;
    const int nT = sc.total();

    // ---- setup: TMEM, barriers, Q tile -------------------------------------------------------
    if (warp == 1) {
        tc::tmem_alloc(tslot, 256);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) {
            const bool per_row = (i >= SFREE && i < PFULL + 2);
            tc::mbar_init(&bar[i], per_row ? 128u : 1u);
        }
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tm_kc);
        tc::tma_prefetch_desc(&tm_vc);
        tc::tma_prefetch_desc(&tm_ks);
        tc::tma_prefetch_desc(&tm_vs);
    }
    const T* Q = reinterpret_cast<const T*>(P.q);
    for (int e = tid; e < 128 * (D / 8); e += kThreadsQ) {
        const int row = e / (D / 8), c16 = e % (D / 8);
        const bool ok = row < len;
        const T* src = ok ? Q + ((int64_t)P.perm[p0 + row] * H + h) * D + c16 * 8 : Q;
        tc::cp_async16(sb + L::kQ + (c16 >> 2) * L::kQReg + tc::sw64(row, c16 & 3), src, ok ? 16u : 0u);
    }
    tc::cp_async_wait_all();
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tslot;

    const T* KS = reinterpret_cast<const T*>(P.ks) + (int64_t)h * P.Npad * D;
    const T* VS = reinterpret_cast<const T*>(P.vs) + (int64_t)h * P.Npad * D;

    // P V of tile i has completed. Its barrier (V stage i&1, phase i>>1) is committed right after
    // that MMA. Waits on a barrier's phases must not skip one: a parity wait only tells the
    // current phase from the one before it, and the tensor core may finish a later S before an
    // earlier P V. Every user of these barriers waits for P V of tile i-2 before tile i.
    auto pv_done = [&](int i) -> bool {
        return wait_or_flag(&bar[VEMPTY + (i & 1)], (uint32_t)(i >> 1) & 1u, P.status);
    };

    if (warp == 0) {
        // ================================ producer ============================================
        for (int j = 0; j < nT; ++j) {
            const int ph = sc.phase(j), t = sc.local(j), s = j & 1;
            const uint32_t par_e = (uint32_t)((j >> 1) - 1) & 1u;
            const uint32_t kdst = sb + L::kK + s * L::kTileBytes;
            const uint32_t vdst = sb + L::kV + s * L::kTileBytes;
            const int cnt = ph == 2 ? min(kKT, nwin - kKT * t) : kKT;
            // K tile
            if (j >= 2 && !wait_or_flag(&bar[KEMPTY + s], par_e, P.status)) break;
            if (ph < 2) {
                if (lane == 0) {
                    const CUtensorMap* tm = ph == 0 ? &tm_kc : &tm_ks;
                    const int32_t y = ph == 0 ? (int32_t)(h * P.Mb + bl + kKT * t)
                                              : (int32_t)(h * P.Npad + r0 + kKT * t);
                    tc::mbar_arrive_expect_tx(&bar[KFULL + s], L::kTileBytes);
                    for (int c = 0; c < (int)L::kCh; ++c)
                        tc::tma_load_2d(kdst + c * L::kKVReg, tm, 32 * c, y, &bar[KFULL + s]);
                }
            } else {
                for (int e = lane; e < kKT * (D / 8); e += 32) {
                    const int row = e / (D / 8), c16 = e % (D / 8);
                    const bool ok = row < cnt;
                    const T* src = ok ? KS + (int64_t)P.wt_keys[w0 + kKT * t + row] * D + c16 * 8 : KS;
                    tc::cp_async16(kdst + (c16 >> 2) * L::kKVReg + tc::sw64(row, c16 & 3), src, ok ? 16u : 0u);
                }
                tc::cp_async_wait_all();
                tc::fence_proxy_async();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bar[KFULL + s]);
            }
            // V tile and the keys' coordinates
            if (j >= 2 && !wait_or_flag(&bar[VEMPTY + s], par_e, P.status)) break;
            if (ph > 0) {
                for (int i = lane; i < kKT; i += 32) {
                    int4 mc = make_int4(1 << 28, 1 << 28, 1 << 28, -1);
                    if (ph == 1 && kKT * t + i < nrow) mc = P.scoord[r0 + kKT * t + i];
                    if (ph == 2 && i < cnt) mc = P.scoord[P.wt_keys[w0 + kKT * t + i]];
                    meta[s * kKT + i] = mc;
                }
                __syncwarp();
            }
            if (ph < 2) {
                if (lane == 0) {
                    const CUtensorMap* tm = ph == 0 ? &tm_vc : &tm_vs;
                    const int32_t y = ph == 0 ? (int32_t)(h * P.Mb + bl + kKT * t)
                                              : (int32_t)(h * P.Npad + r0 + kKT * t);
                    tc::mbar_arrive_expect_tx(&bar[VFULL + s], L::kTileBytes);
                    for (int c = 0; c < (int)L::kCh; ++c)
                        tc::tma_load_2d(vdst + c * L::kKVReg, tm, 32 * c, y, &bar[VFULL + s]);
                }
            } else {
                for (int e = lane; e < kKT * (D / 8); e += 32) {
                    const int row = e / (D / 8), c16 = e % (D / 8);
                    const bool ok = row < cnt;
                    const T* src = ok ? VS + (int64_t)P.wt_keys[w0 + kKT * t + row] * D + c16 * 8 : VS;
                    tc::cp_async16(vdst + (c16 >> 2) * L::kKVReg + tc::sw64(row, c16 & 3), src, ok ? 16u : 0u);
                }
                tc::cp_async_wait_all();
                tc::fence_proxy_async();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bar[VFULL + s]);
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ==========================================
        if (lane == 0) {
            const uint32_t idesc_s = tc::idesc_f16(kBf16, 128, kKT, false);
            const uint32_t idesc_o = tc::idesc_f16(kBf16, 128, D, true);
            auto issue_pv = [&](int i) -> bool {
                const int bb = i & 1;
                if (!wait_or_flag(&bar[PFULL + bb], (uint32_t)(i >> 1) & 1u, P.status)) return false;
                if (!wait_or_flag(&bar[VFULL + bb], (uint32_t)(i >> 1) & 1u, P.status)) return false;
                tc::fence_after_sync();
                const uint32_t pbase = sb + L::kP + bb * 2 * L::kPReg;
                const uint32_t vbase = sb + L::kV + bb * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kKT / 16; ++kk)
                    tc::mma_f16_ss(tmem + 128, tc::desc_kmajor_r(pbase, kk, L::kPReg),
                                   tc::desc_mnmajor_r(vbase, kk, L::kKVReg), idesc_o,
                                   (sc.first(i) && kk == 0) ? 0u : 1u);
                tc::mma_commit(&bar[VEMPTY + bb]);   // P V of tile i done: V stage, P buffer, O
                return true;
            };
            bool ok = true;
            for (int j = 0; j < nT && ok; ++j) {
                const int s = j & 1;
                if (!wait_or_flag(&bar[KFULL + s], (uint32_t)(j >> 1) & 1u, P.status)) break;
                if (j >= 2 && !wait_or_flag(&bar[SFREE + s], (uint32_t)((j >> 1) - 1) & 1u, P.status)) break;
                tc::fence_after_sync();
                const uint32_t kbase = sb + L::kK + s * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::mma_f16_ss(tmem + s * kKT, tc::desc_kmajor_r(sb + L::kQ, kk, L::kQReg),
                                   tc::desc_kmajor_r(kbase, kk, L::kKVReg), idesc_s, kk > 0 ? 1u : 0u);
                tc::mma_commit(&bar[SFULL + s]);
                tc::mma_commit(&bar[KEMPTY + s]);
                if (j >= 1) ok = issue_pv(j - 1);
            }
            if (ok && nT > 0) issue_pv(nT - 1);
        }
    } else {
        // ================================ softmax =============================================
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t o_tm = tmem + lane_base + 128;
        const bool row_ok = row < len;
        const int32_t pos = p0 + (row_ok ? row : len - 1);
        const int32_t tok = P.perm[pos];
        const int32_t ob = P.tok_blk[tok];
        const int4 qc = P.scoord[P.blk_poff[ob] + (pos - P.blk_off[ob])];
        const float* gt = P.gates + ((int64_t)tok * H + h) * 3;
        const float gc = gt[0], gw = gt[2];
        float* brow = P.base + ((int64_t)pos * H + h) * D;
        const int rr = P.r;
        const float sl = P.sl;
        float tv[KM];
        int32_t ti[KM];
#pragma unroll
        for (int u = 0; u < KM; ++u) {
            tv[u] = -INFINITY;
            ti[u] = -1;
        }
        float m = -INFINITY, l = 0.0f;

        // O of the finished phase `ph` -> its destination (warp-collective TMEM reads)
        auto epilogue = [&](int ph) {
            tc::fence_after_sync();
            if (ph == 1) {
                store_partial_tm<T, D>(P, pos, h, 0, row_ok, o_tm, m, l);
                return;
            }
            const float f = row_ok ? (ph == 0 ? gc : gw) / l : 0.0f;
#pragma unroll 1
            for (int d0 = 0; d0 < D; d0 += 16) {
                float o[16];
                tc::tmem_ld16(o_tm + d0, o);
                if (!row_ok) continue;
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    float4 v = make_float4(o[e] * f, o[e + 1] * f, o[e + 2] * f, o[e + 3] * f);
                    if (ph == 2) {
                        const float4 b = *reinterpret_cast<const float4*>(brow + d0 + e);
                        v.x += b.x; v.y += b.y; v.z += b.z; v.w += b.w;
                    }
                    *reinterpret_cast<float4*>(brow + d0 + e) = v;
                }
            }
            if (ph == 0 && row_ok) {
                int32_t* srow = P.sel + ((int64_t)pos * H + h) * P.k;
                srow[0] = ob;
#pragma unroll
                for (int u = 0; u < KM; ++u)
                    if (u + 1 < P.k) srow[u + 1] = ti[u];
            }
        };

        bool ok = true;
        for (int j = 0; j < nT; ++j) {
            const int ph = sc.phase(j), t = sc.local(j), b = j & 1;
            if (sc.first(j) && j > 0) {
                if (!(ok = pv_done(j - 1))) break;
                epilogue(sc.phase(j - 1));
                m = -INFINITY;
                l = 0.0f;
            }
            if (!(ok = wait_or_flag(&bar[SFULL + b], (uint32_t)(j >> 1) & 1u, P.status))) break;
            if (ph > 0 && !(ok = wait_or_flag(&bar[VFULL + b], (uint32_t)(j >> 1) & 1u, P.status))) break;
            tc::fence_after_sync();
            const uint32_t s_tm = tmem + lane_base + b * kKT;
            const int4* km = meta + b * kKT;
            const int lim = ph == 0 ? nkeys - kKT * t : nwin - kKT * t;
            const int32_t bbase = bl + kKT * t;
            // pass 1: tile max (+ running top-k of the other blocks in phase 0)
            const float tmax =
                ph == 0 ? softmax_pass1<0, KM>(s_tm, km, lim, qc, ob, rr, bbase, tv, ti)
                : ph == 1 ? softmax_pass1<1, KM>(s_tm, km, lim, qc, ob, rr, bbase, tv, ti)
                          : softmax_pass1<2, KM>(s_tm, km, lim, qc, ob, rr, bbase, tv, ti);
            const float tm = tmax * sl;
            bool rescale = false;
            float alpha = 1.0f;
            if (tm > m + 8.0f) {
                const bool had = m != -INFINITY;
                alpha = had ? tc::ex2(m - tm) : 0.0f;
                rescale = had && !sc.first(j);
                l *= alpha;
                m = tm;
            }
            if (__any_sync(0xffffffffu, rescale)) {
                // O must hold P V of the previous tile before it is rescaled
                if (!(ok = pv_done(j - 1))) break;
                tc::fence_after_sync();
                const float f = rescale ? alpha : 1.0f;
#pragma unroll 1
                for (int d0 = 0; d0 < D; d0 += 16) {
                    float o[16];
                    tc::tmem_ld16(o_tm + d0, o);
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] *= f;
                    tc::tmem_st16(o_tm + d0, o);
                }
            }
            // P buffer b was last read by P V of tile j-2: wait for it explicitly (its completion
            // releases V stage b), MMA completion order is not relied upon
            if (j >= 2 && !(ok = wait_or_flag(&bar[VEMPTY + b], (uint32_t)((j >> 1) - 1) & 1u, P.status)))
                break;
            // pass 2: P = 2^(z*sl - m), rounded to T, into P buffer b (this row, swizzled)
            uint8_t* pbuf = g + L::kP + b * 2 * L::kPReg;
            if (ph == 0) softmax_pass2<T, 0, L::kPReg>(s_tm, km, lim, qc, ob, rr, sl, m, pbuf, row, l);
            else if (ph == 1) softmax_pass2<T, 1, L::kPReg>(s_tm, km, lim, qc, ob, rr, sl, m, pbuf, row, l);
            else softmax_pass2<T, 2, L::kPReg>(s_tm, km, lim, qc, ob, rr, sl, m, pbuf, row, l);
            tc::fence_proxy_async();
            tc::fence_before_sync();
            tc::mbar_arrive(&bar[SFREE + b]);
            tc::mbar_arrive(&bar[PFULL + b]);
        }
        if (ok && nT > 0 && pv_done(nT - 1))
            epilogue(sc.phase(nT - 1));
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

// ---- host: tensor maps -------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)f;
    }
    return fn;
}

// rows x D matrix of 16-bit elements, boxes of 32 columns x 64 rows, 64-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int D, bool bf16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {32, (cuuint32_t)kKT};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, int KM>
bool run(const Plan* p, const FwdParams& P, const CUtensorMap* tm, cudaStream_t st) {
    using L = QL<D>;
    static_assert(L::kAlloc <= 227u * 1024u, "shared-memory layout exceeds the per-CTA limit");
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(k_qmajor<T, D, KM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)L::kAlloc) != cudaSuccess)
            return false;
        configured = true;
    }
    k_qmajor<T, D, KM><<<dim3((unsigned)p->n_qtiles, (unsigned)P.H), kThreadsQ, L::kAlloc, st>>>(
        P, tm[0], tm[1], tm[2], tm[3]);
    return cudaPeekAtLastError() == cudaSuccess;
}

template <typename T, int D>
bool run_km(const Plan* p, const FwdParams& P, const CUtensorMap* tm, cudaStream_t st) {
    if (P.k - 1 <= 8) return run<T, D, 8>(p, P, tm, st);
    if (P.k - 1 <= 16) return run<T, D, 16>(p, P, tm, st);
    return run<T, D, 32>(p, P, tm, st);
}

}  // namespace

bool launch_qmajor(const Plan* p, const Workspace& w, const FwdParams& P, cudaStream_t st) {
    const bool bf16 = w.dtype == SSA_BF16;
    CUtensorMap tm[4];
    if (!make_map(&tm[0], w.kc, (int64_t)w.H * p->Mb, w.D, bf16) ||
        !make_map(&tm[1], w.vc, (int64_t)w.H * p->Mb, w.D, bf16) ||
        !make_map(&tm[2], w.ks, (int64_t)w.H * p->Npad, w.D, bf16) ||
        !make_map(&tm[3], w.vs, (int64_t)w.H * p->Npad, w.D, bf16))
        return false;
    note_launch();
    switch (w.D) {
    case 32: return bf16 ? run_km<__nv_bfloat16, 32>(p, P, tm, st) : run_km<__half, 32>(p, P, tm, st);
    case 64: return bf16 ? run_km<__nv_bfloat16, 64>(p, P, tm, st) : run_km<__half, 64>(p, P, tm, st);
    case 96: return bf16 ? run_km<__nv_bfloat16, 96>(p, P, tm, st) : run_km<__half, 96>(p, P, tm, st);
    default: return bf16 ? run_km<__nv_bfloat16, 128>(p, P, tm, st) : run_km<__half, 128>(p, P, tm, st);
    }
}

}  // namespace attn
}  // namespace ssa
