// Fused forward of Spatial Sparse Attention on the sm_100a tensor cores, bf16 / fp16 inputs with
// fp32 accumulation (Direct3D-S2 summary page, "Technical principles", SSA item: compressed block
// tokens, selection of the important blocks from the compression branch's attention scores, a
// local window, and the gated sum of the three branches).
//
// One CTA per (query tile of 128 tokens in block order, head). The CTA streams 64-key tiles
// through three phases, each one softmax per row:
//   C  the compressed tokens of the sequence (block mean . Wc). The rows' selected blocks (own
//      block plus the top-(k-1) others by compressed logit) come from the selection kernel.
//   S  the selected tokens: the union over the tile's rows of their k selected blocks, each row
//      masked to its own k blocks (a row's valid keys are k ranges of the union stream). Blocks
//      of at most 7 tokens come from their sequence's packed pool instead when the tile selects
//      more of them than the pool has 8-row groups.
//   W  the tile's window key union (Chebyshev radius r), masked by distance.
// out = g0 o_cmp + g1 o_sel + g2 o_win is assembled in an fp32 row buffer and written in the
// input type after phase W. On request each phase also writes its normalised output (fp32).
//
// Warp roles (192 threads):
//   warp 0    producer: K and V tiles into two-stage shared-memory rings by 1D bulk copies. The
//             K/V copies in global memory are stored as 8-row groups already in the tensor cores'
//             swizzled operand order, so a run of consecutive groups is one copy: the compressed
//             tokens are one run, each selected block is one run (or the small blocks together
//             are the one run of their pool), and the window union is the plan's list of runs
//             (its per-row key masks come from the plan as well);
//   warp 1    MMA issuer (one thread): S = Q K^T into one of two TMEM buffers; O += P V with P
//             read from TMEM (it overwrites S in place);
//   warps 2-5 softmax, one thread per row (its TMEM lane): S into registers once, mask, running
//             max with a lazy rescale (O and the row sum are rescaled only when the max grows by
//             more than 2^8), P = 2^(s - m) rounded to the input type back into TMEM.
// The tensor core computes S of tile j+1 while the softmax works on tile j. Between phases C and S
// the softmax warps build the union of the selected blocks in shared memory (a bitmap over the
// sequence's blocks, aliasing the idle K/V rings) and each row's key ranges.
// Every wait is bounded; a wait that runs out records DEV_TIMEOUT and the CTA winds down.
#include <algorithm>

#include "attn_common.cuh"

namespace ssa {

namespace {

using namespace attn;

constexpr int kKT = 64;          // keys per tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;   // S/P buffers at columns 0 and 64, O at 128

template <int D, int KM>
struct FL {
    static constexpr uint32_t kCh = D / 32;              // 32-element column chunks
    static constexpr uint32_t kQReg = 128 * 64;          // one chunk of the 128-row Q tile
    static constexpr uint32_t kGB = kCh * 512;           // one 8-row group (grouped order)
    static constexpr uint32_t kTile = 8 * kGB;           // one K or V stage: 64 rows
    static constexpr uint32_t kSlots = KM + 1;           // selected blocks per row (bound)
    static constexpr uint32_t kUCap = 128 * kSlots;      // union capacity in blocks
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kCh * kQReg;
    static constexpr uint32_t kV = kK + 2 * kTile;
    static constexpr uint32_t kUnion = kV + 2 * kTile;   // int2 [kUCap+1] (first group, stream group offset)
    static constexpr uint32_t kRange = kUnion + (kUCap + 1) * 8;   // int2 [kSlots][128] key ranges
    // during phase C the union and range area holds one 64-score tile per row (float4 [16][128])
    static constexpr uint32_t kUREnd = kRange + kSlots * 128 * 8;
    static constexpr uint32_t kBar = kUREnd > kUnion + 64u * 128u * 4u ? kUREnd : kUnion + 64u * 128u * 4u;
    static constexpr uint32_t kMisc = kBar + 16 * 8;
    static constexpr uint32_t kBytes = kMisc + 64;
    static constexpr uint32_t kAlloc = kBytes + 1024;
    // the union build's bitmap and word prefix alias the two K and two V stages
    static constexpr uint32_t kScratchWords = (4 * kTile) / 8;
    static constexpr int64_t kMaxSeqBlocks = 32 * (int64_t)kScratchWords;
    static constexpr int kMinBlocks = kAlloc <= 113u * 1024u ? 2 : 1;
};

enum : int { KFULL = 0, KEMPTY = 2, VFULL = 4, PVD = 6, SFULL = 8, PFULL = 10, FIN = 12, NBAR = 13 };
// misc words
enum : int { M_TMEM = 0, M_ABORT = 1, M_U = 2, M_L = 3, M_RED = 4 };

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, int32_t* status,
                                             volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (tc::mbar_wait(bar, parity, kWaitCycles)) return true;
    atomicOr(status, DEV_TIMEOUT);
    *abort_flag = 1;
    return false;
}

// Bits [a, b) of a 64-bit word, a and b clamped to [0, 64].
__device__ __forceinline__ uint64_t span_bits(int a, int b) {
    a = max(a, 0);
    b = min(b, 64);
    if (a >= b) return 0ull;
    const uint64_t hi = b >= 64 ? ~0ull : ((1ull << b) - 1ull);
    return hi & (~0ull << a);
}

// *p += v (four fp32 lanes, one vector reduction; p 16-byte aligned; no value returned)
__device__ __forceinline__ void red_add4(float* p, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

// s[c] = -inf where bit c of vm is clear
__device__ __forceinline__ void apply_bits(float (&s)[64], uint64_t vm) {
    const uint32_t lo = (uint32_t)vm, hi = (uint32_t)(vm >> 32);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        s[e] = (lo >> e) & 1u ? s[e] : -INFINITY;
        s[e + 32] = (hi >> e) & 1u ? s[e + 32] : -INFINITY;
    }
}

// Exclusive prefix sum over the 128 softmax threads (local index t); `red` holds 4 ints.
__device__ __forceinline__ int scan128(int v, int t, int* red, int& total) {
    const int lane = t & 31, w = t >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) red[w] = x;
    tc::named_sync(2, 128);
    int pre = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = red[i];
        pre += i < w ? r : 0;
        tot += r;
    }
    tc::named_sync(2, 128);
    total = tot;
    return pre + x - v;
}

template <typename T, int D, int KM>
__global__ void __launch_bounds__(kThreads, FL<D, KM>::kMinBlocks) k_ssa_fwd(const __grid_constant__ FwdParams P) {
    using L = FL<D, KM>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* g = align1024(smem_raw);
    const uint32_t sb = tc::smem_u32(g);
    uint64_t* bar = reinterpret_cast<uint64_t*>(g + L::kBar);
    int* misc = reinterpret_cast<int*>(g + L::kMisc);
    volatile int* abort_flag = misc + M_ABORT;
    int2* un = reinterpret_cast<int2*>(g + L::kUnion);
    int2* rng = reinterpret_cast<int2*>(g + L::kRange);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, H = P.H;

    // ---- per-CTA schedule --------------------------------------------------------------------
    const int32_t p0 = P.qt_pos[tile], len = P.qt_len[tile], seq = P.qt_seq[tile];
    const int32_t bl = P.seq_blk[seq], nblk = P.seq_blk[seq + 1] - bl;
    const int32_t cg0 = bl >> 3, cg1 = (bl + nblk + 7) >> 3;   // groups of the compressed tokens
    const int32_t wr0 = P.wr_off[tile], nwr = P.wr_off[tile + 1] - wr0;
    const int nc = (cg1 - cg0 + 7) >> 3;
    const int nw = (P.wg_cnt[tile] + 7) >> 3;
    const int32_t wm0 = P.wm_off[tile];

    // ---- setup: TMEM, barriers, Q tile, zeroed K/V stages --------------------------------------
    if (warp == 1) {
        tc::tmem_alloc(reinterpret_cast<uint32_t*>(misc + M_TMEM), kTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) tc::mbar_init(&bar[i], (i == PFULL || i == PFULL + 1) ? 4u : 1u);
        misc[M_ABORT] = 0;
        tc::fence_mbar_init();
    }
    const T* Q = reinterpret_cast<const T*>(P.q);
    for (int e = tid; e < 128 * (D / 8); e += kThreads) {
        const int row = e / (D / 8), c16 = e % (D / 8);
        const bool ok = row < len;
        const T* src = ok ? Q + ((int64_t)P.perm[p0 + row] * H + h) * D + c16 * 8 : Q;
        tc::cp_async16(sb + L::kQ + (c16 >> 2) * L::kQReg + tc::sw64(row, c16 & 3), src, ok ? 16u : 0u);
    }
    // groups a tile does not fill keep the previous contents; start from zeros (finite) so that
    // masked keys (weight 0) never meet a non-finite V entry
    for (uint32_t o = tid * 16u; o < 4u * L::kTile; o += kThreads * 16u)
        *reinterpret_cast<uint4*>(g + L::kK + o) = make_uint4(0u, 0u, 0u, 0u);
    // attention prologue: the rotary table (frequency and axis of each channel pair) and the
    // query weights, in the union area (unused until phase C)
    double* pro_freq = reinterpret_cast<double*>(g + L::kUnion);
    int* pro_axis = reinterpret_cast<int*>(g + L::kUnion + 64 * 8);
    float* pro_gamma = reinterpret_cast<float*>(g + L::kUnion + 64 * 12);
    if (P.q_gamma) {
        if (tid < D / 2) rope_pair(D, tid, P.theta, pro_axis[tid], pro_freq[tid]);
        if (tid < D) pro_gamma[tid] = P.q_gamma[tid];
    }
    tc::cp_async_wait_all();
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = (uint32_t)misc[M_TMEM];
    if (P.q_gamma) {
        // the query tile in place: RMS normalisation over the head dimension, then the 3D rotary
        // embedding at the token's coordinates; each softmax thread takes its own row
        if (tid >= 64 && tid - 64 < len)
            qtile_prologue<T, D>(g + L::kQ, L::kQReg, tid - 64, P.perm[p0 + tid - 64], P.coords, pro_freq,
                                 pro_axis, pro_gamma, P.eps);
        tc::fence_proxy_async();   // generic-proxy writes of the tile, read next by the tensor cores
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    }

    if (warp == 0) {
        // ================================ producer ============================================
        // Every phase is a stream of runs of consecutive 8-row groups (compressed tokens: one run;
        // selected blocks: one run per union block, or per kept block plus the pool; window: the
        // plan's runs). A 64-key tile takes the next 8 groups; lane l < 8 copies the part of run
        // ri + l that falls in the tile.
        const uint8_t* ksh = static_cast<const uint8_t*>(P.ks) + (int64_t)h * P.Nks * D * 2;
        const uint8_t* vsh = static_cast<const uint8_t*>(P.vs) + (int64_t)h * P.Nks * D * 2;
        const uint8_t* kch = static_cast<const uint8_t*>(P.kcg) + (int64_t)h * P.Mb8 * D * 2;
        const uint8_t* vch = static_cast<const uint8_t*>(P.vcg) + (int64_t)h * P.Mb8 * D * 2;
        int ri = 0, rskip = 0;   // next run, groups of it already streamed
        int U = 0, ns = 0;
        auto run_of = [&](int ph, int i) -> int2 {
            if (ph == 0) return make_int2(cg0, cg1 - cg0);
            if (ph == 1) return make_int2(un[i].x, un[i + 1].y - un[i].y);
            return P.wr_runs[wr0 + i];
        };
        auto produce = [&](int j, int ph) -> bool {
            const int s = j & 1;
            const uint32_t par_e = (uint32_t)((j >> 1) - 1) & 1u;
            const uint32_t kdst = sb + L::kK + s * L::kTile;
            const uint32_t vdst = sb + L::kV + s * L::kTile;
            const int nruns = ph == 0 ? 1 : (ph == 1 ? U : nwr);
            // this lane's segment: source group, destination group slot, groups
            int32_t first = 0, n = 0;
            if (lane < 8 && ri + lane < nruns) {
                const int2 rr = run_of(ph, ri + lane);
                first = rr.x + (lane == 0 ? rskip : 0);
                n = rr.y - (lane == 0 ? rskip : 0);
            }
            int pre = n;
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, pre, o);
                if (lane >= o) pre += y;
            }
            const int start = pre - n;
            const int take = lane < 8 ? max(0, min(pre, 8) - start) : 0;
            const int total = min(__shfl_sync(0xffffffffu, pre, 7), 8);
            const unsigned over = __ballot_sync(0xffffffffu, lane < 8 && pre > 8);
            if (over) {
                const int Lr = __ffs(over) - 1;
                const int sL = __shfl_sync(0xffffffffu, start, Lr);
                rskip = (Lr == 0 ? rskip : 0) + (8 - sL);
                ri += Lr;
            } else {
                ri = min(ri + 8, nruns);
                rskip = 0;
            }
            if (j >= 2 && !wait_or_flag(&bar[KEMPTY + s], par_e, P.status, abort_flag)) return false;
            const uint8_t* ksrc = ph == 0 ? kch : ksh;
            const uint8_t* vsrc = ph == 0 ? vch : vsh;
            if (lane == 0) tc::mbar_arrive_expect_tx(&bar[KFULL + s], (uint32_t)total * L::kGB);
            __syncwarp();
            if (take > 0)
                tc::bulk_load(kdst + start * L::kGB, ksrc + (int64_t)first * L::kGB, (uint32_t)take * L::kGB,
                              &bar[KFULL + s]);
            // V stage and the key coordinates are free once P V of tile j-2 completed
            if (j >= 2 && !wait_or_flag(&bar[PVD + s], par_e, P.status, abort_flag)) return false;
            if (lane == 0) tc::mbar_arrive_expect_tx(&bar[VFULL + s], (uint32_t)total * L::kGB);
            __syncwarp();
            if (take > 0)
                tc::bulk_load(vdst + start * L::kGB, vsrc + (int64_t)first * L::kGB, (uint32_t)take * L::kGB,
                              &bar[VFULL + s]);
            return true;
        };
        bool ok = true;
        for (int j = 0;; ++j) {
            if (j == nc) {
                __syncwarp();
                tc::named_sync(1, kThreads);   // union of the selected blocks is built
                U = misc[M_U];
                ns = (misc[M_L] + 7) >> 3;
            }
            if (j == nc || j == nc + ns) {
                ri = 0;
                rskip = 0;
            }
            if (j >= nc && (!ok || *abort_flag || j >= nc + ns + nw)) break;
            if (!ok) continue;   // phase C stopped early: still meet the others at the union barrier
            ok = produce(j, j < nc ? 0 : (j < nc + ns ? 1 : 2));
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ==========================================
        const uint32_t idesc_s = tc::idesc_f16(kBf16, 128, kKT, false);
        const uint32_t idesc_o = tc::idesc_f16(kBf16, 128, D, true);
        auto mma_s = [&](int j) -> bool {
            const int b = j & 1;
            if (!wait_or_flag(&bar[KFULL + b], (uint32_t)(j >> 1) & 1u, P.status, abort_flag)) return false;
            // TMEM buffer b holds P of tile j-2 until P V of that tile completed
            if (j >= 2 && !wait_or_flag(&bar[PVD + b], (uint32_t)((j >> 1) - 1) & 1u, P.status, abort_flag))
                return false;
            tc::fence_after_sync();
            const uint32_t kbase = sb + L::kK + b * L::kTile;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                tc::mma_f16_ss(tmem + b * kKT, tc::desc_kmajor_r(sb + L::kQ, kk, L::kQReg),
                               tc::desc_kmajor_g(kbase, kk, L::kCh), idesc_s, kk > 0 ? 1u : 0u);
            tc::mma_commit(&bar[SFULL + b]);
            tc::mma_commit(&bar[KEMPTY + b]);
            return true;
        };
        auto mma_pv = [&](int i, bool first) -> bool {
            const int b = i & 1;
            if (!wait_or_flag(&bar[PFULL + b], (uint32_t)(i >> 1) & 1u, P.status, abort_flag)) return false;
            if (!wait_or_flag(&bar[VFULL + b], (uint32_t)(i >> 1) & 1u, P.status, abort_flag)) return false;
            tc::fence_after_sync();
            const uint32_t vbase = sb + L::kV + b * L::kTile;
#pragma unroll
            for (int kk = 0; kk < kKT / 16; ++kk)
                tc::mma_f16_ts(tmem + 128, tmem + b * kKT + kk * 8, tc::desc_mnmajor_g(vbase, kk, L::kCh),
                               idesc_o, (first && kk == 0) ? 0u : 1u);
            if (kBf16) {
                // bf16: P = P_hi + P_lo, the low part in the buffer's upper 32 columns
#pragma unroll
                for (int kk = 0; kk < kKT / 16; ++kk)
                    tc::mma_f16_ts(tmem + 128, tmem + b * kKT + 32 + kk * 8,
                                   tc::desc_mnmajor_g(vbase, kk, L::kCh), idesc_o, 1u);
            }
            tc::mma_commit(&bar[PVD + b]);   // P V of tile i done: V stage, P buffer, O
            return true;
        };
        if (lane == 0) {
            bool ok = true;
            for (int j = 0; j < nc && ok; ++j) {
                ok = mma_s(j);
                if (ok && j >= 1) ok = mma_pv(j - 1, j - 1 == 0);
            }
            if (ok) mma_pv(nc - 1, nc == 1);
        }
        __syncwarp();
        tc::named_sync(1, kThreads);
        const int ns = (misc[M_L] + 7) >> 3;
        const int nT = nc + ns + nw;
        if (lane == 0) {
            bool ok = !*abort_flag;
            for (int j = nc; j < nT && ok; ++j) {
                ok = mma_s(j);
                if (ok && j > nc) ok = mma_pv(j - 1, j - 1 == nc || j - 1 == nc + ns);
            }
            if (ok && nT > nc) ok = mma_pv(nT - 1, nT - 1 == nc || nT - 1 == nc + ns);
            // drain the tensor pipe before TMEM is released
            tc::mma_commit(&bar[FIN]);
            tc::mbar_wait(&bar[FIN], 0u, kWaitCycles);
        }
        __syncwarp();
    } else {
        // ================================ softmax =============================================
        // One loop over all tiles; the phase only changes how a tile's key mask is formed, so
        // the tile body, the epilogue and the top-k insertion each exist once in the code.
        const int t128 = tid - 64;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t o_tm = tmem + lane_base + 128;
        const bool row_ok = row < len;
        const int32_t pos = p0 + (row_ok ? row : len - 1);
        const int32_t tok = P.perm[pos];
        const int32_t ob = P.tok_blk[tok];
        const float* gt = P.gates + ((int64_t)tok * H + h) * 3;
        // the fp32 row buffer of this (query tile, head): [D/4][128 rows][4] so that a warp's
        // 16-byte accesses to one column quad cover 512 contiguous bytes
        float* brow = P.base + ((int64_t)tile * H + h) * 128 * D + row * 4;
        const float sl = P.sl;
        const int ksel = P.k;
        float m = -INFINITY, l = 0.0f;
        int pv_seen = 0;   // P V completions observed, in order (waits never skip a phase)
        auto wait_pv = [&](int i) -> bool {
            while (pv_seen <= i) {
                if (!wait_or_flag(&bar[PVD + (pv_seen & 1)], (uint32_t)(pv_seen >> 1) & 1u, P.status, abort_flag))
                    return false;
                ++pv_seen;
            }
            return true;
        };
        int ns = 0, nT = 1 << 30, ri = 0, nr = 0;
        int2 rcur = make_int2(0x7fffffff, 0x7fffffff);
        const uint64_t* wrow = P.wmask + (int64_t)wm0 * 128 + row;
        uint64_t wnext = 0ull;
        bool ok = true;
        for (int j = 0;; ++j) {
            // ---- phase boundaries: O of the finished phase to its destination ----------------
            const int ph_end = j == nc ? 0 : (j == nc + ns && ns > 0 ? 1 : (j == nT ? 2 : -1));
            if (ph_end >= 0) {
                ok = __all_sync(0xffffffffu, ok && wait_pv(j - 1));
                if (ok) {
                    tc::fence_after_sync();
                    const float f = row_ok ? gt[ph_end] / l : 0.0f;
                    T* orow = reinterpret_cast<T*>(P.out) + ((int64_t)tok * H + h) * D;
                    // optional branch output (normalised, before the gate), token order
                    float* bo = P.bout[ph_end];
                    if (bo) bo += ((int64_t)tok * H + h) * D;
                    const float il = 1.0f / l;
#pragma unroll 1
                    for (int d0 = 0; d0 < D; d0 += 32) {
                        float o[32];
                        tc::tmem_ld32(o_tm + d0, o);   // warp-collective
                        if (!row_ok) continue;
                        if (bo) {
#pragma unroll
                            for (int e = 0; e < 32; e += 4)
                                *reinterpret_cast<float4*>(bo + d0 + e) =
                                    make_float4(o[e] * il, o[e + 1] * il, o[e + 2] * il, o[e + 3] * il);
                        }
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            float4 a = make_float4(o[e] * f, o[e + 1] * f, o[e + 2] * f, o[e + 3] * f);
                            float4 c = make_float4(o[e + 4] * f, o[e + 5] * f, o[e + 6] * f, o[e + 7] * f);
                            float* bq = brow + (d0 + e) * 128;   // column quad (d0+e)/4, this row
                            if (ph_end == 2) {
                                const float4 a0 = *reinterpret_cast<const float4*>(bq);
                                const float4 c0 = *reinterpret_cast<const float4*>(bq + 512);
                                a.x += a0.x; a.y += a0.y; a.z += a0.z; a.w += a0.w;
                                c.x += c0.x; c.y += c0.y; c.z += c0.z; c.w += c0.w;
                            }
                            if (ph_end == 0) {
                                *reinterpret_cast<float4*>(bq) = a;
                                *reinterpret_cast<float4*>(bq + 512) = c;
                            } else if (ph_end == 1) {
                                // added without reading back (no load latency on this thread)
                                red_add4(bq, a);
                                red_add4(bq + 512, c);
                            } else {
                                *reinterpret_cast<uint4*>(orow + d0 + e) =
                                    make_uint4(pack2<T>(a.x, a.y), pack2<T>(a.z, a.w), pack2<T>(c.x, c.y),
                                               pack2<T>(c.z, c.w));
                            }
                        }
                    }
                }
                m = -INFINITY;
                l = 0.0f;
                if (ph_end == 2) break;
            }
            if (j == nc) {
                // ---- selection, union of the selected blocks, this row's key ranges ----------
                // this row's selection, written by the selection kernel (global block indices)
                int32_t ti[KM];
                const int32_t* srow = P.sel + ((int64_t)pos * H + h) * ksel;
#pragma unroll
                for (int u = 0; u < KM; ++u) ti[u] = u + 1 < ksel ? srow[u + 1] : -1;
                uint32_t* words = reinterpret_cast<uint32_t*>(g + L::kK);
                const int W = (nblk + 31) >> 5;
                int32_t* wpre = reinterpret_cast<int32_t*>(words + W);
                int* red = misc + M_RED;
                for (int i = t128; i < W; i += 128) words[i] = 0u;
                tc::named_sync(2, 128);
                // own block, then the top-(k-1) (local block indices; -1 = none)
                int32_t mine[L::kSlots];
                mine[0] = row_ok ? ob - bl : -1;
#pragma unroll
                for (int u = 0; u < KM; ++u)
                    mine[u + 1] = (row_ok && u + 1 < ksel && ti[u] >= 0) ? ti[u] - bl : -1;
#pragma unroll
                for (int a = 0; a < (int)L::kSlots; ++a)
                    if (mine[a] >= 0 && mine[a] < nblk) atomicOr(&words[mine[a] >> 5], 1u << (mine[a] & 31));
                tc::named_sync(2, 128);
                // union index of every set bit: exclusive prefix of the word popcounts
                const int cw = (W + 127) >> 7;
                const int wl = min(t128 * cw, W), wh = min(wl + cw, W);
                int cnt = 0;
                for (int i = wl; i < wh; ++i) cnt += __popc(words[i]);
                int U = 0;
                int pre = scan128(cnt, t128, red, U);
                U = min(U, (int)L::kUCap);
                for (int i = wl; i < wh; ++i) {
                    wpre[i] = pre;
                    uint32_t wd = words[i];
                    while (wd) {
                        const int bit = __ffs(wd) - 1;
                        wd &= wd - 1;
                        if (pre < (int)L::kUCap) un[pre].x = 32 * i + bit;   // local block index
                        ++pre;
                    }
                }
                tc::named_sync(2, 128);
                // first group and group count of every union block (independent loads); a block
                // with a copy in the sequence's pool (always one group) is marked by a count of -1
                int tcnt = 0;
                for (int u = t128; u < U; u += 128) {
                    const int b = bl + un[u].x;
                    const int2 bi = P.blk_info[b];
                    const bool small = P.blk_tpool[b] >= 0;
                    un[u] = make_int2(bi.x, small ? -1 : (bi.y + 7) >> 3);
                    tcnt += small ? 1 : 0;
                }
                // The pool replaces the small blocks' own groups when it is shorter than they are
                // together (one group each); it then follows the other blocks in the stream.
                int Ut = 0;
                scan128(tcnt, t128, red, Ut);   // its barriers also publish the entries above
                const int2 sp = P.seq_pool[seq];
                const bool use_pool = sp.y > 0 && Ut > sp.y;
                // stream offsets (in groups): exclusive prefix of the blocks' group counts
                const int cu = (U + 127) >> 7;
                const int ul = min(t128 * cu, U), uh = min(ul + cu, U);
                int ssum = 0;
                for (int u = ul; u < uh; ++u) {
                    const int n = un[u].y;
                    ssum += n >= 0 ? n : (use_pool ? 0 : 1);
                }
                int Lg = 0;
                int off = scan128(ssum, t128, red, Lg);
                for (int u = ul; u < uh; ++u) {
                    const int n = un[u].y;
                    un[u].y = off;
                    if (n < 0 && use_pool) un[u].x = -1;   // left out of the stream below
                    off += n >= 0 ? n : (use_pool ? 0 : 1);
                }
                tc::named_sync(2, 128);
                // this row's ranges [first key, last key + 1) in the stream, ascending; with the
                // pool, the keys of pooled blocks follow all others (sort key raised by nblk)
#pragma unroll
                for (int a = 0; a < (int)L::kSlots; ++a) {
                    if (mine[a] >= nblk) mine[a] = -1;
                    if (use_pool && mine[a] >= 0 && P.blk_tpool[bl + mine[a]] >= 0) mine[a] += nblk;
                }
#pragma unroll
                for (int a = 0; a < (int)L::kSlots; ++a) {
                    if (mine[a] < 0) continue;
                    int rank = 0;
#pragma unroll
                    for (int c = 0; c < (int)L::kSlots; ++c) rank += (mine[c] >= 0 && mine[c] < mine[a]) ? 1 : 0;
                    const bool pooled = mine[a] >= nblk;
                    const int b = pooled ? mine[a] - nblk : mine[a];
                    const int nb = P.blk_info[bl + b].y;
                    if (pooled) {
                        const int k0 = 8 * Lg + P.blk_tpool[bl + b];
                        rng[rank * 128 + row] = make_int2(k0, k0 + nb);
                    } else {
                        const int wi = b >> 5;
                        const int u = wpre[wi] + __popc(words[wi] & ((1u << (b & 31)) - 1u));
                        if (u < U) rng[rank * 128 + row] = make_int2(8 * un[u].y, 8 * un[u].y + nb);
                    }
                    ++nr;
                }
                tc::named_sync(2, 128);
                if (use_pool) {
                    // drop the pooled blocks' runs in place, 128 entries at a time (an entry only
                    // moves down, to a place whose entry was read in this or an earlier step),
                    // and append the pool as the last run
                    int kept = 0;
                    for (int c0 = 0; c0 < U; c0 += 128) {
                        const int e = c0 + t128;
                        const int2 v = e < U ? un[e] : make_int2(-1, 0);
                        const int keep = v.x >= 0 ? 1 : 0;
                        int tot = 0;
                        const int at = scan128(keep, t128, red, tot);
                        if (keep) un[kept + at] = v;
                        kept += tot;
                        tc::named_sync(2, 128);
                    }
                    if (t128 == 0) {
                        un[kept] = make_int2(sp.x, Lg);
                        un[kept + 1] = make_int2(0, Lg + sp.y);
                        misc[M_U] = kept + 1;
                        misc[M_L] = Lg + sp.y;
                    }
                } else if (t128 == 0) {
                    un[U] = make_int2(0, Lg);
                    misc[M_U] = U;
                    misc[M_L] = Lg;
                }
                tc::named_sync(1, kThreads);   // the producer may now overwrite the rings
                rcur = nr > 0 ? rng[row] : make_int2(0x7fffffff, 0x7fffffff);
                ns = (misc[M_L] + 7) >> 3;
                nT = nc + ns + nw;
                if (nw > 0) wnext = wrow[0];
            }
            // after a wait ran out the tiles of phase C are skipped up to the union build, which
            // every softmax thread must reach (its barriers have no time limit); then the CTA ends
            if (!ok && j >= nc) break;
            if (!ok) continue;
            const int ph = j < nc ? 0 : (j < nc + ns ? 1 : 2);
            const bool first = j == 0 || j == nc || j == nc + ns;
            const int b = j & 1;
            // ---- the key mask of this tile -------------------------------------------------------
            uint64_t vm = ~0ull;
            if (ph == 0) {
                // compressed tokens: the sequence's blocks [bl, bl + nblk); column 0 is block bbase
                const int32_t bbase = 8 * cg0 + kKT * j;
                vm = span_bits(bl - bbase, bl + nblk - bbase);
            } else if (ph == 1) {
                // this row's ranges in ascending order; the current one is kept in registers
                const int base = kKT * (j - nc);
                vm = 0ull;
                while (rcur.x < base + kKT) {
                    vm |= span_bits(rcur.x - base, rcur.y - base);
                    if (rcur.y > base + kKT) break;
                    ++ri;
                    rcur = ri < nr ? rng[ri * 128 + row] : make_int2(0x7fffffff, 0x7fffffff);
                }
            } else {
                // the plan's window mask words, loaded one tile ahead
                const int w = j - nc - ns;
                vm = wnext;
                if (w + 1 < nw) wnext = wrow[(int64_t)(w + 1) * 128];
            }
            // ---- S from TMEM buffer b ------------------------------------------------------------
            ok = wait_or_flag(&bar[SFULL + b], (uint32_t)(j >> 1) & 1u, P.status, abort_flag);
            // Observe P V of tile j-2 (already complete: S of tile j was issued after it). Keeping
            // the observed count within one phase of the barriers keeps later parity waits exact.
            if (ok && j >= 2) ok = wait_pv(j - 2);
            if (!(ok = __all_sync(0xffffffffu, ok))) continue;
            tc::fence_after_sync();
            const uint32_t s_tm = tmem + lane_base + b * kKT;
            float s[64];
            tc::tmem_ld64(s_tm, s);
            if (__any_sync(0xffffffffu, vm != ~0ull)) apply_bits(s, vm);
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                mx[i] = tc::fmax3(s[i], s[i + 8], s[i + 16]);
                mx[i] = tc::fmax3(mx[i], s[i + 24], s[i + 32]);
                mx[i] = tc::fmax3(mx[i], s[i + 40], s[i + 48]);
                mx[i] = fmaxf(mx[i], s[i + 56]);
            }
            const float tmax = tc::fmax3(tc::fmax3(mx[0], mx[1], mx[2]), tc::fmax3(mx[3], mx[4], mx[5]),
                                         fmaxf(mx[6], mx[7]));
            // ---- running max, lazy rescale, P = 2^(s*sl - m) ------------------------------------
            const float tm = tmax * sl;
            bool resc = false;
            float alpha = 1.0f;
            if (tm > m + 8.0f) {
                const bool had = m != -INFINITY;
                alpha = had ? tc::ex2(m - tm) : 0.0f;
                resc = had && !first;
                l *= alpha;
                m = tm;
            }
            if (__any_sync(0xffffffffu, resc)) {
                // O must hold P V of the previous tile before it is rescaled
                if (!(ok = __all_sync(0xffffffffu, wait_pv(j - 1)))) continue;
                tc::fence_after_sync();
                const float f = resc ? alpha : 1.0f;
#pragma unroll 1
                for (int d0 = 0; d0 < D; d0 += 32) {
                    float o[32];
                    tc::tmem_ld32(o_tm + d0, o);
                    uint32_t ob32[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) ob32[e] = __float_as_uint(o[e] * f);
                    tc::tmem_st32(o_tm + d0, ob32);
                }
            }
            const float mu = m == -INFINITY ? 0.0f : m;
            uint32_t pk[32];
            float ls[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                s[2 * i] = tc::ex2(fmaf(s[2 * i], sl, -mu));
                s[2 * i + 1] = tc::ex2(fmaf(s[2 * i + 1], sl, -mu));
                pk[i] = pack2<T>(s[2 * i], s[2 * i + 1]);
                ls[i & 3] += s[2 * i] + s[2 * i + 1];
            }
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            tc::tmem_st32(s_tm, pk);
            if (kBf16) {
                // bf16 keeps 8 significant bits: the weights go to the tensor cores as P_hi + P_lo
                // (both bf16, the low part in the upper 32 columns), so P V carries ~16 bits of P
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    pk[i] = pack2<T>(s[2 * i] - unpack_lo<T>(pk[i]), s[2 * i + 1] - unpack_hi<T>(pk[i]));
                tc::tmem_st32(s_tm + 32, pk);
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bar[PFULL + b]);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- selection export -------------------------------------------------------------------------
__global__ void k_export_sel(const int32_t* __restrict__ sel, const int32_t* __restrict__ tok_pos,
                             int64_t N, int H, int k, int32_t* __restrict__ out) {
    int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_tok = (int64_t)H * k;
    if (e >= N * per_tok) return;
    const int64_t tok = e / per_tok, rest = e % per_tok;
    out[e] = sel[(int64_t)tok_pos[tok] * per_tok + rest];
}

// ---- host: launch -------------------------------------------------------------------------------
template <typename T, int D, int KM>
ssa_status_t run(const Plan* p, const FwdParams& P, int64_t max_seq_blocks, cudaStream_t st) {
    using L = FL<D, KM>;
    static_assert(L::kAlloc <= 227u * 1024u, "shared-memory layout exceeds the per-CTA limit");
    if (max_seq_blocks > L::kMaxSeqBlocks) return SSA_ERR_UNSUPPORTED;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(k_ssa_fwd<T, D, KM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)L::kAlloc) != cudaSuccess)
            return SSA_ERR_CUDA;
        configured = true;
    }
    k_ssa_fwd<T, D, KM><<<dim3((unsigned)p->n_qtiles, (unsigned)P.H), kThreads, L::kAlloc, st>>>(P);
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

template <typename T, int D>
ssa_status_t run_km(const Plan* p, const FwdParams& P, int64_t mb, cudaStream_t st) {
    // KM: the other selected blocks per row, k - 1 rounded up to 7, 15 or 31 (k <= 32)
    if (P.k <= 8) return run<T, D, 7>(p, P, mb, st);
    if (P.k <= 16) return run<T, D, 15>(p, P, mb, st);
    return run<T, D, 31>(p, P, mb, st);
}

template <typename T>
ssa_status_t run_d(const Plan* p, const FwdParams& P, int D, int64_t mb, cudaStream_t st) {
    switch (D) {
    case 32: return run_km<T, 32>(p, P, mb, st);
    case 64: return run_km<T, 64>(p, P, mb, st);
    case 96: return run_km<T, 96>(p, P, mb, st);
    default: return run_km<T, 128>(p, P, mb, st);
    }
}

}  // namespace

ssa_status_t launch_forward_tc(const Plan* p, const Workspace& w, const void* q, const float* gates,
                               void* out, const BranchOut& bo, const Prologue& pro, cudaStream_t st) {
    const bool bf16 = w.dtype == SSA_BF16;
    int64_t max_seq_blocks = 0;
    for (size_t s = 0; s + 1 < p->seq_blk.size(); ++s)
        max_seq_blocks = std::max<int64_t>(max_seq_blocks, p->seq_blk[s + 1] - p->seq_blk[s]);
    FwdParams P;
    P.q = q;
    P.ks = w.ks;
    P.vs = w.vs;
    P.kcg = w.kcg;
    P.vcg = w.vcg;
    P.gates = gates;
    P.perm = p->perm;
    P.tok_blk = p->tok_blk;
    P.blk_off = p->blk_off;
    P.blk_poff = p->blk_poff;
    P.blk_info = p->blk_info;
    P.blk_tpool = p->blk_tpool;
    P.seq_pool = p->seq_pool;
    P.scoord = p->scoord;
    P.qt_pos = p->qt_pos;
    P.qt_len = p->qt_len;
    P.qt_seq = p->qt_seq;
    P.seq_blk = p->seq_blk_d;
    P.wr_off = p->wr_off;
    P.wr_runs = p->wr_runs;
    P.wg_cnt = p->wg_cnt;
    P.wm_off = p->wm_off;
    P.wmask = p->wmask;
    P.sel = w.sel;
    P.base = w.base;
    P.out = out;
    for (int b = 0; b < 3; ++b) P.bout[b] = bo.o[b];
    P.q_gamma = pro.on() ? pro.q_gamma : nullptr;
    P.coords = p->coords;
    P.theta = pro.theta;
    P.eps = pro.eps;
    P.status = p->d_status;
    P.N = p->N;
    P.Nks = p->Nks;
    P.Mb = p->Mb;
    P.Mb8 = w.Mb8;
    P.H = w.H;
    P.k = w.k;
    P.r = p->r;
    P.sl = (float)(1.4426950408889634 / sqrt((double)w.D));
    ProfScope ps("k_ssa_fwd", st);
    if (bf16) return run_d<__nv_bfloat16>(p, P, w.D, max_seq_blocks, st);
    return run_d<__half>(p, P, w.D, max_seq_blocks, st);
}

void launch_export_sel(const Plan* p, const Workspace& w, int32_t* sel_out, cudaStream_t st) {
    const int64_t n = p->N * w.H * w.k;
    k_export_sel<<<(unsigned)cdiv(n, 256), 256, 0, st>>>(w.sel, p->tok_pos, p->N, w.H, w.k, sel_out);
    note_launch();
}

}  // namespace ssa
