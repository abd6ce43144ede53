// Block selection for the bf16 / fp16 path: for every (token, head), the own block plus the top
// (k-1) other blocks of its sequence by compressed logit (Direct3D-S2 summary page, "Technical
// principles", SSA item: the important blocks are chosen from the compression module's attention
// scores). It runs before the fused attention kernel, which reads the selection back. On request
// it also predicts the gates from the query tile it holds (same item: the branches are
// aggregated with predicted gating scores).
//
// One CTA per (query tile of 128 tokens in block order, head), 192 threads:
//   warp 0     producer: the sequence's compressed keys, 64 per tile, into a two-stage ring by 1D
//              bulk copies (the grouped operand order the fused kernel streams them in);
//   warp 1     MMA issuer (one thread): S = Q Kc^T into one of two TMEM buffers;
//   warps 2-5  one thread per query row (its TMEM lane), keeping a running top-(k-1) list.
// Only the scores are needed (no softmax, no P V, no output accumulator), so a CTA holds far less
// state than the fused kernel and three run per SM. A score enters the candidate loop only if it
// can beat the list's last entry; on the first tile, which starts from an empty list, only if it
// is at least the smallest of the tile's 16 group-of-4 maxima (at least 15 other blocks score
// that much, so nothing below it can be in the top k-1).
//
// Ranking keys: the logit's order-preserving bits with the low kbits replaced by (klo - local
// block index), so keys order by logit and equal logits by lower block index. Masked columns and
// the own block get key 0 and never enter. Logits closer than 2^(kbits-23) of their size order by
// block index instead (a near tie of the method). Every wait is bounded; a wait that runs out
// records DEV_TIMEOUT and the CTA winds down.
#include "attn_common.cuh"

namespace ssa {

namespace {

using namespace attn;

constexpr int kKT = 64;          // keys per tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 128;   // two S buffers

template <int D>
struct SL {
    static constexpr uint32_t kCh = D / 32;
    static constexpr uint32_t kQReg = 128 * 64;
    static constexpr uint32_t kGB = kCh * 512;        // one 8-row group (grouped order)
    static constexpr uint32_t kTile = 8 * kGB;        // 64 compressed keys
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kCh * kQReg;
    static constexpr uint32_t kStage = kK + 2 * kTile;  // float4 [8][128]: half a tile's scores
    static constexpr uint32_t kPro = kStage + 8 * 128 * 16;    // rotary table and weights
    static constexpr uint32_t kBar = kPro + 64 * 12 + 128 * 4;
    static constexpr uint32_t kMisc = kBar + 16 * 8;
    static constexpr uint32_t kBytes = kMisc + 64;
    static constexpr uint32_t kAlloc = kBytes + 1024;
};

enum : int { KFULL = 0, KEMPTY = 2, SFULL = 4, SFREE = 6, FIN = 8, NBAR = 9 };   // SFREE: 4 warps
enum : int { M_TMEM = 0, M_ABORT = 1 };

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, int32_t* status,
                                             volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (tc::mbar_wait(bar, parity, kWaitCycles)) return true;
    atomicOr(status, DEV_TIMEOUT);
    *abort_flag = 1;
    return false;
}

template <typename T, int D, int KM>
__global__ void __launch_bounds__(kThreads, 3) k_ssa_select(const __grid_constant__ FwdParams P) {
    using L = SL<D>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* g = align1024(smem_raw);
    const uint32_t sb = tc::smem_u32(g);
    uint64_t* bar = reinterpret_cast<uint64_t*>(g + L::kBar);
    int* misc = reinterpret_cast<int*>(g + L::kMisc);
    volatile int* abort_flag = misc + M_ABORT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x, h = blockIdx.y, H = P.H;

    const int32_t p0 = P.qt_pos[tile], len = P.qt_len[tile], seq = P.qt_seq[tile];
    const int32_t bl = P.seq_blk[seq], nblk = P.seq_blk[seq + 1] - bl;
    const int32_t cg0 = bl >> 3, ng = ((bl + nblk + 7) >> 3) - cg0;   // groups of the compressed keys
    const int nc = P.k > 1 ? (ng + 7) >> 3 : 0;   // k = 1: the own block alone, nothing to rank

    // ---- setup: TMEM, barriers, Q tile, zeroed K stages, prologue table ------------------------
    if (warp == 1) {
        tc::tmem_alloc(reinterpret_cast<uint32_t*>(misc + M_TMEM), kTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) tc::mbar_init(&bar[i], (i == SFREE || i == SFREE + 1) ? 4u : 1u);
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
    // key groups a tile does not fill keep zeros (finite scores, masked by their column)
    for (uint32_t o = tid * 16u; o < 2u * L::kTile; o += kThreads * 16u)
        *reinterpret_cast<uint4*>(g + L::kK + o) = make_uint4(0u, 0u, 0u, 0u);
    double* pro_freq = reinterpret_cast<double*>(g + L::kPro);
    int* pro_axis = reinterpret_cast<int*>(g + L::kPro + 64 * 8);
    float* pro_gamma = reinterpret_cast<float*>(g + L::kPro + 64 * 12);
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
        if (tid >= 64 && tid - 64 < len)
            qtile_prologue<T, D>(g + L::kQ, L::kQReg, tid - 64, P.perm[p0 + tid - 64], P.coords, pro_freq,
                                 pro_axis, pro_gamma, P.eps);
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    }

    if (warp == 0) {
        // ================================ producer ============================================
        const uint8_t* kch = static_cast<const uint8_t*>(P.kcg) + (int64_t)h * P.Mb8 * D * 2;
        int last = -1;   // last tile issued (the one before it went into the other stage)
        for (int j = 0; j < nc; ++j) {
            const int s = j & 1;
            if (j >= 2 && !wait_or_flag(&bar[KEMPTY + s], (uint32_t)((j >> 1) - 1) & 1u, P.status, abort_flag))
                break;
            const uint32_t n = (uint32_t)min(8, ng - 8 * j);
            if (lane == 0) {
                tc::mbar_arrive_expect_tx(&bar[KFULL + s], n * L::kGB);
                tc::bulk_load(sb + L::kK + s * L::kTile, kch + (int64_t)(cg0 + 8 * j) * L::kGB, n * L::kGB,
                              &bar[KFULL + s]);
            }
            last = j;
        }
        // the copies must have landed before the CTA can end (bounded; normally already done)
        if (lane == 0)
            for (int j = max(last - 1, 0); j <= last; ++j)
                tc::mbar_wait(&bar[KFULL + (j & 1)], (uint32_t)(j >> 1) & 1u, kWaitCycles);
        __syncwarp();
    } else if (warp == 1) {
        // ================================ MMA issuer ==========================================
        if (lane == 0) {
            const uint32_t idesc_s = tc::idesc_f16(kBf16, 128, kKT, false);
            for (int j = 0; j < nc; ++j) {
                const int b = j & 1;
                if (!wait_or_flag(&bar[KFULL + b], (uint32_t)(j >> 1) & 1u, P.status, abort_flag)) break;
                // TMEM buffer b holds S of tile j-2 until both ranking threads of every row read it
                if (j >= 2 && !wait_or_flag(&bar[SFREE + b], (uint32_t)((j >> 1) - 1) & 1u, P.status, abort_flag))
                    break;
                tc::fence_after_sync();
                const uint32_t kbase = sb + L::kK + b * L::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::mma_f16_ss(tmem + b * kKT, tc::desc_kmajor_r(sb + L::kQ, kk, L::kQReg),
                                   tc::desc_kmajor_g(kbase, kk, L::kCh), idesc_s, kk > 0 ? 1u : 0u);
                tc::mma_commit(&bar[SFULL + b]);
                tc::mma_commit(&bar[KEMPTY + b]);
            }
            // drain the tensor pipe before TMEM is released
            tc::mma_commit(&bar[FIN]);
            tc::mbar_wait(&bar[FIN], 0u, kWaitCycles);
        }
        __syncwarp();
    } else {
        // ================================ ranking =============================================
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const bool row_ok = row < len;
        const int32_t pos = p0 + (row_ok ? row : len - 1);
        const int32_t tok = P.perm[pos];
        const int32_t ob_loc = P.tok_blk[tok] - bl;
        const int ksel = P.k;
        const uint32_t kbits = 32u - __clz((unsigned)max(nblk - 1, 1));
        const uint32_t klo = (1u << kbits) - 1u;
        uint32_t tk[KM];
#pragma unroll
        for (int u = 0; u < KM; ++u) tk[u] = 0u;
        auto push = [&](uint32_t key) {
#pragma unroll
            for (int q = KM - 1; q > 0; --q) tk[q] = max(tk[q], min(tk[q - 1], key));
            tk[0] = max(tk[0], key);
        };
        if (P.gate_w && row_ok) {
            // gates predicted from this row's query (as the attention sees it, after the prologue):
            // sigmoid(q . gate_w + gate_b), one per branch
            float t0 = P.gate_b[0], t1 = P.gate_b[1], t2 = P.gate_b[2];
#pragma unroll 1
            for (int c16 = 0; c16 < D / 8; ++c16) {
                const uint4 u = *reinterpret_cast<const uint4*>(g + L::kQ + (c16 >> 2) * L::kQReg +
                                                                 tc::sw64(row, c16 & 3));
                const uint32_t* wv = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int d = c16 * 8 + 2 * q;
                    const float a = unpack_lo<T>(wv[q]), bq = unpack_hi<T>(wv[q]);
                    const float* w0 = P.gate_w + d * 3;
                    t0 = fmaf(a, w0[0], fmaf(bq, w0[3], t0));
                    t1 = fmaf(a, w0[1], fmaf(bq, w0[4], t1));
                    t2 = fmaf(a, w0[2], fmaf(bq, w0[5], t2));
                }
            }
            float* go = P.gates_out + ((int64_t)tok * H + h) * 3;
            go[0] = 1.0f / (1.0f + __expf(-t0));
            go[1] = 1.0f / (1.0f + __expf(-t1));
            go[2] = 1.0f / (1.0f + __expf(-t2));
        }
        float4* stage4 = reinterpret_cast<float4*>(g + L::kStage) + row;
        const float* stage1 = reinterpret_cast<const float*>(stage4);
        bool ok = true;
        for (int j = 0; j < nc && ok; ++j) {
            const int b = j & 1;
            ok = __all_sync(0xffffffffu, wait_or_flag(&bar[SFULL + b], (uint32_t)(j >> 1) & 1u, P.status,
                                                      abort_flag));
            if (!ok) break;
            tc::fence_after_sync();
            float s[64];
            tc::tmem_ld64(tmem + lane_base + b * kKT, s);
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bar[SFREE + b]);   // this warp is done with S of tile j
            // columns outside the sequence's blocks (first and last tiles) never compete
            const int32_t cbase = 8 * cg0 + kKT * j - bl;   // local block index of column 0
            if (cbase < 0 || cbase + kKT > nblk) {
#pragma unroll
                for (int e = 0; e < 64; ++e) s[e] = (cbase + e >= 0 && cbase + e < nblk) ? s[e] : -INFINITY;
            }
            // maxima of the 16 groups of 4 consecutive columns: their smallest and their largest
            float glo = INFINITY, tmax = -INFINITY;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float gq = fmaxf(tc::fmax3(s[4 * q], s[4 * q + 1], s[4 * q + 2]), s[4 * q + 3]);
                glo = fminf(glo, gq);
                tmax = fmaxf(tmax, gq);
            }
            float thr_f;
            if (tk[KM - 1] == 0u) {
                // the list is not full. On the first tile a score below the smallest group maximum
                // trails at least 15 other blocks of this tile (16 groups, at most one of them the
                // own block), so it cannot be among the top k-1 for k-1 <= 15. Otherwise every
                // score is a candidate.
                thr_f = (j == 0 && ksel - 1 <= 15) ? glo : -INFINITY;
            } else {
                // only scores at or above the float whose key prefix is the list's last entry
                const uint32_t th = tk[KM - 1] & ~klo;
                thr_f = __uint_as_float((th & 0x80000000u) ? (th & 0x7fffffffu) : ~th);
            }
            if (tmax >= thr_f) {
                // half a tile at a time through shared memory (quad q of row r at float4 q*128 + r)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t cand = 0u;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int c = 32 * hf + 4 * q;
                        stage4[q * 128] = make_float4(s[c], s[c + 1], s[c + 2], s[c + 3]);
#pragma unroll
                        for (int i = 0; i < 4; ++i) cand |= (uint32_t)(s[c + i] >= thr_f) << (4 * q + i);
                    }
                    // candidates in column order; the next score is loaded before this one is pushed
                    int e = cand ? __ffs(cand) - 1 : 0;
                    float z = stage1[(e >> 2) * 512 + (e & 3)];
                    while (cand) {
                        cand &= cand - 1;
                        const int e2 = cand ? __ffs(cand) - 1 : e;
                        const float z2 = stage1[(e2 >> 2) * 512 + (e2 & 3)];
                        const int32_t blk = cbase + 32 * hf + e;
                        const uint32_t u = __float_as_uint(z);
                        const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
                        const uint32_t key = (blk >= 0 && blk < nblk && blk != ob_loc && z != -INFINITY)
                                                 ? ((o & ~klo) | (klo - (uint32_t)blk))
                                                 : 0u;
                        if (key > tk[KM - 1]) push(key);
                        e = e2;
                        z = z2;
                    }
                }
            }
        }
        if (row_ok && !*abort_flag) {
            int32_t* srow = P.sel + ((int64_t)pos * H + h) * ksel;
            srow[0] = bl + ob_loc;
#pragma unroll
            for (int u = 0; u < KM; ++u)
                if (u + 1 < ksel) srow[u + 1] = tk[u] ? bl + (int32_t)(klo - (tk[u] & klo)) : -1;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- selection shared by the queries of a 4x4x4 sub-block --------------------------------------
// One CTA per (selection tile, head), 192 threads in the roles of k_ssa_select. A tile holds whole
// sub-blocks of one sequence (at most 128 rows and 32 sub-blocks), its rows grouped by sub-block.
// The compressed keys stream twice. Pass 1 gives each row the base-2 log-sum-exp of its scaled
// compressed logits; pass 2 its weights p = 2^(z sl - lse2), staged in shared memory and summed
// per (sub-block, column) in a fixed order over the sub-block's rows. The thread that forms a sum
// also tests it against its sub-block's current entry threshold and marks the column; the thread
// that owns the sub-block's list then inserts the marked columns only. Lists hold 64-bit keys: the
// fp32 sum's bits, then the block index complemented, so equal sums go to the lower block index
// and the ranking of the fp32 sums is exact.
constexpr int kMaxSub = 32;   // sub-blocks per selection tile

template <int D>
struct SLS {
    static constexpr uint32_t kCh = D / 32;
    static constexpr uint32_t kQReg = 128 * 64;
    static constexpr uint32_t kGB = kCh * 512;
    static constexpr uint32_t kTile = 8 * kGB;
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kCh * kQReg;
    static constexpr uint32_t kPS = 68;                          // floats per staged row (padded)
    static constexpr uint32_t kStage = kK + 2 * kTile;           // float [128][kPS]; after the loop
                                                                 // int32 [kMaxSub][32]: the lists
    static constexpr uint32_t kSum = kStage + 128 * kPS * 4;     // float [kMaxSub][64]
    static constexpr uint32_t kThr = kSum + kMaxSub * 64 * 4;    // uint64 [kMaxSub]: entry keys
    static constexpr uint32_t kCand = kThr + kMaxSub * 8;        // uint32 [kMaxSub][2]: marked columns
    static constexpr uint32_t kSeg = kCand + kMaxSub * 8;        // int32 [3][kMaxSub] first, rows, own; count
    static constexpr uint32_t kRowKey = kSeg + (3 * kMaxSub + 4) * 4;   // int32 [128]
    static constexpr uint32_t kPro = kRowKey + 128 * 4;          // rotary table and weights
    static constexpr uint32_t kBar = kPro + 64 * 12 + 128 * 4;
    static constexpr uint32_t kMisc = kBar + 16 * 8;
    static constexpr uint32_t kBytes = kMisc + 64;
    static constexpr uint32_t kAlloc = kBytes + 1024;
};

// Named barrier that also returns the AND of `v` over the `count` threads (whole warps).
__device__ __forceinline__ bool named_sync_and(uint32_t id, uint32_t count, bool v) {
    __syncwarp();
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(count)
        : "memory");
    return r != 0u;
}

// selection tiles, their rows in sub-block order
struct SubParams {
    FwdParams f;
    const int4* sst;
    const int32_t* sb_rows;
};

template <typename T, int D, int KM>
__global__ void __launch_bounds__(kThreads, 2) k_ssa_select_sub(const __grid_constant__ SubParams S) {
    using L = SLS<D>;
    const FwdParams& P = S.f;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* g = align1024(smem_raw);
    const uint32_t sb = tc::smem_u32(g);
    uint64_t* bar = reinterpret_cast<uint64_t*>(g + L::kBar);
    int* misc = reinterpret_cast<int*>(g + L::kMisc);
    volatile int* abort_flag = misc + M_ABORT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, H = P.H;

    const int4 tl = S.sst[blockIdx.x];   // (first index into sb_rows, rows, sequence, sub-blocks)
    const int32_t r0 = tl.x, len = tl.y, seq = tl.z;
    const int32_t bl = P.seq_blk[seq], nblk = P.seq_blk[seq + 1] - bl;
    const int32_t cg0 = bl >> 3, ng = ((bl + nblk + 7) >> 3) - cg0;
    const int nc = P.k > 1 ? (ng + 7) >> 3 : 0;   // k = 1: the own block alone, nothing to rank

    // ---- setup: TMEM, barriers, Q tile, zeroed K stages, prologue table, sub-blocks ------------
    if (warp == 1) {
        tc::tmem_alloc(reinterpret_cast<uint32_t*>(misc + M_TMEM), kTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) tc::mbar_init(&bar[i], (i == SFREE || i == SFREE + 1) ? 4u : 1u);
        misc[M_ABORT] = 0;
        tc::fence_mbar_init();
    }
    const T* Q = reinterpret_cast<const T*>(P.q);
    for (int e = tid; e < 128 * (D / 8); e += kThreads) {
        const int row = e / (D / 8), c16 = e % (D / 8);
        const bool ok = row < len;
        const T* src = ok ? Q + ((int64_t)P.perm[S.sb_rows[r0 + row]] * H + h) * D + c16 * 8 : Q;
        tc::cp_async16(sb + L::kQ + (c16 >> 2) * L::kQReg + tc::sw64(row, c16 & 3), src, ok ? 16u : 0u);
    }
    for (uint32_t o = tid * 16u; o < 2u * L::kTile; o += kThreads * 16u)
        *reinterpret_cast<uint4*>(g + L::kK + o) = make_uint4(0u, 0u, 0u, 0u);
    double* pro_freq = reinterpret_cast<double*>(g + L::kPro);
    int* pro_axis = reinterpret_cast<int*>(g + L::kPro + 64 * 8);
    float* pro_gamma = reinterpret_cast<float*>(g + L::kPro + 64 * 12);
    if (P.q_gamma) {
        if (tid < D / 2) rope_pair(D, tid, P.theta, pro_axis[tid], pro_freq[tid]);
        if (tid < D) pro_gamma[tid] = P.q_gamma[tid];
    }
    // (block, sub-block) key of every row; rows come grouped by it
    int* row_key = reinterpret_cast<int*>(g + L::kRowKey);
    int* seg = reinterpret_cast<int*>(g + L::kSeg);   // first row | rows | own block (global) | count
    uint64_t* thr = reinterpret_cast<uint64_t*>(g + L::kThr);
    uint32_t* cand = reinterpret_cast<uint32_t*>(g + L::kCand);
    if (tid < 128) {
        int key = -1;
        if (tid < len) {
            const int32_t tok = P.perm[S.sb_rows[r0 + tid]];
            const int32_t* c = P.coords + 3 * (int64_t)tok;
            key = 8 * P.tok_blk[tok] + ((((c[0] >> 2) & 1) << 2) | (((c[1] >> 2) & 1) << 1) | ((c[2] >> 2) & 1));
        }
        row_key[tid] = key;
    }
    if (tid < kMaxSub) {
        thr[tid] = 0ull;
        cand[2 * tid] = 0u;
        cand[2 * tid + 1] = 0u;
    }
    tc::cp_async_wait_all();
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = (uint32_t)misc[M_TMEM];
    if (tid == 0) {
        int n = 0;
        for (int r = 0; r < len && n <= kMaxSub; ++r) {
            if (r == 0 || row_key[r] != row_key[r - 1]) {
                if (n == kMaxSub) {   // more sub-blocks than the plan packs: give up on the tile
                    n = kMaxSub + 1;
                    break;
                }
                seg[n] = r;
                seg[kMaxSub + n] = 0;
                seg[2 * kMaxSub + n] = row_key[r] >> 3;
                ++n;
            }
            seg[kMaxSub + n - 1] += 1;
        }
        if (n > kMaxSub) {
            atomicOr(P.status, DEV_BAD_INDEX);
            n = 0;
        }
        seg[3 * kMaxSub] = n;
    }
    if (P.q_gamma && tid >= 64 && tid - 64 < len)
        qtile_prologue<T, D>(g + L::kQ, L::kQReg, tid - 64, P.perm[S.sb_rows[r0 + tid - 64]], P.coords, pro_freq,
                             pro_axis, pro_gamma, P.eps);
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const int nseg = seg[3 * kMaxSub];

    if (warp == 0) {
        // ================================ producer: the compressed keys, twice ================
        const uint8_t* kch = static_cast<const uint8_t*>(P.kcg) + (int64_t)h * P.Mb8 * D * 2;
        int last = -1;
        for (int j = 0; j < 2 * nc && nseg > 0; ++j) {
            const int s = j & 1, jt = j < nc ? j : j - nc;
            if (j >= 2 && !wait_or_flag(&bar[KEMPTY + s], (uint32_t)((j >> 1) - 1) & 1u, P.status, abort_flag))
                break;
            const uint32_t n = (uint32_t)min(8, ng - 8 * jt);
            if (lane == 0) {
                tc::mbar_arrive_expect_tx(&bar[KFULL + s], n * L::kGB);
                tc::bulk_load(sb + L::kK + s * L::kTile, kch + (int64_t)(cg0 + 8 * jt) * L::kGB, n * L::kGB,
                              &bar[KFULL + s]);
            }
            last = j;
        }
        if (lane == 0)
            for (int j = max(last - 1, 0); j <= last; ++j)
                tc::mbar_wait(&bar[KFULL + (j & 1)], (uint32_t)(j >> 1) & 1u, kWaitCycles);
        __syncwarp();
    } else if (warp == 1) {
        // ================================ MMA issuer ==========================================
        if (lane == 0) {
            const uint32_t idesc_s = tc::idesc_f16(kBf16, 128, kKT, false);
            for (int j = 0; j < 2 * nc && nseg > 0; ++j) {
                const int b = j & 1;
                if (!wait_or_flag(&bar[KFULL + b], (uint32_t)(j >> 1) & 1u, P.status, abort_flag)) break;
                if (j >= 2 && !wait_or_flag(&bar[SFREE + b], (uint32_t)((j >> 1) - 1) & 1u, P.status, abort_flag))
                    break;
                tc::fence_after_sync();
                const uint32_t kbase = sb + L::kK + b * L::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::mma_f16_ss(tmem + b * kKT, tc::desc_kmajor_r(sb + L::kQ, kk, L::kQReg),
                                   tc::desc_kmajor_g(kbase, kk, L::kCh), idesc_s, kk > 0 ? 1u : 0u);
                tc::mma_commit(&bar[SFULL + b]);
                tc::mma_commit(&bar[KEMPTY + b]);
            }
            tc::mma_commit(&bar[FIN]);
            tc::mbar_wait(&bar[FIN], 0u, kWaitCycles);
        }
        __syncwarp();
    } else {
        // ================================ rows: softmax statistics, weights, sums ==============
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int t128 = tid - 64;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const bool row_ok = row < len;
        const int32_t pos = row_ok ? S.sb_rows[r0 + row] : 0;
        const int32_t tok = P.perm[pos];
        const int ksel = P.k;
        const float sl = P.sl;
        if (P.gate_w && row_ok) {
            float t0 = P.gate_b[0], t1 = P.gate_b[1], t2 = P.gate_b[2];
#pragma unroll 1
            for (int c16 = 0; c16 < D / 8; ++c16) {
                const uint4 u = *reinterpret_cast<const uint4*>(g + L::kQ + (c16 >> 2) * L::kQReg +
                                                                 tc::sw64(row, c16 & 3));
                const uint32_t* wv = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int d = c16 * 8 + 2 * q;
                    const float a = unpack_lo<T>(wv[q]), bq = unpack_hi<T>(wv[q]);
                    const float* w0 = P.gate_w + d * 3;
                    t0 = fmaf(a, w0[0], fmaf(bq, w0[3], t0));
                    t1 = fmaf(a, w0[1], fmaf(bq, w0[4], t1));
                    t2 = fmaf(a, w0[2], fmaf(bq, w0[5], t2));
                }
            }
            float* go = P.gates_out + ((int64_t)tok * H + h) * 3;
            go[0] = 1.0f / (1.0f + __expf(-t0));
            go[1] = 1.0f / (1.0f + __expf(-t1));
            go[2] = 1.0f / (1.0f + __expf(-t2));
        }
        float* stage = reinterpret_cast<float*>(g + L::kStage);
        float* sums = reinterpret_cast<float*>(g + L::kSum);
        uint64_t tk[KM];   // the list of sub-block t128 (t128 < nseg), best first; 0 = empty
#pragma unroll
        for (int u = 0; u < KM; ++u) tk[u] = 0ull;
        float m = -INFINITY, l = 0.0f, lse = 0.0f;
        bool ok = nseg > 0, p1_ok = true;
        for (int j = 0; j < 2 * nc && ok; ++j) {
            const int b = j & 1, jt = j < nc ? j : j - nc;
            if (j < nc) {
                // pass 1 has no named barrier: a warp whose wait ran out skips its tiles, and the
                // four row warps decide together at the end of the pass
                const bool wok = p1_ok && __all_sync(0xffffffffu, wait_or_flag(&bar[SFULL + b], (uint32_t)(j >> 1) & 1u,
                                                                            P.status, abort_flag));
                p1_ok = wok;
                if (!wok) {
                    if (j == nc - 1 && !(ok = named_sync_and(1, 128, false))) break;
                    continue;
                }
            } else {
                // one decision for all four row warps, so that they meet the same named barriers
                ok = named_sync_and(1, 128, wait_or_flag(&bar[SFULL + b], (uint32_t)(j >> 1) & 1u, P.status,
                                                         abort_flag));
                if (!ok) break;
            }
            tc::fence_after_sync();
            float s[64];
            tc::tmem_ld64(tmem + lane_base + b * kKT, s);
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bar[SFREE + b]);
            const int32_t cbase = 8 * cg0 + kKT * jt - bl;   // local block index of column 0
            if (cbase < 0 || cbase + kKT > nblk) {
#pragma unroll
                for (int e = 0; e < 64; ++e) s[e] = (cbase + e >= 0 && cbase + e < nblk) ? s[e] : -INFINITY;
            }
            if (j < nc) {
                // pass 1: running maximum and sum of 2^(z sl)
                float tmax = -INFINITY;
#pragma unroll
                for (int e = 0; e < 64; e += 4) tmax = fmaxf(tmax, tc::fmax3(s[e], s[e + 1], fmaxf(s[e + 2], s[e + 3])));
                const float tm = tmax * sl;
                if (tm > m) {
                    l *= tc::ex2(m - tm);
                    m = tm;
                }
                float ls[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int e = 0; e < 64; ++e) ls[e & 3] += tc::ex2(fmaf(s[e], sl, -m));
                l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
                if (j == nc - 1) {
                    lse = m + __log2f(l);
                    if (!(ok = named_sync_and(1, 128, true))) break;
                }
                continue;
            }
            // pass 2: this row's weights into the stage
            float4* srow = reinterpret_cast<float4*>(stage + row * L::kPS);
#pragma unroll
            for (int e = 0; e < 64; e += 4)
                srow[e >> 2] = make_float4(tc::ex2(fmaf(s[e], sl, -lse)), tc::ex2(fmaf(s[e + 1], sl, -lse)),
                                           tc::ex2(fmaf(s[e + 2], sl, -lse)), tc::ex2(fmaf(s[e + 3], sl, -lse)));
            tc::named_sync(1, 128);
            // sum of column c over the rows of sub-blocks q = t128 / 64, + 2, ... (four partial sums
            // in a fixed pattern), and a mark where it can enter the sub-block's list
            {
                const int c = t128 & 63;
                const int32_t blk = cbase + c;
                const bool col_ok = blk >= 0 && blk < nblk;
                for (int q = t128 >> 6; q < nseg; q += 2) {
                    const int a = seg[q], n = seg[kMaxSub + q];
                    const float* sc = stage + a * L::kPS + c;
                    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
                    int r = 0;
                    for (; r + 4 <= n; r += 4) {
                        a0 += sc[r * L::kPS];
                        a1 += sc[(r + 1) * L::kPS];
                        a2 += sc[(r + 2) * L::kPS];
                        a3 += sc[(r + 3) * L::kPS];
                    }
                    for (; r < n; ++r) a0 += sc[r * L::kPS];
                    const float acc = (a0 + a1) + (a2 + a3);
                    sums[q * 64 + c] = acc;
                    const uint64_t key = ((uint64_t)__float_as_uint(acc) << 32) | (uint32_t)(0x7fffffff - blk);
                    if (col_ok && blk != seg[2 * kMaxSub + q] - bl && key > thr[q])
                        atomicOr(&cand[2 * q + (c >> 5)], 1u << (c & 31));
                }
            }
            tc::named_sync(1, 128);
            if (t128 < nseg) {
                const float* sq = sums + t128 * 64;
#pragma unroll 1
                for (int hw = 0; hw < 2; ++hw) {
                    uint32_t mk = cand[2 * t128 + hw];
                    while (mk) {
                        const int e = 32 * hw + __ffs(mk) - 1;
                        mk &= mk - 1;
                        const int32_t blk = cbase + e;
                        const uint64_t key = ((uint64_t)__float_as_uint(sq[e]) << 32) | (uint32_t)(0x7fffffff - blk);
                        if (key > tk[KM - 1]) {
#pragma unroll
                            for (int q = KM - 1; q > 0; --q) tk[q] = max(tk[q], min(tk[q - 1], key));
                            tk[0] = max(tk[0], key);
                        }
                    }
                    cand[2 * t128 + hw] = 0u;
                }
                thr[t128] = tk[KM - 1];
            }
        }
        tc::named_sync(1, 128);   // the stage is free: the lists go there
        int32_t* lists = reinterpret_cast<int32_t*>(g + L::kStage);
        if (t128 < nseg) {
#pragma unroll
            for (int u = 0; u < KM; ++u)
                lists[t128 * 32 + u] = tk[u] ? bl + (0x7fffffff - (int32_t)(uint32_t)(tk[u] & 0xffffffffull)) : -1;
        }
        tc::named_sync(1, 128);
        if (row_ok && nseg > 0 && !*abort_flag) {
            int q = 0;
            while (q + 1 < nseg && row >= seg[q + 1]) ++q;
            int32_t* so = P.sel + ((int64_t)pos * H + h) * ksel;
            so[0] = seg[2 * kMaxSub + q];
#pragma unroll
            for (int u = 0; u < KM; ++u)
                if (u + 1 < ksel) so[u + 1] = nc > 0 ? lists[q * 32 + u] : -1;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

template <typename T, int D, int KM>
ssa_status_t run_sub(const Plan* p, const FwdParams& P, cudaStream_t st) {
    SubParams S;
    S.f = P;
    S.sst = p->sst;
    S.sb_rows = p->sb_rows;
    using L = SLS<D>;
    static_assert(L::kAlloc <= 113u * 1024u, "at least two CTAs per SM");
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(k_ssa_select_sub<T, D, KM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)L::kAlloc) != cudaSuccess)
            return SSA_ERR_CUDA;
        configured = true;
    }
    if (p->n_sst == 0) return SSA_OK;
    k_ssa_select_sub<T, D, KM><<<dim3((unsigned)p->n_sst, (unsigned)P.H), kThreads, L::kAlloc, st>>>(S);
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

template <typename T, int D, int KM>
ssa_status_t run(const Plan* p, const FwdParams& P, cudaStream_t st) {
    using L = SL<D>;
    static_assert(L::kAlloc <= 113u * 1024u, "at least two CTAs per SM");
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(k_ssa_select<T, D, KM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)L::kAlloc) != cudaSuccess)
            return SSA_ERR_CUDA;
        configured = true;
    }
    k_ssa_select<T, D, KM><<<dim3((unsigned)p->n_qtiles, (unsigned)P.H), kThreads, L::kAlloc, st>>>(P);
    note_launch();
    return cudaPeekAtLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

template <typename T, int D>
ssa_status_t run_km(const Plan* p, const FwdParams& P, bool shared, cudaStream_t st) {
    // KM: the list length, k - 1 rounded up to 7, 15 or 31 (k <= 32)
    if (shared) {
        if (P.k <= 8) return run_sub<T, D, 7>(p, P, st);
        if (P.k <= 16) return run_sub<T, D, 15>(p, P, st);
        return run_sub<T, D, 31>(p, P, st);
    }
    if (P.k <= 8) return run<T, D, 7>(p, P, st);
    if (P.k <= 16) return run<T, D, 15>(p, P, st);
    return run<T, D, 31>(p, P, st);
}

template <typename T>
ssa_status_t run_d(const Plan* p, const FwdParams& P, int D, bool shared, cudaStream_t st) {
    switch (D) {
    case 32: return run_km<T, 32>(p, P, shared, st);
    case 64: return run_km<T, 64>(p, P, shared, st);
    case 96: return run_km<T, 96>(p, P, shared, st);
    default: return run_km<T, 128>(p, P, shared, st);
    }
}

FwdParams select_params(const Plan* p, const Workspace& w, const void* q, const Prologue& pro,
                        const float* gate_w, const float* gate_b, float* gates_out) {
    FwdParams P = FwdParams();
    P.q = q;
    P.kcg = w.kcg;
    P.perm = p->perm;
    P.tok_blk = p->tok_blk;
    P.qt_pos = p->qt_pos;
    P.qt_len = p->qt_len;
    P.qt_seq = p->qt_seq;
    P.seq_blk = p->seq_blk_d;
    P.sel = w.sel;
    P.status = p->d_status;
    P.q_gamma = pro.on() ? pro.q_gamma : nullptr;
    P.coords = p->coords;
    P.theta = pro.theta;
    P.eps = pro.eps;
    P.gate_w = gate_w;
    P.gate_b = gate_b;
    P.gates_out = gates_out;
    P.N = p->N;
    P.Mb = p->Mb;
    P.Mb8 = w.Mb8;
    P.H = w.H;
    P.k = w.k;
    P.sl = (float)(1.4426950408889634 / sqrt((double)w.D));
    return P;
}

}  // namespace

ssa_status_t launch_select_tc(const Plan* p, const Workspace& w, const void* q, const Prologue& pro,
                              const float* gate_w, const float* gate_b, float* gates_out, cudaStream_t st) {
    const FwdParams P = select_params(p, w, q, pro, gate_w, gate_b, gates_out);
    ProfScope ps("k_ssa_select", st);
    if (w.dtype == SSA_BF16) return run_d<__nv_bfloat16>(p, P, w.D, false, st);
    return run_d<__half>(p, P, w.D, false, st);
}

ssa_status_t launch_select_shared(const Plan* p, const Workspace& w, const void* q, const Prologue& pro,
                                  const float* gate_w, const float* gate_b, float* gates_out,
                                  cudaStream_t st) {
    const FwdParams P = select_params(p, w, q, pro, gate_w, gate_b, gates_out);
    ProfScope ps("k_ssa_select_sub", st);
    if (w.dtype == SSA_BF16) return run_d<__nv_bfloat16>(p, P, w.D, true, st);
    return run_d<__half>(p, P, w.D, true, st);
}

}  // namespace ssa
