// Compression pooling: Kc_b = mean_{j in b}(K_j) . Wc and Vc_b likewise, per head, with
// one D x D map Wc shared by K, V and all heads (Direct3D-S2 summary page, "Technical
// principles", SSA item: block-level tokens from a compression of each block; the concrete
// mean-then-linear-map form is the formulation this library implements).
//
// One CTA per occupied block. Each thread owns one 16-byte column group of the token rows (all
// heads of a token are contiguous), so every token row is read with fully coalesced 128-bit loads;
// sums are fp32. For the tensor-core path the same pass also writes the rows into the padded,
// head-major, block-ordered copies K_s, V_s [H, Nks, D] that the attention tiles read, and the
// compressed tokens a second time in the same order. A block of at most kPoolMaxTokens tokens is
// written twice: at its padded rows and, packed with the other small blocks of its sequence, in
// that sequence's pool after all padded rows.
//
// Grouped order (16-bit types): rows are taken 8 at a time; a group stores its D/32 column chunks
// one after the other, each as a 512-byte atom of 8 rows x 64 bytes in which the four 16-byte
// units of row i are permuted by unit ^= (i >> 1) & 3. This is the shared-memory operand order of
// the tensor cores with 64-byte swizzle, so a run of consecutive groups is copied to shared
// memory with one bulk copy and used there as is.
#include "common.cuh"

namespace ssa {

namespace {

// byte offset of element column d of row `row` (16-byte unit granularity: d % 8 == 0) inside a
// grouped matrix with D columns
__device__ __forceinline__ int64_t grouped_off(int64_t row, int d, int D) {
    const int64_t g = row >> 3;
    const int i = (int)(row & 7), c = d >> 5, u = (d & 31) >> 3;
    return g * (int64_t)(D / 32) * 512 + c * 512 + i * 64 + ((u ^ ((i >> 1) & 3)) << 4);
}

constexpr int kMaxGroupsPerThread = 2;

template <typename T, bool kSorted>
__global__ void __launch_bounds__(1024) k_pool(const T* __restrict__ K, const T* __restrict__ V,
                                               const float* __restrict__ Wc,
                                               const int32_t* __restrict__ perm,
                                               const int32_t* __restrict__ blk_off,
                                               const int32_t* __restrict__ blk_poff,
                                               const int32_t* __restrict__ blk_tpool,
                                               const int32_t* __restrict__ blk_seq,
                                               const int2* __restrict__ seq_pool, int64_t Mb,
                                               int H, int D, int64_t Nks, T* __restrict__ ks,
                                               T* __restrict__ vs, T* __restrict__ kc,
                                               T* __restrict__ vc, int64_t Mb8,
                                               T* __restrict__ kcg, T* __restrict__ vcg) {
    constexpr int kVec = 16 / sizeof(T);
    extern __shared__ float mean[];   // [2][H*D]: K means then V means
    const int64_t b = blockIdx.x;
    const int HD = H * D;
    const int groups = HD / kVec;
    const int32_t lo = blk_off[b], n = blk_off[b + 1] - lo;
    const int32_t prow = blk_poff[b];
    // row of the block's copy in its sequence's pool, -1 if it has none
    const int32_t trow = kSorted && blk_tpool[b] >= 0 ? 8 * seq_pool[blk_seq[b]].x + blk_tpool[b] : -1;

    float sk[kMaxGroupsPerThread][kVec], sv[kMaxGroupsPerThread][kVec];
#pragma unroll
    for (int a = 0; a < kMaxGroupsPerThread; ++a)
#pragma unroll
        for (int e = 0; e < kVec; ++e) sk[a][e] = sv[a][e] = 0.0f;

    for (int t = 0; t < n; ++t) {
        const int64_t tok = perm[lo + t];
        const uint4* krow = reinterpret_cast<const uint4*>(K + tok * HD);
        const uint4* vrow = reinterpret_cast<const uint4*>(V + tok * HD);
#pragma unroll
        for (int a = 0; a < kMaxGroupsPerThread; ++a) {
            const int gidx = threadIdx.x + a * blockDim.x;
            if (gidx >= groups) break;
            const uint4 kq = krow[gidx], vq = vrow[gidx];
            const T* ke = reinterpret_cast<const T*>(&kq);
            const T* ve = reinterpret_cast<const T*>(&vq);
#pragma unroll
            for (int e = 0; e < kVec; ++e) {
                sk[a][e] += Elem<T>::to_f(ke[e]);
                sv[a][e] += Elem<T>::to_f(ve[e]);
            }
            if (kSorted) {
                const int col = gidx * kVec, h = col / D, d = col % D;
                const int64_t hoff = (int64_t)h * Nks * D * (int64_t)sizeof(T);
                const int64_t dst = hoff + grouped_off(prow + t, d, D);
                *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(ks) + dst) = kq;
                *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(vs) + dst) = vq;
                if (trow >= 0) {
                    const int64_t tdst = hoff + grouped_off(trow + t, d, D);
                    *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(ks) + tdst) = kq;
                    *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(vs) + tdst) = vq;
                }
            }
        }
    }
    const float inv = 1.0f / (float)n;
#pragma unroll
    for (int a = 0; a < kMaxGroupsPerThread; ++a) {
        const int gidx = threadIdx.x + a * blockDim.x;
        if (gidx >= groups) break;
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            mean[gidx * kVec + e] = sk[a][e] * inv;
            mean[HD + gidx * kVec + e] = sv[a][e] * inv;
        }
    }
    __syncthreads();
    // Kc[h][b][e] = sum_d mean[h][d] * Wc[d][e]
    for (int o = threadIdx.x; o < HD; o += blockDim.x) {
        const int h = o / D, e = o % D;
        const float* mk = mean + h * D;
        const float* mv = mean + HD + h * D;
        float ak = 0.0f, av = 0.0f;
        for (int d = 0; d < D; ++d) {
            const float w = __ldg(Wc + d * D + e);
            ak = fmaf(mk[d], w, ak);
            av = fmaf(mv[d], w, av);
        }
        const int64_t dst = ((int64_t)h * Mb + b) * D + e;
        kc[dst] = Elem<T>::from_f(ak);
        vc[dst] = Elem<T>::from_f(av);
        if (kSorted) {
            const int64_t gd = (int64_t)h * Mb8 * D * (int64_t)sizeof(T) + grouped_off(b, e & ~7, D) +
                               (e & 7) * (int64_t)sizeof(T);
            *reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(kcg) + gd) = Elem<T>::from_f(ak);
            *reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(vcg) + gd) = Elem<T>::from_f(av);
        }
    }
}

template <typename T>
void run_pool(const Plan* p, const Workspace& w, const void* k, const void* v, const float* wc,
              cudaStream_t st) {
    constexpr int kVec = 16 / sizeof(T);
    const int HD = w.H * w.D;
    const int groups = HD / kVec;
    int threads = (int)round_up(cdiv(groups, kMaxGroupsPerThread), 32);
    if (threads > 1024) threads = 1024;
    if (threads < 128) threads = 128;
    const size_t smem = sizeof(float) * 2 * HD;
    const bool sorted = w.ks != nullptr;
    auto kern = sorted ? k_pool<T, true> : k_pool<T, false>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<(unsigned)p->Mb, threads, smem, st>>>(
        (const T*)k, (const T*)v, wc, p->perm, p->blk_off, p->blk_poff, p->blk_tpool, p->blk_seq,
        p->seq_pool, p->Mb, w.H, w.D, p->Nks,
        (T*)w.ks, (T*)w.vs, (T*)w.kc, (T*)w.vc, w.Mb8, (T*)w.kcg, (T*)w.vcg);
    note_launch();
}

}  // namespace

void launch_pool(const Plan* p, const Workspace& w, const void* k, const void* v, const float* wc,
                 cudaStream_t st) {
    switch (w.dtype) {
    case SSA_F32: run_pool<float>(p, w, k, v, wc, st); break;
    case SSA_BF16: run_pool<__nv_bfloat16>(p, w, k, v, wc, st); break;
    default: run_pool<__half>(p, w, k, v, wc, st); break;
    }
}

}  // namespace ssa
