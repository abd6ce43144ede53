// Compression pooling: Kc_b = mean_{j in b}(K_j) . Wc and Vc_b likewise, per head, with
// one D x D map Wc shared by K, V and all heads (Direct3D-S2 summary page, "Technical
// principles", SSA item: block-level tokens from a compression of each block; the concrete
// mean-then-linear-map form is the formulation this library implements).
//
// One CTA per occupied block; the block's token indices are staged in shared memory, then
// kLanes tokens are read at a time (every row with coalesced 128-bit loads); sums are fp32. For
// the tensor-core path the same pass also writes the rows into the padded, head-major,
// block-ordered copies K_s, V_s [H, Nks, D] that the attention tiles read, and the
// compressed tokens a second time in the same order. A block of at most kPoolMaxTokens tokens is
// written twice: at its padded rows and, packed with the other small blocks of its sequence, in
// that sequence's pool after all padded rows.
//
// With a convolution compression (`means` non-null) the block means go to `means` instead and
// the compressed tokens are made by the convolution kernel (conv.cu).
//
// Grouped order (16-bit types): rows are taken 8 at a time; a group stores its D/32 column chunks
// one after the other, each as a 512-byte atom of 8 rows x 64 bytes in which the four 16-byte
// units of row i are permuted by unit ^= (i >> 1) & 3. This is the shared-memory operand order of
// the tensor cores with 64-byte swizzle, so a run of consecutive groups is copied to shared
// memory with one bulk copy and used there as is.
#include <algorithm>

#include "common.cuh"
#include "prologue.cuh"

namespace ssa {

namespace {

// Work split inside a block's CTA: a thread owns two adjacent 16-byte column units of the token
// rows (32 bytes) and one of kLanes token lanes; lane L visits the block's tokens L, L + kLanes, ...
// The lanes of a column pair are adjacent threads of one warp, so their partial sums are combined
// with shuffles, and every token row is still read with contiguous 32-byte pieces.
constexpr int kLanes = 4;
constexpr int kMaxBlockTokens = 512;   // 8^3 cells

template <typename T, bool kSorted>
__global__ void __launch_bounds__(512, 2) k_pool(const T* __restrict__ K, const T* __restrict__ V,
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
                                               T* __restrict__ kcg, T* __restrict__ vcg,
                                               float* __restrict__ means) {
    constexpr int kVec = 16 / sizeof(T);
    extern __shared__ float mean[];   // [2][H*D]: K means then V means
    __shared__ int32_t toks[kMaxBlockTokens];
    const int64_t b = blockIdx.x;
    const int HD = H * D;
    const int pairs = HD / (2 * kVec);   // 32-byte column pieces of a row
    const int32_t lo = blk_off[b], n = blk_off[b + 1] - lo;
    const int32_t prow = blk_poff[b];
    // row of the block's copy in its sequence's pool, -1 if it has none
    const int32_t trow = kSorted && blk_tpool[b] >= 0 ? 8 * seq_pool[blk_seq[b]].x + blk_tpool[b] : -1;
    for (int t = threadIdx.x; t < n; t += blockDim.x) toks[t] = perm[lo + t];
    __syncthreads();

    const int lane = threadIdx.x % kLanes;
    const int per_pass = blockDim.x / kLanes;   // column pieces handled per pass
    const int passes = (pairs + per_pass - 1) / per_pass;
    // every thread runs every pass (the shuffles below involve whole warps)
    for (int it = 0; it < passes; ++it) {
        const int pc = it * per_pass + (int)threadIdx.x / kLanes;
        const bool active = pc < pairs;
        float sk[2 * kVec], sv[2 * kVec];
#pragma unroll
        for (int e = 0; e < 2 * kVec; ++e) sk[e] = sv[e] = 0.0f;
        const int col = pc * 2 * kVec;   // first element column of the piece
        const int h = col / D, d = col % D;   // both units lie in one head (D % 32 == 0)
        const int64_t hoff = (int64_t)h * Nks * D * (int64_t)sizeof(T);
        if (active) {
            for (int t = lane; t < n; t += kLanes) {
                const int64_t tok = toks[t];
                const uint4* krow = reinterpret_cast<const uint4*>(K + tok * HD + col);
                const uint4* vrow = reinterpret_cast<const uint4*>(V + tok * HD + col);
                const uint4 k0 = krow[0], k1 = krow[1], v0 = vrow[0], v1 = vrow[1];
                const T* ke0 = reinterpret_cast<const T*>(&k0);
                const T* ke1 = reinterpret_cast<const T*>(&k1);
                const T* ve0 = reinterpret_cast<const T*>(&v0);
                const T* ve1 = reinterpret_cast<const T*>(&v1);
#pragma unroll
                for (int e = 0; e < kVec; ++e) {
                    sk[e] += Elem<T>::to_f(ke0[e]);
                    sk[kVec + e] += Elem<T>::to_f(ke1[e]);
                    sv[e] += Elem<T>::to_f(ve0[e]);
                    sv[kVec + e] += Elem<T>::to_f(ve1[e]);
                }
                if (kSorted) {
                    uint8_t* kb = reinterpret_cast<uint8_t*>(ks) + hoff;
                    uint8_t* vb = reinterpret_cast<uint8_t*>(vs) + hoff;
                    const int64_t a0 = grouped_off(prow + t, d, D), a1 = grouped_off(prow + t, d + kVec, D);
                    *reinterpret_cast<uint4*>(kb + a0) = k0;
                    *reinterpret_cast<uint4*>(kb + a1) = k1;
                    *reinterpret_cast<uint4*>(vb + a0) = v0;
                    *reinterpret_cast<uint4*>(vb + a1) = v1;
                    if (trow >= 0) {
                        const int64_t c0 = grouped_off(trow + t, d, D), c1 = grouped_off(trow + t, d + kVec, D);
                        *reinterpret_cast<uint4*>(kb + c0) = k0;
                        *reinterpret_cast<uint4*>(kb + c1) = k1;
                        *reinterpret_cast<uint4*>(vb + c0) = v0;
                        *reinterpret_cast<uint4*>(vb + c1) = v1;
                    }
                }
            }
        }
        // combine the lanes' partial sums (adjacent threads of one warp)
#pragma unroll
        for (int o = 1; o < kLanes; o <<= 1)
#pragma unroll
            for (int e = 0; e < 2 * kVec; ++e) {
                sk[e] += __shfl_xor_sync(0xffffffffu, sk[e], o);
                sv[e] += __shfl_xor_sync(0xffffffffu, sv[e], o);
            }
        if (active && lane == 0) {
            const float inv = 1.0f / (float)n;
#pragma unroll
            for (int e = 0; e < 2 * kVec; ++e) {
                mean[col + e] = sk[e] * inv;
                mean[HD + col + e] = sv[e] * inv;
            }
        }
    }
    __syncthreads();
    if (means) {
        // compression by convolution: the block means go out [2][H][Mb][D] (K, then V)
        for (int o = threadIdx.x; o < 2 * HD; o += blockDim.x) {
            const int which = o / HD, h = (o % HD) / D, e = o % D;
            means[(((int64_t)which * H + h) * Mb + b) * D + e] = mean[o];
        }
        return;
    }
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

// Pooling with the attention prologue applied to K first (16-bit types): the block means, the
// compressed tokens and the grouped copies are all of the normalised, rotated keys. Thread
// (lane L, head h, unit u) handles the 16-byte unit u (8 channels) of head h of the tokens
// L, L + kProLanes, ... of the block; the 16 threads of a (lane, head) are one half-warp, so the
// row's sum of squares is a shuffle reduction over the half-warp (units beyond D/8 contribute
// zero); both half-warps of a warp may belong to different lanes and run their own iterations.
constexpr int kProLanes = 2;

template <typename T>
__global__ void __launch_bounds__(512, 2) k_pool_pro(const T* __restrict__ K, const T* __restrict__ V,
                                                   const float* __restrict__ Wc,
                                                   const int32_t* __restrict__ perm,
                                                   const int32_t* __restrict__ blk_off,
                                                   const int32_t* __restrict__ blk_poff,
                                                   const int32_t* __restrict__ blk_tpool,
                                                   const int32_t* __restrict__ blk_seq,
                                                   const int2* __restrict__ seq_pool,
                                                   const int32_t* __restrict__ coords,
                                                   const float* __restrict__ k_gamma, double theta,
                                                   float eps, int64_t Mb, int H, int D, int64_t Nks,
                                                   T* __restrict__ ks, T* __restrict__ vs,
                                                   T* __restrict__ kc, T* __restrict__ vc,
                                                   int64_t Mb8, T* __restrict__ kcg,
                                                   T* __restrict__ vcg, float* __restrict__ means) {
    constexpr int kVec = 8;
    extern __shared__ float part[];   // [kProLanes][2][H*D] per-lane sums, then the means
    __shared__ int32_t toks[kMaxBlockTokens];
    const int64_t b = blockIdx.x;
    const int HD = H * D;
    const int32_t lo = blk_off[b], n = blk_off[b + 1] - lo;
    const int32_t prow = blk_poff[b];
    const int32_t trow = blk_tpool[b] >= 0 ? 8 * seq_pool[blk_seq[b]].x + blk_tpool[b] : -1;
    for (int t = threadIdx.x; t < n; t += blockDim.x) toks[t] = perm[lo + t];
    const int hpp = blockDim.x / (16 * kProLanes);   // heads per pass
    const int lane = threadIdx.x / (16 * hpp);
    const int hh = (threadIdx.x / 16) % hpp;
    const int u = threadIdx.x % 16;
    const unsigned hmask = 0xffffu << (threadIdx.x & 16);   // this half-warp
    const bool unit_ok = u < D / kVec;
    const int d0 = u * kVec;
    // this thread's four channel pairs: axis, frequency, weights (the same for every head)
    int ax[4];
    double fr[4];
    float gm[kVec];
#pragma unroll
    for (int q = 0; q < 4; ++q) rope_pair(D, (unit_ok ? d0 / 2 : 0) + q, theta, ax[q], fr[q]);
#pragma unroll
    for (int e = 0; e < kVec; ++e) gm[e] = unit_ok ? k_gamma[d0 + e] : 0.0f;
    __syncthreads();
    const float inv_d = 1.0f / (float)D;
    for (int h0 = 0; h0 < H; h0 += hpp) {
        const int h = h0 + hh;
        const bool ok = unit_ok && h < H;
        const int col = h * D + d0;
        const int64_t hoff = (int64_t)h * Nks * D * (int64_t)sizeof(T);
        float sk[kVec], sv[kVec];
#pragma unroll
        for (int e = 0; e < kVec; ++e) sk[e] = sv[e] = 0.0f;
        // every thread of a half-warp runs the same iterations (the shuffles need all 16)
        for (int t = lane; t < n; t += kProLanes) {
            const int64_t tok = toks[t];
            uint4 kq = make_uint4(0u, 0u, 0u, 0u), vq = kq;
            if (ok) {
                kq = *reinterpret_cast<const uint4*>(K + tok * HD + col);
                vq = *reinterpret_cast<const uint4*>(V + tok * HD + col);
            }
            const T* ke = reinterpret_cast<const T*>(&kq);
            const T* ve = reinterpret_cast<const T*>(&vq);
            float x[kVec], ss = 0.0f;
#pragma unroll
            for (int e = 0; e < kVec; ++e) {
                x[e] = Elem<T>::to_f(ke[e]);
                ss = fmaf(x[e], x[e], ss);
                sv[e] += Elem<T>::to_f(ve[e]);
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(hmask, ss, o, 16);
            const float inv = rsqrtf(ss * inv_d + eps);
            const int32_t cx = coords[3 * tok], cy = coords[3 * tok + 1], cz = coords[3 * tok + 2];
            uint4 ko;
            uint32_t* kw = reinterpret_cast<uint32_t*>(&ko);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float c, sn;
                rope_cos_sin(axis_coord(ax[q], cx, cy, cz), fr[q], c, sn);
                const float a = x[2 * q] * inv * gm[2 * q], bq = x[2 * q + 1] * inv * gm[2 * q + 1];
                // the transformed keys are values of the input type: the copies and the block
                // means both use the rounded values
                const T ta = Elem<T>::from_f(a * c - bq * sn), tb = Elem<T>::from_f(a * sn + bq * c);
                sk[2 * q] += Elem<T>::to_f(ta);
                sk[2 * q + 1] += Elem<T>::to_f(tb);
                kw[q] = (uint32_t)(*reinterpret_cast<const uint16_t*>(&ta)) |
                        ((uint32_t)(*reinterpret_cast<const uint16_t*>(&tb)) << 16);
            }
            if (ok) {
                uint8_t* kb = reinterpret_cast<uint8_t*>(ks) + hoff;
                uint8_t* vb = reinterpret_cast<uint8_t*>(vs) + hoff;
                const int64_t a0 = grouped_off(prow + t, d0, D);
                *reinterpret_cast<uint4*>(kb + a0) = ko;
                *reinterpret_cast<uint4*>(vb + a0) = vq;
                if (trow >= 0) {
                    const int64_t c0 = grouped_off(trow + t, d0, D);
                    *reinterpret_cast<uint4*>(kb + c0) = ko;
                    *reinterpret_cast<uint4*>(vb + c0) = vq;
                }
            }
        }
        if (ok) {
#pragma unroll
            for (int e = 0; e < kVec; ++e) {
                part[(lane * 2 + 0) * HD + col + e] = sk[e];
                part[(lane * 2 + 1) * HD + col + e] = sv[e];
            }
        }
    }
    __syncthreads();
    const float invn = 1.0f / (float)n;
    for (int o = threadIdx.x; o < 2 * HD; o += blockDim.x) {
        const int which = o / HD, c = o % HD;
        float acc = 0.0f;
        for (int l = 0; l < kProLanes; ++l) acc += part[(l * 2 + which) * HD + c];
        part[o] = acc * invn;   // lane 0's slots now hold the means (K then V)
    }
    __syncthreads();
    const float* mean = part;
    if (means) {
        for (int o = threadIdx.x; o < 2 * HD; o += blockDim.x) {
            const int which = o / HD, h = (o % HD) / D, e = o % D;
            means[(((int64_t)which * H + h) * Mb + b) * D + e] = mean[o];
        }
        return;
    }
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
        const int64_t gd = (int64_t)h * Mb8 * D * (int64_t)sizeof(T) + grouped_off(b, e & ~7, D) +
                           (e & 7) * (int64_t)sizeof(T);
        *reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(kcg) + gd) = Elem<T>::from_f(ak);
        *reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(vcg) + gd) = Elem<T>::from_f(av);
    }
}

template <typename T>
void run_pool_pro(const Plan* p, const Workspace& w, const void* k, const void* v, const float* wc,
                  const Prologue& pro, float* means, cudaStream_t st) {
    // heads per pass: as few passes over the block's tokens as 512 threads allow, heads spread evenly
    const int max_hpp = 512 / (16 * kProLanes);
    const int hpp = (int)cdiv(w.H, cdiv(w.H, max_hpp));
    const int threads = hpp * 16 * kProLanes;
    const size_t smem = sizeof(float) * 2 * kProLanes * w.H * w.D;
    if (smem > 40 * 1024)
        cudaFuncSetAttribute(k_pool_pro<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_pool_pro<T><<<(unsigned)p->Mb, threads, smem, st>>>(
        (const T*)k, (const T*)v, wc, p->perm, p->blk_off, p->blk_poff, p->blk_tpool, p->blk_seq,
        p->seq_pool, p->coords, pro.k_gamma, pro.theta, pro.eps, p->Mb, w.H, w.D, p->Nks,
        (T*)w.ks, (T*)w.vs, (T*)w.kc, (T*)w.vc, w.Mb8, (T*)w.kcg, (T*)w.vcg, means);
    note_launch();
}

template <typename T>
void run_pool(const Plan* p, const Workspace& w, const void* k, const void* v, const float* wc,
              float* means, cudaStream_t st) {
    constexpr int kVec = 16 / sizeof(T);
    const int HD = w.H * w.D;
    const int pairs = HD / (2 * kVec);
    // as few passes over the block's tokens as 512 threads allow, the pieces spread evenly
    const int64_t passes = cdiv((int64_t)pairs * kLanes, 512);
    int threads = (int)round_up(cdiv(pairs, passes) * kLanes, 32);
    if (threads < 128) threads = 128;
    const size_t smem = sizeof(float) * 2 * HD;
    const bool sorted = w.ks != nullptr;
    auto kern = sorted ? k_pool<T, true> : k_pool<T, false>;
    if (smem > 40 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<(unsigned)p->Mb, threads, smem, st>>>(
        (const T*)k, (const T*)v, wc, p->perm, p->blk_off, p->blk_poff, p->blk_tpool, p->blk_seq,
        p->seq_pool, p->Mb, w.H, w.D, p->Nks,
        (T*)w.ks, (T*)w.vs, (T*)w.kc, (T*)w.vc, w.Mb8, (T*)w.kcg, (T*)w.vcg, means);
    note_launch();
}

}  // namespace

void launch_pool(const Plan* p, const Workspace& w, const void* k, const void* v, const float* wc,
                 const Prologue& pro, float* means, cudaStream_t st) {
    if (pro.on() && w.dtype != SSA_F32) {
        if (w.dtype == SSA_BF16) run_pool_pro<__nv_bfloat16>(p, w, k, v, wc, pro, means, st);
        else run_pool_pro<__half>(p, w, k, v, wc, pro, means, st);
        return;
    }
    switch (w.dtype) {
    case SSA_F32: run_pool<float>(p, w, k, v, wc, means, st); break;
    case SSA_BF16: run_pool<__nv_bfloat16>(p, w, k, v, wc, means, st); break;
    default: run_pool<__half>(p, w, k, v, wc, means, st); break;
    }
}

}  // namespace ssa
