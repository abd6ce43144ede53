// Device pieces of the tensor-core forward: the parameter block and 16-bit packing.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "prologue.cuh"
#include "tc.cuh"

namespace ssa {
namespace attn {

constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 2 GHz

struct FwdParams {
    const void* q;
    const void* ks;    // grouped order, [H, Nks, D]: padded block rows, then the pools
    const void* vs;
    const void* kcg;   // grouped order, [H, Mb8, D]
    const void* vcg;
    const float* gates;
    const int32_t* perm;
    const int32_t* tok_blk;
    const int32_t* blk_off;
    const int32_t* blk_poff;
    const int2* blk_info;     // (first 8-row group, tokens) per block
    const int32_t* blk_tpool; // row of a small block in its sequence's pool (relative), -1 if none
    const int2* seq_pool;     // (first 8-row group, groups) of each sequence's pool
    const int4* scoord;
    const int32_t* qt_pos;
    const int32_t* qt_len;
    const int32_t* qt_seq;
    const int32_t* seq_blk;
    const int32_t* wr_off;
    const int2* wr_runs;
    const int32_t* wg_cnt;
    const int32_t* wm_off;
    const uint64_t* wmask;
    int32_t* sel;
    float* base;
    void* out;
    float* bout[3];   // optional per-branch outputs (fp32, token order), null when not wanted
    // gates predicted from the queries (selection kernel; null gate_w = off)
    const float* gate_w;
    const float* gate_b;
    float* gates_out;
    // attention prologue on the query tiles (null q_gamma = off)
    const float* q_gamma;
    const int32_t* coords;
    double theta;
    float eps;
    int32_t* status;
    int64_t N, Nks, Mb, Mb8;
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

// Attention prologue on a query tile held in shared memory in the chunked, 64-byte-swizzled
// operand order (32-column chunks `qreg` bytes apart): row `row` (token `tok`) is RMS-normalised
// over the head dimension and turned by the 3D rotary embedding, in place, in fp32, and rounded
// back to T. freq / axis: the rotary table of the D/2 channel pairs; gamma: [D] weights.
template <typename T, int D>
__device__ __forceinline__ void qtile_prologue(uint8_t* qtile, uint32_t qreg, int row, int32_t tok,
                                               const int32_t* coords, const double* freq,
                                               const int* axis, const float* gamma, float eps) {
    const int32_t cx = coords[3 * tok], cy = coords[3 * tok + 1], cz = coords[3 * tok + 2];
    float ss = 0.0f;
#pragma unroll 1
    for (int c16 = 0; c16 < D / 8; ++c16) {
        const uint4 u = *reinterpret_cast<const uint4*>(qtile + (c16 >> 2) * qreg + tc::sw64(row, c16 & 3));
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a = unpack_lo<T>(w[q]), b = unpack_hi<T>(w[q]);
            ss = fmaf(a, a, fmaf(b, b, ss));
        }
    }
    const float inv = rsqrtf(ss / (float)D + eps);
#pragma unroll 1
    for (int c16 = 0; c16 < D / 8; ++c16) {
        uint4* up = reinterpret_cast<uint4*>(qtile + (c16 >> 2) * qreg + tc::sw64(row, c16 & 3));
        uint4 u = *up;
        uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int pr = c16 * 4 + q;
            float c, sn;
            rope_cos_sin(axis_coord(axis[pr], cx, cy, cz), freq[pr], c, sn);
            const float a = unpack_lo<T>(w[q]) * inv * gamma[2 * pr];
            const float b = unpack_hi<T>(w[q]) * inv * gamma[2 * pr + 1];
            w[q] = pack2<T>(a * c - b * sn, a * sn + b * c);
        }
        *up = u;
    }
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    uint32_t s = tc::smem_u32(p);
    return p + ((1024u - (s & 1023u)) & 1023u);
}

}  // namespace attn
}  // namespace ssa
