// Device pieces of the tensor-core forward: the parameter block, 16-bit packing and the register
// top-k list.
#pragma once

#include <type_traits>

#include "common.cuh"
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

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    uint32_t s = tc::smem_u32(p);
    return p + ((1024u - (s & 1023u)) & 1023u);
}

// Sorted top list (logit descending; among equal logits, lower block index first). Blocks are
// offered in ascending index order, so a new entry goes after every entry whose logit is >= its
// own. All positions are updated from the old list at once (no serial chain).
template <int KM>
__device__ __forceinline__ void topk_push(float (&tv)[KM], int32_t (&ti)[KM], float z, int32_t b) {
    bool c[KM];
#pragma unroll
    for (int t = 0; t < KM; ++t) c[t] = z > tv[t];
#pragma unroll
    for (int t = KM - 1; t > 0; --t) {
        tv[t] = c[t] ? (c[t - 1] ? tv[t - 1] : z) : tv[t];
        ti[t] = c[t] ? (c[t - 1] ? ti[t - 1] : b) : ti[t];
    }
    tv[0] = c[0] ? z : tv[0];
    ti[0] = c[0] ? b : ti[0];
}

}  // namespace attn
}  // namespace ssa
