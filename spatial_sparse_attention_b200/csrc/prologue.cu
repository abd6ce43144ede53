// Attention prologue as a separate pass for the fp32 path (Hi3D v1.0 pipeline page, "Stage 3:
// sparse flow sampling": RMS normalisation and rotary position embedding of the self-attention
// queries and keys). The 16-bit path applies the same transform inside the pooling kernel (keys)
// and after each query tile's load in the fused kernel (queries) instead.
//
// One half-warp per (token, head) row: thread i of it holds channels [i*D/16, (i+1)*D/16), an even
// count, so every rotated pair is thread-local; the sum of squares is a half-warp reduction.
#include "prologue.cuh"

namespace ssa {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) k_qk_prologue_f32(const float* __restrict__ x,
                                                              const int32_t* __restrict__ coords,
                                                              const float* __restrict__ gamma,
                                                              double theta, float eps, int64_t N,
                                                              int H, int D, float* __restrict__ out) {
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;   // token * H + head
    const int i = threadIdx.x & 15;
    const unsigned hmask = 0xffffu << (threadIdx.x & 16);
    const bool ok = row < N * H;
    const int per = D / 16;   // 2, 4, 6 or 8 channels
    const int64_t base = (ok ? row : 0) * D + i * per;
    float v[8], ss = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        v[e] = (ok && e < per) ? x[base + e] : 0.0f;
        ss = fmaf(v[e], v[e], ss);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(hmask, ss, o, 16);
    if (!ok) return;
    const float inv = rsqrtf(ss / (float)D + eps);
    const int64_t tok = row / H;
    const int32_t cx = coords[3 * tok], cy = coords[3 * tok + 1], cz = coords[3 * tok + 2];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if (2 * q >= per) break;
        const int d = i * per + 2 * q;
        int axis;
        double freq;
        rope_pair(D, d / 2, theta, axis, freq);
        float c, s;
        rope_cos_sin(axis_coord(axis, cx, cy, cz), freq, c, s);
        const float a = v[2 * q] * inv * gamma[d], b = v[2 * q + 1] * inv * gamma[d + 1];
        out[base + 2 * q] = a * c - b * s;
        out[base + 2 * q + 1] = a * s + b * c;
    }
}

}  // namespace

void launch_qk_prologue_f32(const Plan* p, const float* x, const float* gamma, const Prologue& pro,
                            int H, int D, float* out, cudaStream_t st) {
    const int64_t threads = p->N * H * 16;
    k_qk_prologue_f32<<<(unsigned)cdiv(threads, kThreads), kThreads, 0, st>>>(
        x, p->coords, gamma, pro.theta, pro.eps, p->N, H, D, out);
    note_launch();
}

}  // namespace ssa
