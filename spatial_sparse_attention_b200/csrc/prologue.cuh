// Attention prologue shared by the kernels that apply it: RMS normalisation of a query or key row
// over the head dimension, then the 3D rotary embedding at the token's voxel coordinates
// (Hi3D v1.0 pipeline page, "Stage 3: sparse flow sampling": rotary position embeddings and RMS
// normalisation of the self-attention queries and keys, over sparse voxel tokens).
//
// Layout of the rotary embedding: the head dimension is cut into an x part of D - 2c channels and
// y and z parts of c = 2 floor(D/6) channels each; channel pair (2p, 2p+1) belongs to the part its
// first channel falls in and, as the j-th pair of a part of width w, turns by the angle
// coordinate * theta^(-2j/w): (u, v) -> (u cos t - v sin t, u sin t + v cos t).
#pragma once

#include "common.cuh"

namespace ssa {

// Axis (0, 1, 2) and angular frequency theta^(-2j/w) of channel pair p of a head of D channels.
__device__ __forceinline__ void rope_pair(int D, int p, double theta, int& axis, double& freq) {
    const int c = 2 * (D / 6);
    const int wx = D - 2 * c;
    int j, w;
    if (2 * p < wx) {
        axis = 0; j = p; w = wx;
    } else if (2 * p < wx + c) {
        axis = 1; j = p - wx / 2; w = c;
    } else {
        axis = 2; j = p - (wx + c) / 2; w = c;
    }
    freq = pow(theta, -2.0 * (double)j / (double)w);
}

// Coordinate of a token along `axis` (selects, no indexed array).
__device__ __forceinline__ int32_t axis_coord(int axis, int32_t x, int32_t y, int32_t z) {
    return axis == 0 ? x : (axis == 1 ? y : z);
}

// cos and sin of coordinate * freq: the angle is formed in turns (freq / 2pi, exact enough in
// double) and reduced to [-1/2, 1/2] of a turn in double, so the result keeps fp32 accuracy at any
// coordinate of the supported grids.
__device__ __forceinline__ void rope_cos_sin(int32_t coord, double freq, float& c, float& s) {
    const double turns = (double)coord * (freq * 0.15915494309189533577);   // freq / (2 pi)
    const float r = (float)(turns - rint(turns)) * 6.2831853071795864769f;
    __sincosf(r, &s, &c);
}

}  // namespace ssa
