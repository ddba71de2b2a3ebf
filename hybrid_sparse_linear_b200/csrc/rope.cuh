// Rotary position embedding on the device: the linear layers' half of HyPE (MiniCPM-SALA
// summaries, JA section 2.2 "positional encoding (HyPE)", DE section 2 "HyPE": the linear
// attention layers rotate queries and keys by position, the sparse layers do not).
//
// Pairs: element i with element i + d/2 (i < d/2); frequency theta_i = base^(-2i/d); the angle of
// position p is p * theta_i:
//   x'_i       = x_i cos - x_{i+d/2} sin
//   x'_{i+d/2} = x_{i+d/2} cos + x_i sin
// Positions reach 2^20 and more, where a single-precision p * theta_i is off by a few hundredths
// of a radian, so the angle is reduced in turns in double precision first: t = p * theta_i / 2pi
// (relative error ~1e-16, i.e. ~1e-10 turns at p = 2^20), its fractional part in [-1/2, 1/2],
// then the multi-function unit's sine and cosine of 2 pi t, an angle in [-pi, pi] (absolute
// error ~1e-6, far below a bf16 rounding of the rotated values).
#pragma once

#include "common.cuh"

namespace sala {

// theta_i / (2 pi) in double.
__device__ __forceinline__ double rope_turn(double base, int i, int d) {
    return pow(base, -2.0 * (double)i / (double)d) * 0.15915494309189533577;
}

// cos and sin of p * theta_i, given turn = rope_turn(base, i, d).
__device__ __forceinline__ void rope_cs(double turn, int64_t p, float& c, float& s) {
    double t = (double)p * turn;
    t -= rint(t);
    __sincosf((float)(t * 6.283185307179586), &s, &c);
}

// (x0, x1) <- (x0 c - x1 s, x1 c + x0 s)
__device__ __forceinline__ void rope_rot(float& x0, float& x1, float c, float s) {
    const float a = x0 * c - x1 * s, b = x1 * c + x0 * s;
    x0 = a;
    x1 = b;
}

}  // namespace sala
