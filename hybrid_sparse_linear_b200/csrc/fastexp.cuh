// 2^y on the FMA pipe, for spreading the softmax exponentials over two execution units: the
// multi-function unit (ex2.approx) and the fp32 FMA pipe (this polynomial), the split
// FlashAttention-4 uses on this architecture.
//
// Method (two values at a time on the packed two-wide fp32 path):
//   1. clamp y to [-125, +inf) so that every result below is a normal fp32 number;
//   2. Cody-Waite style reduction: j = round(y) by adding and subtracting 1.5 * 2^23 (the integer
//      lands in the low mantissa bits of the shifted sum), f = y - j in [-1/2, 1/2];
//   3. 2^f ~ p(f), the degree-3 polynomial minimax in relative error on [-1/2, 1/2], fitted by
//      Lawson's iteration (fit_exp2_poly.py beside this file), evaluated by Horner; max relative
//      error 7.5e-5, below a bf16 rounding (2^-9) by a factor of 26;
//   4. 2^y = p(f) * 2^j by adding j to the exponent field (an integer add of j << 23).
// Valid for y <= 127 (larger y would overflow the exponent field).  y = -inf gives 2^-125, a
// value below every fp32 ulp the callers accumulate it into (their sums hold at least one term
// equal to 1), never 0: a caller that must tell "no term at all" apart checks that itself.
#pragma once

#include "ptx.cuh"

namespace sala {

constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.24261100590229034f;
constexpr float kExp2C3 = 0.055171530693769455f;

// (y0, y1) <- (2^y0, 2^y1).
__device__ __forceinline__ void exp2_poly2(float& y0, float& y1) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    y0 = fmaxf(y0, -125.f);
    y1 = fmaxf(y1, -125.f);
    float t0, t1, j0, j1, f0, f1, p0, p1;
    ptx::fma2_bcast(t0, t1, y0, y1, 1.f, kShift);        // t = y + shift: round(y) in the low bits
    ptx::fma2_bcast(j0, j1, t0, t1, 1.f, -kShift);       // j = t - shift (exact)
    asm("{\n\t.reg .b64 ya, ja, fa;\n\t"
        "mov.b64 ya, {%2, %3};\n\tmov.b64 ja, {%4, %5};\n\t"
        "sub.rn.f32x2 fa, ya, ja;\n\t"
        "mov.b64 {%0, %1}, fa;\n\t}"
        : "=f"(f0), "=f"(f1)
        : "f"(y0), "f"(y1), "f"(j0), "f"(j1));           // f = y - j, exact
    // Horner on pairs: p = ((c3 f + c2) f + c1) f + c0
    asm("{\n\t.reg .b64 fa, pa, ca;\n\t"
        "mov.b64 fa, {%2, %3};\n\t"
        "mov.b64 pa, {%4, %4};\n\t"
        "mov.b64 ca, {%5, %5};\n\t"
        "fma.rn.f32x2 pa, pa, fa, ca;\n\t"
        "mov.b64 ca, {%6, %6};\n\t"
        "fma.rn.f32x2 pa, pa, fa, ca;\n\t"
        "mov.b64 ca, {%7, %7};\n\t"
        "fma.rn.f32x2 pa, pa, fa, ca;\n\t"
        "mov.b64 {%0, %1}, pa;\n\t}"
        : "=f"(p0), "=f"(p1)
        : "f"(f0), "f"(f1), "f"(kExp2C3), "f"(kExp2C2), "f"(kExp2C1), "f"(kExp2C0));
    y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
    y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

}  // namespace sala
