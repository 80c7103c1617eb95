// Packed fp32 pair arithmetic of the softmax warps (fma.rn.f32x2 /
// add.f32x2, sm_100) and the FMA-pipe exponential built on it.  Kept in a
// header of its own so that a test can compile exp2_poly2 into a small
// kernel and check it against exp2 in float64.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lf {

// Packed fp32 pair arithmetic (fma.rn.f32x2 / add.f32x2, sm_100).
static __device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
static __device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// 2^x for a pair on the FMA/ALU pipes, to take load off the MUFU unit
// (16 results per clock per SM).  Cody-Waite reduction x = n + f with
// n = round(x) (|f| <= 1/2, via the 1.5 * 2^23 rounding constant), then a
// cubic for 2^f whose coefficients were fitted for this kernel by iteratively
// reweighted least squares (Lawson) on Chebyshev nodes of [-1/2, 1/2]
// (max relative error 7.5e-5, below the rounding of P to fp16/bf16); the
// exponent n is added to the bits of the result.  x is clamped at -125 so the
// result stays a normal number (the cubic dips just below 1 at f = 0, so
// n = -126 would reach the subnormal range; 2^-125 rounds to 0 in fp16 and is
// far below anything that changes a sum in bf16).
static __device__ __forceinline__ float2 exp2_poly2(float2 x) {
    const float2 t = make_float2(fmaxf(x.x, -125.0f), fmaxf(x.y, -125.0f));
    const float2 rnd = make_float2(12582912.0f, 12582912.0f);
    const float2 j = fadd2(t, rnd);                                       // n in the low mantissa bits
    const float2 nf = fadd2(j, make_float2(-12582912.0f, -12582912.0f));  // n as a float
    const float2 f = ffma2(nf, make_float2(-1.0f, -1.0f), t);             // t - n, exact
    float2 q = ffma2(make_float2(0.0551716648f, 0.0551716648f), f, make_float2(0.2426111251f, 0.2426111251f));
    q = ffma2(q, f, make_float2(0.6932609677f, 0.6932609677f));
    q = ffma2(q, f, make_float2(0.9999280572f, 0.9999280572f));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(j.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(j.y) << 23)));
}

}  // namespace lf
