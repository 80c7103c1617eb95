// GELU in the erf form, 0.5 x (1 + erf(x / sqrt 2)), for the GEMM and fused
// FFN epilogues.  erf is evaluated with the rational approximation of
// Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26
// (after C. Hastings):
//   erf(u) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-u^2),
//   t = 1 / (1 + p u), u >= 0, |error| <= 1.5e-7,
// with erf odd, so 1 + erf(-u) = t (...) exp(-u^2) needs no subtraction.
// One reciprocal and one exp2 on the MUFU unit and six FMAs per value.
#pragma once

namespace lf {

__device__ __forceinline__ float gelu_erf_as(float x) {
    constexpr float kP = 0.3275911f, kA1 = 0.254829592f, kA2 = -0.284496736f, kA3 = 1.421413741f,
                    kA4 = -1.453152027f, kA5 = 1.061405429f;
    const float u = fabsf(x) * 0.70710678118654752f;  // |x| / sqrt 2
    float t, e;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(kP, u, 1.0f)));
    float y = fmaf(t, kA5, kA4);
    y = fmaf(t, y, kA3);
    y = fmaf(t, y, kA2);
    y = fmaf(t, y, kA1);
    y *= t;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-u * u * 1.4426950408889634f));  // exp(-u^2)
    const float tail = y * e;                                // 1 - erf(u)
    const float phi2 = x >= 0.0f ? 2.0f - tail : tail;        // 1 + erf(x / sqrt 2)
    return 0.5f * x * phi2;
}

}  // namespace lf
