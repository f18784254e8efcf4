// Coefficients of the FMA-pipe exp2 of the attention kernel: 2^r ~ c0 + c1 r +
// ... + c5 r^5 on r in [-1/2, 1/2], a least-squares fit of the relative error on
// Chebyshev nodes in FP64 with c0 = 1, rounded to FP32 (exp2_poly_fit.py
// reproduces them).  Maximum relative error of the FP32 Horner evaluation:
// 1.6e-7 (the MUFU ex2.approx.f32 it stands in for has a maximum relative
// error of about 2^-22).
#pragma once

namespace h3 {
constexpr float kExp2C0 = 1.0f;
constexpr float kExp2C1 = 0.6931468844413757f;
constexpr float kExp2C2 = 0.24022237956523895f;
constexpr float kExp2C3 = 0.05550893023610115f;
constexpr float kExp2C4 = 0.009671698324382305f;
constexpr float kExp2C5 = 0.0013218672247603536f;
}  // namespace h3
