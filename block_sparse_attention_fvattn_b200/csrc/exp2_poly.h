// exp2_poly.h -- coefficients of p(f) ~ 2^f on [-1/2, 1/2] (degree 3).
//
// Minimax for the relative error, fitted with the Remez exchange algorithm
// (exp2_poly_fit.py in this directory); max relative error 7.5e-5 in fp32
// Horner evaluation. Used as 2^x = 2^round(x) * p(x - round(x)).
#pragma once
#define FV_EXP2_C0 0.9999280571937561f
#define FV_EXP2_C1 0.6932609677314758f
#define FV_EXP2_C2 0.2426111251115799f
#define FV_EXP2_C3 0.0551716685295105f
