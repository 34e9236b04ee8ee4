// e^x in float64 for x <= 0, branch-free, for the integer masses of the mask
// cut (floor(e^x * 2^40) is 0 below x = -27.73, so only that range matters).
//
// Method (Cody and Waite, "Software Manual for the Elementary Functions",
// 1980): x = n ln2 + r with n the integer nearest x log2(e), r computed with
// ln2 split into a 32-bit head (n * head is exact for |n| < 2^21) and a tail,
// |r| <= ln2 / 2; e^r by its Taylor polynomial of degree 13 (truncation error
// below 5e-18 relative), Horner with fused multiply-adds; then 2^n added to
// the exponent field.  Arguments are clamped at -700 so that the result stays
// a normal number; x = -inf gives e^-700.  Every operation is a fixed fma/add,
// so independent calls interleave freely.  Its error is below one unit in the
// last place of e^x on [-30, 0] in a 50-digit check; a GPU test compares it
// with CUDA's exp.
#pragma once

namespace nabla {

__device__ __forceinline__ double exp_nonpos(double x) {
    const double kLog2e = 0x1.71547652b82fep+0;   // 1 / ln 2
    const double kLn2Hi = 0x1.62e42fee00000p-1;   // ln 2, leading 32 bits
    const double kLn2Lo = 0x1.a39ef35793c76p-33;  // ln 2 - kLn2Hi
    const double kRound = 0x1.8p52;               // adding it rounds to an integer
    const double xc = fmax(x, -700.0);
    const double t = fma(xc, kLog2e, kRound);     // n in the low mantissa bits
    const double n = t - kRound;
    double r = fma(-n, kLn2Hi, xc);
    r = fma(-n, kLn2Lo, r);
    // 1/k! rounded to double, k = 13 .. 2
    double p = 0x1.6124613a86d09p-33;
    p = fma(p, r, 0x1.1eed8eff8d898p-29);
    p = fma(p, r, 0x1.ae64567f544e4p-26);
    p = fma(p, r, 0x1.27e4fb7789f5cp-22);
    p = fma(p, r, 0x1.71de3a556c734p-19);
    p = fma(p, r, 0x1.a01a01a01a01ap-16);
    p = fma(p, r, 0x1.a01a01a01a01ap-13);
    p = fma(p, r, 0x1.6c16c16c16c17p-10);
    p = fma(p, r, 0x1.1111111111111p-7);
    p = fma(p, r, 0x1.5555555555555p-5);
    p = fma(p, r, 0x1.5555555555555p-3);
    p = fma(p, r, 0.5);
    p = fma(p, r, 1.0);
    p = fma(p, r, 1.0);
    const int ni = __double2loint(t);  // n, exact: |n| < 2^11
    return __hiloint2double(__double2hiint(p) + (ni << 20), __double2loint(p));
}

}  // namespace nabla
