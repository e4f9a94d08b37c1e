// sv_exp64.cuh -- 2^z in fp64 for z <= 0, table driven.
//
// Method: P. T. P. Tang, "Table-driven implementation of the exponential
// function in IEEE floating-point arithmetic", ACM TOMS 15(2), 1989.
// Reduce z = e + j/256 + r with integer e, j in [0, 256) and |r| <= 1/512;
// 2^z = 2^e * 2^(j/256) * 2^r, where 2^(j/256) comes from a 256-entry table
// and 2^r = 1 + r q(r) with q(r) = (2^r - 1)/r from the Taylor series of
// exp(r ln 2), kept to degree 3 (the first omitted term is below
// (ln2/512)^5 / 120 ~ 3.8e-17 relative).  2^(j/256 + r) is formed as
// tj + (tj r) q(r), so the product tj r runs beside the Horner chain.
//
// The table (2^(j/256), j = 0..255, 2 KB) lives in shared memory; the
// caller fills it once per block.
#pragma once

#include <cstdint>

namespace sv {

constexpr int kExp2Tab = 256;

// Taylor coefficients (ln 2)^n / n!, formed from ln 2 in double arithmetic.
constexpr double kLn2 = 0.69314718055994530941723212145818;
constexpr double kE1 = kLn2;
constexpr double kE2 = kE1 * kLn2 / 2.0;
constexpr double kE3 = kE2 * kLn2 / 3.0;
constexpr double kE4 = kE3 * kLn2 / 4.0;

// 2^z for z <= 0.  Results below 2^-1020 (and NaN arguments) give 0: such
// terms cannot move a sum whose largest term is 1, and an entry whose logit
// is -inf must keep weight exactly 0.  2^floor(k/256) enters the exponent
// field of the table value, beside the polynomial chain.
__device__ __forceinline__ double exp2_fp64(double z, const double *tab)
{
    constexpr double kMagic = 6755399441055744.0;  // 1.5 * 2^52: rounds to an integer
    const double t = fma(z, 256.0, kMagic);
    const int k = __double2loint(t);                     // round(256 z), two's complement
    const double r = fma(t - kMagic, -0.00390625, z);    // z - k/256, exact
    const double tj = tab[k & 255];                      // 2^(j/256)
    const unsigned ehi = static_cast<unsigned>(__double2hiint(tj)) + (static_cast<unsigned>(k >> 8) << 20);
    const double ts = __hiloint2double(static_cast<int>(ehi), __double2loint(tj));  // 2^(k/256), z > -1020
    double q = fma(kE4, r, kE3);
    q = fma(q, r, kE2);
    q = fma(q, r, kE1);
    const double y = fma(ts * r, q, ts);
    return z > -1020.0 ? y : 0.0;
}


}  // namespace sv
