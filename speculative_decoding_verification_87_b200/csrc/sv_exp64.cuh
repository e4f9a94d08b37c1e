// sv_exp64.cuh -- 2^z in fp64 for z <= 0, table driven.
//
// Method: P. T. P. Tang, "Table-driven implementation of the exponential
// function in IEEE floating-point arithmetic", ACM TOMS 15(2), 1989.
// Reduce z = e + j/64 + r with integer e, j in [0, 64) and |r| <= 1/128;
// 2^z = 2^e * 2^(j/64) * 2^r, where 2^(j/64) comes from a 64-entry table and
// 2^r = exp(r ln 2) from its Taylor polynomial of degree 5 (the first omitted
// term is below (ln2/128)^6 / 720 ~ 3.5e-17 relative).
//
// The table lives in registers, two entries per lane (lane L holds
// 2^(L/64) and 2^((L+32)/64)), and is read with a warp shuffle, so every
// lane of the warp must call exp2_fp64 together.
#pragma once

#include <cstdint>

namespace sv {

// Taylor coefficients (ln 2)^n / n!, formed from ln 2 in double arithmetic.
constexpr double kLn2 = 0.69314718055994530941723212145818;
constexpr double kE1 = kLn2;
constexpr double kE2 = kE1 * kLn2 / 2.0;
constexpr double kE3 = kE2 * kLn2 / 3.0;
constexpr double kE4 = kE3 * kLn2 / 4.0;
constexpr double kE5 = kE4 * kLn2 / 5.0;

// Two table entries of this lane: 2^(lane/64) (lo) and 2^((lane+32)/64) (hi).
struct Exp2Table {
    double lo, hi;
};

// 2^z for z <= 0.  Results below 2^-1020 are returned as 0 (they cannot
// move a sum whose largest term is 1).  Warp-collective.
__device__ __forceinline__ double exp2_fp64(double z, const Exp2Table &tab)
{
    const bool tiny = !(z > -1020.0);
    const double zz = tiny ? 0.0 : z;
    constexpr double kMagic = 6755399441055744.0;  // 1.5 * 2^52: rounds to an integer
    const double t = fma(zz, 64.0, kMagic);
    const int k = __double2loint(t);               // round(64 z), two's complement
    const double kd = t - kMagic;
    const double r = fma(kd, -0.015625, zz);       // z - k/64, exact
    double p = fma(kE5, r, kE4);
    p = fma(p, r, kE3);
    p = fma(p, r, kE2);
    p = fma(p, r, kE1);
    p = p * r;                                     // 2^r - 1
    const int j = k & 63;
    const double lo = __shfl_sync(0xFFFFFFFFu, tab.lo, j & 31);
    const double hi = __shfl_sync(0xFFFFFFFFu, tab.hi, j & 31);
    const double tj = (j & 32) ? hi : lo;          // 2^(j/64)
    const double y = fma(tj, p, tj);               // 2^(j/64 + r), in [1, 2)
    const int e = k >> 6;                          // floor(k / 64), >= -1020
    const double scaled = __hiloint2double(__double2hiint(y) + (e << 20), __double2loint(y));
    return tiny ? 0.0 : scaled;
}

// Exact widening of a bf16 bit pattern (low 16 bits of h) to fp64 with
// integer operations only; subnormal values become signed zero (no fp64
// quantity here can tell them apart), infinities and NaN keep their class.
__device__ __forceinline__ double bf16_to_f64(uint32_t h)
{
    const uint32_t sign = (h & 0x8000u) << 16;
    const uint32_t e = (h >> 7) & 0xFFu;
    const uint32_t m = (h & 0x7Fu) << 13;
    const uint32_t hi = e == 0xFFu ? (sign | 0x7FF00000u | m)
                      : e == 0u    ? sign
                                   : (sign | ((e + 896u) << 20) | m);
    return __hiloint2double(static_cast<int>(hi), 0);
}

}  // namespace sv
