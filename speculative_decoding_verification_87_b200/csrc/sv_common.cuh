// sv_common.cuh -- shared device helpers of the verification sampler kernels.
//
// Element storage tags, 16-byte vector loads, NaN-propagating max, warp and
// block reductions and the per-call parameter block.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sv_exp64.cuh"

namespace sv {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xFFFFFFFFu;

// Per-request status bits (mirror SPEC_STATUS_* in the public header).
enum : int { kStToken = 1, kStTree = 2, kStLogit = 4, kStTimeout = 8 };

// Philox counter purposes.
enum : uint32_t { kPurposeAccept = 0, kPurposeSample = 1 };

// Pass-2 segment: 2048 vocabulary entries, 64 contiguous entries per lane.
constexpr int kSeg2 = 512;
constexpr int kLane2 = kSeg2 / 32;

// Storage tags: element type and entries per 16-byte vector.
struct Bf16 {
    using elem = uint16_t;
    static constexpr int kVec = 8;
    static constexpr uint32_t kNegInfWord = 0xFF80FF80u;  // two bf16 -inf
};
struct F32 {
    using elem = float;
    static constexpr int kVec = 4;
    static constexpr uint32_t kNegInfWord = 0xFF800000u;  // fp32 -inf
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 2^x on the special-function unit (flushes subnormal results to zero).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two fp32 lanes in one 64-bit register pair, and the packed fp32x2 FMA and
// add of sm_100 (each lane rounded as its scalar instruction would be).
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x for x <= 0 on the FMA pipe: round x to the nearest integer n with the
// 1.5 * 2^23 shift, evaluate 2^f (f = x - n in [-1/2, 1/2]) by its Taylor
// polynomial of degree 6 (sum (f ln 2)^k / k!, truncation below 1.2e-7
// relative) and add n to the exponent field.  Results below 2^-125 are 0.
// Used for part of the pass-1 exponentials so that the special-function
// unit, which the rest can saturate, is not the limit.
constexpr float kF1 = 0.693147180559945309f;
constexpr float kF2 = 0.240226506959100712f;
constexpr float kF3 = 0.0555041086648215800f;
constexpr float kF4 = 0.00961812910762847716f;
constexpr float kF5 = 0.00133335581464284434f;
constexpr float kF6 = 0.000154035303933816099f;
__device__ __forceinline__ float ex2_fma(float x)
{
    const float xc = fmaxf(x, -125.0f);
    const float t = __fadd_rn(xc, 12582912.0f);  // 1.5 * 2^23
    const float f = xc - __fadd_rn(t, -12582912.0f);
    float q = fmaf(kF6, f, kF5);
    q = fmaf(q, f, kF4);
    q = fmaf(q, f, kF3);
    q = fmaf(q, f, kF2);
    q = fmaf(q, f, kF1);
    q = fmaf(q, f, 1.0f);
    const int n = __float_as_int(t) - 0x4B400000;
    const float r = __int_as_float(__float_as_int(q) + (n << 23));
    return x < -125.0f ? 0.0f : r;
}

// Exact float -> double widening with integer operations only (no
// conversion instruction); subnormal floats become signed zero, which no
// fp64 quantity here can tell apart from them.
__device__ __forceinline__ double f32_to_f64(float v)
{
    const uint32_t u = __float_as_uint(v);
    const uint32_t sign = u & 0x80000000u;
    const uint32_t e = (u >> 23) & 0xFFu;
    const uint32_t m = u & 0x7FFFFFu;
    uint32_t hi, lo;
    if (e == 0xFFu) {
        hi = sign | 0x7FF00000u | (m >> 3);
        lo = m << 29;
    } else if (e == 0u) {
        hi = sign;
        lo = 0u;
    } else {
        hi = sign | ((e + 896u) << 20) | (m >> 3);
        lo = m << 29;
    }
    return __hiloint2double(static_cast<int>(hi), static_cast<int>(lo));
}

// n / d and n % d for a divisor fixed per launch, by multiply-high and
// shift (no division instruction): with l = ceil(log2 d) and
// m = floor(2^(32+l) / d) + 1, q = (n * m) >> (32 + l) is exact for
// n, d < 2^31.
struct FastDiv {
    uint32_t d;
    uint32_t shift;
    uint64_t m;
};
__host__ __device__ inline FastDiv make_fastdiv(uint32_t d)
{
    FastDiv f;
    f.d = d;
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    f.shift = 32 + l;
    f.m = ((1ull << (32 + l)) / d) + 1;
    return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f)
{
    return static_cast<uint32_t>((static_cast<uint64_t>(n) * f.m) >> f.shift);
}

// max that returns NaN when either input is NaN (a NaN logit must poison
// the row so that the request is reported, never silently skipped).
__device__ __forceinline__ float max_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ uint4 ldg_vec(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// One logit, widened exactly to fp32.
template <class Tag>
__device__ __forceinline__ float load_logit(const void *base, int64_t index);
template <>
__device__ __forceinline__ float load_logit<Bf16>(const void *base, int64_t index)
{
    return __uint_as_float(uint32_t(__ldg(reinterpret_cast<const uint16_t *>(base) + index)) << 16);
}
template <>
__device__ __forceinline__ float load_logit<F32>(const void *base, int64_t index)
{
    return __ldg(reinterpret_cast<const float *>(base) + index);
}

// Replace entries [nvalid, kVec) of a raw vector by -inf.
template <class Tag>
__device__ __forceinline__ uint4 mask_tail(uint4 v, int nvalid);
template <>
__device__ __forceinline__ uint4 mask_tail<Bf16>(uint4 v, int nvalid)
{
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; ++e)
        if (e >= nvalid) {
            if (e & 1) w[e >> 1] = (w[e >> 1] & 0x0000FFFFu) | 0xFF800000u;
            else w[e >> 1] = (w[e >> 1] & 0xFFFF0000u) | 0x0000FF80u;
        }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ uint4 mask_tail<F32>(uint4 v, int nvalid)
{
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
        if (e >= nvalid) w[e] = 0xFF800000u;
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Unpack a raw vector to fp32 values.
template <class Tag>
__device__ __forceinline__ void unpack(uint4 v, float (&x)[Tag::kVec]);
template <>
__device__ __forceinline__ void unpack<Bf16>(uint4 v, float (&x)[8])
{
    x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x);
    x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
    x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z);
    x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}
template <>
__device__ __forceinline__ void unpack<F32>(uint4 v, float (&x)[4])
{
    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
}

// NaN-propagating max of a raw vector.
template <class Tag>
__device__ __forceinline__ float vec_max(uint4 v);
template <>
__device__ __forceinline__ float vec_max<Bf16>(uint4 v)
{
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&v.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&v.y);
    __nv_bfloat162 c = *reinterpret_cast<__nv_bfloat162 *>(&v.z);
    __nv_bfloat162 d = *reinterpret_cast<__nv_bfloat162 *>(&v.w);
    __nv_bfloat162 m = __hmax2_nan(__hmax2_nan(a, b), __hmax2_nan(c, d));
    return max_nan(__low2float(m), __high2float(m));
}
template <>
__device__ __forceinline__ float vec_max<F32>(uint4 v)
{
    return max_nan(max_nan(__uint_as_float(v.x), __uint_as_float(v.y)),
                   max_nan(__uint_as_float(v.z), __uint_as_float(v.w)));
}

// Argmax combine: larger value wins, ties go to the lower index.
__device__ __forceinline__ void argmax_take(float &bv, int &bi, float ov, int oi)
{
    if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
    }
}


// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_max_nan(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max_nan(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ int warp_min(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ int warp_max(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

// ------------------------------------------------------- per-call parameters
// What the final draw of one request needs.
enum : int { kModeNone = 0, kModeTargetRow = 1, kModeResidual = 2 };
struct __align__(64) ReqInfo {
    int64_t t_off;   // element offset of the target row of the final draw
    int64_t d_off;   // element offset of the draft row (residual only)
    double u;        // uniform of the final draw
    double rho_lo;   // bounds on S_t / S_d (row normalisers relative to their
    double rho_hi;   //   maxima) from the fp32 pass (residual only)
    float mt, md;    // row maxima
    int mode;        // kMode*
    int out_index;   // flat index into out_tokens of the drawn token
    float kc;        // (mt - md) c + log2(rho0), rho0 the pass-1 estimate of
                     //   S_t / S_d: log2(e/f) - log2(rho0) = (l_t - l_d) c - kc
    float tcls;      // |(l_t - l_d) c - kc| <= tcls: the sign of p - q is not
                     //   certain from fp32 (residual only)
};

enum : int { kLinear = 0, kTreeStochastic = 1, kTreeGreedy = 2 };

struct Params {
    const void *tl;          // target logits
    const void *dl;          // draft logits (may be null for greedy trees)
    int64_t stride;          // row pitch in elements
    const int32_t *tokens;   // linear: draft tokens [B][k]; tree: node tokens [B][N]
    const int32_t *parents;  // tree only
    int B, k, N, max_depth, V;
    int R;                   // rows per request streamed by pass 1
    int S;                   // pass-1 items per row
    int S2;                  // pass-2 segments per row
    int W32;                 // 32-bit words of one request's ambiguity bitmap
    unsigned nA, nP;         // pass-1 and pass-2 item counts
    FastDiv div_req;         // by R * S (pass-1 items per request)
    FastDiv div_s;           // by S
    FastDiv div_s2;          // by S2
    float c;                 // log2(e) / T, fp32
    double c64;              // log2(e) / T, fp64
    double inv_t;            // 1 / T, fp64
    uint64_t seed;
    uint32_t offset;
    int32_t *out;            // [B][W]
    int32_t *acc;            // [B]
    int32_t *path;           // tree only, nullable
    float *dbg_lp, *dbg_lq;  // linear only, nullable
    int32_t *status;         // nullable
    // workspace
    float2 *rowpart;         // [B][R][S] pass-1 partials
    ReqInfo *req;            // [B]
    double4 *p2part;         // [B][S2] (sum e, sum f, sum e over p>q, sum f over p>q)
    int *p2amb;              // [B][S2] undecided entries per segment
    unsigned *ambbits;       // [B][W32] undecided entries, one bit each
    double *p2w;             // [B][2][S2] finalize scratch (vocabularies too large for shared memory)
    double2 *p2lane;         // [B][S2][32] per-lane sums of pass 2 (decided part)
    // one-kernel linear path (set to all ones per call, with rowpart)
    unsigned *p2cnt;         // [B] pass-2 items completed per request
    unsigned *p2claim;       // tasks claimed
    unsigned *a_claim;       // pass-1 chunks claimed past nAs
    unsigned *decided;       // [B] 1 once the request's decision is published
    unsigned nAs;            // pass-1 items taken in static round robin
    unsigned poll_limit;     // polls before a wait gives up (SPEC_STATUS_TIMEOUT)
    int diag_no_partials;    // diagnostic only: pass 1 stores no partial, so every wait expires
    double exp2tab[kExp2Tab]; // 2^(j/256), j = 0..255
};

__device__ __forceinline__ void report(int32_t *status, int bits)
{
    if (status && bits) atomicOr(status, bits);
}

}  // namespace sv
