// sv_common.cuh -- shared device helpers of the verification sampler kernels.
//
// Element storage tags, 16-byte vector loads, NaN-propagating max, warp and
// block reductions and the per-call parameter block.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sv {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xFFFFFFFFu;

// Per-request status bits (mirror SPEC_STATUS_* in the public header).
enum : int { kStToken = 1, kStTree = 2, kStLogit = 4 };

// Philox counter purposes.
enum : uint32_t { kPurposeAccept = 0, kPurposeSample = 1 };

// Pass-2 segment: 4096 vocabulary entries, 16 contiguous entries per thread.
constexpr int kSeg2 = 4096;
constexpr int kPerThread2 = kSeg2 / kThreads;

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

// Block-wide reductions over kThreads threads; every thread gets the result.
// `red` is shared scratch of at least kWarps elements of the value type.
__device__ __forceinline__ float block_max_nan(float v, float *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_max_nan(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) r = max_nan(r, red[w]);
    return r;
}
__device__ __forceinline__ float block_sum(float v, float *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) r += red[w];
    return r;
}
__device__ __forceinline__ double block_sum(double v, double *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double r = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) r += red[w];
    return r;
}
__device__ __forceinline__ int block_min(int v, int *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_min(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int r = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) r = min(r, red[w]);
    return r;
}
__device__ __forceinline__ int block_max(int v, int *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_max(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int r = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) r = max(r, red[w]);
    return r;
}

// ------------------------------------------------------- per-call parameters
// Merged statistics of one logit row.
struct RowStat {
    float m;   // row maximum (greedy: maximum value)
    int idx;   // greedy: argmax (lowest index on ties)
    double s;  // stochastic: sum_v exp((l_v - m) / T)
};

// What pass 2 must do for one request.
enum : int { kModeNone = 0, kModeTargetRow = 1, kModeResidual = 2 };
struct __align__(64) ReqInfo {
    int64_t t_off;   // element offset of the target row pass 2 reads
    int64_t d_off;   // element offset of the draft row (residual only)
    double u;        // uniform of the final sample
    double inv_sp;   // 1 / sum_v exp((l_v - m_t) / T), fp64 (residual only)
    double inv_sq;   // 1 / sum_v exp((d_v - m_d) / T), fp64 (residual only)
    float mt, md;    // row maxima
    int mode;        // kMode*
    int out_index;   // flat index into out_tokens of the sampled token
};

enum : int { kLinear = 0, kTreeStochastic = 1, kTreeGreedy = 2 };

struct Params {
    const void *tl;          // target logits
    const void *dl;          // draft logits (may be null for greedy trees)
    int64_t stride;          // row pitch in elements
    const int32_t *tokens;   // linear: draft tokens [B][k]; tree: node tokens [B][N]
    const int32_t *parents;  // tree only
    int B, k, N, max_depth, V;
    int R;                   // rows per request handled by pass 1
    int S;                   // pass-1 segments per row
    int seg;                 // pass-1 segment length (entries)
    int S2;                  // pass-2 segments per row
    float c;                 // log2(e) / T, fp32
    double inv_t;            // 1 / T, fp64
    uint64_t seed;
    uint32_t offset;
    int32_t *out;            // [B][W]
    int32_t *acc;            // [B]
    int32_t *path;           // tree only, nullable
    float *dbg_lp, *dbg_lq;  // linear only, nullable
    int32_t *status;         // nullable
    // workspace regions
    float2 *rowpart;         // [B][R][S]
    RowStat *rowstat;        // [B][R]
    ReqInfo *req;            // [B]
    double2 *p2a;            // [B][S2]
    double *p2b;             // [B][S2]
    unsigned *cnt1, *cnt2a, *cnt2b;  // [B] each
};

__device__ __forceinline__ void report(int32_t *status, int bits)
{
    if (status && bits) atomicOr(status, bits);
}

// "Last block done" counter: returns true in every thread of exactly one
// block (the last of `total` arrivals); that block resets the counter to
// zero, so the workspace is left zero-filled for the next call.  Callers
// write their partial results before calling.  No block ever waits.
__device__ __forceinline__ bool arrive_last(unsigned *counter, unsigned total)
{
    __shared__ int last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned prev = atomicAdd(counter, 1u);
        last = (prev == total - 1);
        if (last) {
            atomicExch(counter, 0u);
            __threadfence();
        }
    }
    __syncthreads();
    return last != 0;
}

}  // namespace sv
