// sv_stats.cuh -- pass 1: one streaming read of every logit row.
//
// "Accelerating Sonar through speculation", section "Target-Draft":
// acceptance compares the full draft and target distributions, so each row
// needs its whole-vocabulary normaliser.  A block reduces one segment of one
// row to (max, sum exp((l - max)/T)) (stochastic modes) or to (max value,
// lowest argmax) (greedy trees) and stores the partial in the workspace.
// The last block of a request to finish runs that request's decide step
// (sv_decide.cuh), so no block ever waits for another.
#pragma once

#include "sv_common.cuh"

namespace sv {

// Load the thread's U vectors of [seg_begin, seg_end); entries past seg_end
// read as -inf.  All loads are issued before any is consumed.
template <class Tag, int U>
__device__ __forceinline__ void load_segment(const char *row, int seg_begin, int seg_end,
                                             uint4 (&raw)[U])
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e0 = seg_begin + (threadIdx.x + u * kThreads) * kVec;
        raw[u] = e0 < seg_end ? ldg_vec(row + static_cast<int64_t>(e0) * kEsz)
                              : make_uint4(Tag::kNegInfWord, Tag::kNegInfWord, Tag::kNegInfWord,
                                           Tag::kNegInfWord);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int e0 = seg_begin + (threadIdx.x + u * kThreads) * kVec;
        if (e0 < seg_end && e0 + kVec > seg_end) raw[u] = mask_tail<Tag>(raw[u], seg_end - e0);
    }
}

// Segment softmax partial: M = max (NaN if any NaN), S = sum 2^((l - M) c)
// with c = log2(e)/T, i.e. sum exp((l - M)/T).  Valid in every thread.
template <class Tag, int U>
__device__ __forceinline__ float2 segment_softmax_partial(const uint4 (&raw)[U], float c,
                                                          float *red)
{
    constexpr int kVec = Tag::kVec;
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < U; ++u) m = max_nan(m, vec_max<Tag>(raw[u]));
    float s = 0.f;
    if (m != -INFINITY) {  // a NaN maximum enters too and poisons s
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float x[kVec];
            unpack<Tag>(raw[u], x);
#pragma unroll
            for (int e = 0; e < kVec; ++e) s += ex2_approx((x[e] - m) * c);
        }
    }
    const float M = block_max_nan(m, red);
    const float sr = (m == -INFINITY) ? 0.f : s * ex2_approx((m - M) * c);
    const float S = block_sum(sr, red);
    return make_float2(M, S);
}

// Argmax combine: larger value wins, ties go to the lower index.
__device__ __forceinline__ void argmax_take(float &bv, int &bi, float ov, int oi)
{
    if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
    }
}

// Segment argmax partial: (value, index as bits); value is NaN when the
// segment holds a NaN; index INT_MAX when every entry is -inf.
template <class Tag, int U>
__device__ __forceinline__ float2 segment_argmax_partial(const uint4 (&raw)[U], int seg_begin,
                                                         float *redf, int *redi)
{
    constexpr int kVec = Tag::kVec;
    float best = -INFINITY;
    int idx = INT_MAX;
    bool nan = false;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        float x[kVec];
        unpack<Tag>(raw[u], x);
        const int e0 = seg_begin + (threadIdx.x + u * kThreads) * kVec;
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            nan |= (x[e] != x[e]);
            if (x[e] > best) {
                best = x[e];
                idx = e0 + e;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(kFull, best, o);
        const int oi = __shfl_xor_sync(kFull, idx, o);
        argmax_take(best, idx, ov, oi);
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int any_nan = block_max(nan ? 1 : 0, redi);
    __syncthreads();  // every thread has read redi before it is reused
    if (lane == 0) {
        redf[warp] = best;
        redi[warp] = idx;
    }
    __syncthreads();
    float bv = redf[0];
    int bi = redi[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) argmax_take(bv, bi, redf[w], redi[w]);
    __syncthreads();
    return make_float2(any_nan ? __int_as_float(0x7FC00000) : bv, __int_as_float(bi));
}

// Does tree node `node` of request b have a child?  (Only those nodes'
// draft rows are read.)  Block-uniform result.
__device__ __forceinline__ bool node_has_child(const Params &p, int b, int node)
{
    const int32_t *pa = p.parents + static_cast<int64_t>(b) * p.N;
    int found = 0;
    for (int j = node + 1 + threadIdx.x; j < p.N; j += kThreads) found |= (__ldg(pa + j) == node);
    return __syncthreads_or(found) != 0;
}

}  // namespace sv
