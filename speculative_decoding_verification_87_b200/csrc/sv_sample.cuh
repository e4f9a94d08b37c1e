// sv_sample.cuh -- pass 2: the one row (or row pair) per request that the
// final sample needs, in fp64.
//
// Residual ("Speculative decoding explained", section "Draft and
// verification loop": a rejected draft is replaced by a token from an
// adjusted distribution; Leviathan et al.: norm(max(0, p_n - q_n))) and the
// bonus token ("Accelerating Sonar through speculation", section
// "Target-Draft": the target always yields one more set of logits after the
// accepted drafts), both by inverse CDF: the token is the smallest v whose
// running weight sum exceeds u times the total.
//
// Why fp64: with V ~ 1.3e5 buckets, an fp32 running sum misplaces u*Z by a
// sizeable fraction of a typical bucket.  Every weight here is
// exp((l - m)/T) evaluated in fp64 (and, for the residual, divided by fp64
// normalisers recomputed over the whole row), so the bucket edges agree with
// an fp64 reference to ~1e-13 of their width.
//
// 2a (residual only): per-segment fp64 sums of exp((l - m)/T) for target row
//    n and draft row n; the last block inverts the totals.
// 2b: per-segment fp64 weight totals; the last block of the request runs the
//    search (2c): segment prefix -> chosen segment -> block scan inside it.
#pragma once

#include "sv_common.cuh"

namespace sv {

// Weights of the thread's kPerThread2 contiguous entries of segment s2.
// Entries at or past V weigh 0.  Returns their sequential sum.
template <class Tag>
__device__ __forceinline__ double thread_weights(const Params &p, const ReqInfo &info, int mode,
                                                 int s2, double (&w)[kPerThread2])
{
    constexpr int kVec = Tag::kVec;
    constexpr int kNV = kPerThread2 / kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    const int base = s2 * kSeg2 + threadIdx.x * kPerThread2;
    const char *trow = static_cast<const char *>(p.tl) + info.t_off * kEsz;
    const char *drow = static_cast<const char *>(p.dl) + info.d_off * kEsz;
    uint4 tv[kNV], dv[kNV];
#pragma unroll
    for (int v = 0; v < kNV; ++v) {
        const int e0 = base + v * kVec;
        tv[v] = make_uint4(0, 0, 0, 0);
        dv[v] = make_uint4(0, 0, 0, 0);
        if (e0 < p.V) {
            tv[v] = ldg_vec(trow + static_cast<int64_t>(e0) * kEsz);
            if (mode == kModeResidual) dv[v] = ldg_vec(drow + static_cast<int64_t>(e0) * kEsz);
        }
    }
    const double mt = static_cast<double>(info.mt), md = static_cast<double>(info.md);
    double sum = 0.0;
#pragma unroll
    for (int v = 0; v < kNV; ++v) {
        float x[kVec], y[kVec];
        unpack<Tag>(tv[v], x);
        unpack<Tag>(dv[v], y);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            const int idx = base + v * kVec + e;
            double wv = 0.0;
            if (idx < p.V) {
                const double ep = exp((static_cast<double>(x[e]) - mt) * p.inv_t);
                if (mode == kModeResidual) {
                    const double eq = exp((static_cast<double>(y[e]) - md) * p.inv_t);
                    const double pp = ep * info.inv_sp, qq = eq * info.inv_sq;
                    wv = pp > qq ? pp - qq : 0.0;
                } else {
                    wv = ep;
                }
            }
            w[v * kVec + e] = wv;
            sum += wv;
        }
    }
    return sum;
}

__device__ __forceinline__ double warp_incl_scan(double v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double n = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Block exclusive scan of one double per thread.  Returns the exclusive
// prefix; `total` (every thread) is the last thread's prefix plus its value,
// i.e. exactly the largest running sum the search below can see.
__device__ __forceinline__ double block_excl_scan(double v, double &total, double *sh)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const double incl = warp_incl_scan(v);
    double wexcl = __shfl_up_sync(kFull, incl, 1);
    if (lane == 0) wexcl = 0.0;
    __syncthreads();
    if (lane == 31) sh[warp] = incl;
    __syncthreads();
    double woff = 0.0;
    for (int w = 0; w < warp; ++w) woff += sh[w];
    const double excl = woff + wexcl;
    __syncthreads();
    if (threadIdx.x == kThreads - 1) sh[kWarps] = excl + v;
    __syncthreads();
    total = sh[kWarps];
    return excl;
}

// 2a: fp64 normalisers of target row n and draft row n (residual requests).
template <class Tag>
__global__ void __launch_bounds__(kThreads) k_pass2a(const Params p)
{
    __shared__ double red[kWarps];
    const int b = blockIdx.x / p.S2, s2 = blockIdx.x % p.S2;
    const ReqInfo info = p.req[b];
    if (info.mode != kModeResidual) return;  // uniform over the request's blocks

    constexpr int kVec = Tag::kVec;
    constexpr int kNV = kPerThread2 / kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    const int base = s2 * kSeg2 + threadIdx.x * kPerThread2;
    const char *trow = static_cast<const char *>(p.tl) + info.t_off * kEsz;
    const char *drow = static_cast<const char *>(p.dl) + info.d_off * kEsz;
    uint4 tv[kNV], dv[kNV];
#pragma unroll
    for (int v = 0; v < kNV; ++v) {
        const int e0 = base + v * kVec;
        tv[v] = make_uint4(0, 0, 0, 0);
        dv[v] = make_uint4(0, 0, 0, 0);
        if (e0 < p.V) {
            tv[v] = ldg_vec(trow + static_cast<int64_t>(e0) * kEsz);
            dv[v] = ldg_vec(drow + static_cast<int64_t>(e0) * kEsz);
        }
    }
    const double mt = static_cast<double>(info.mt), md = static_cast<double>(info.md);
    double se = 0.0, sf = 0.0;
#pragma unroll
    for (int v = 0; v < kNV; ++v) {
        float x[kVec], y[kVec];
        unpack<Tag>(tv[v], x);
        unpack<Tag>(dv[v], y);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            if (base + v * kVec + e < p.V) {
                se += exp((static_cast<double>(x[e]) - mt) * p.inv_t);
                sf += exp((static_cast<double>(y[e]) - md) * p.inv_t);
            }
        }
    }
    se = block_sum(se, red);
    sf = block_sum(sf, red);
    if (threadIdx.x == 0) p.p2a[static_cast<int64_t>(b) * p.S2 + s2] = make_double2(se, sf);
    if (arrive_last(&p.cnt2a[b], static_cast<unsigned>(p.S2)) && threadIdx.x < 32) {
        const int lane = threadIdx.x;
        double E = 0.0, F = 0.0;
        for (int s = lane; s < p.S2; s += 32) {
            const double2 v = __ldcg(p.p2a + static_cast<int64_t>(b) * p.S2 + s);
            E += v.x;
            F += v.y;
        }
        E = warp_sum(E);
        F = warp_sum(F);
        if (lane == 0) {
            p.req[b].inv_sp = 1.0 / E;
            p.req[b].inv_sq = 1.0 / F;
        }
    }
}

// Segment prefix over W[0..S2): returns the total Z (pass `target` < 0) or
// finds the first segment whose inclusive prefix exceeds `target`, with the
// prefix before it.  Warp 0 only; fixed association order, so the prefix
// values are identical between the two passes.
__device__ __forceinline__ double segment_prefix(const double *W, int S2, double target,
                                                 int &sstar, double &before)
{
    const int lane = threadIdx.x & 31;
    double carry = 0.0;
    sstar = -1;
    before = 0.0;
    int last_pos = -1;
    for (int base0 = 0; base0 < S2; base0 += 32) {
        const int s = base0 + lane;
        const double w = s < S2 ? __ldcg(W + s) : 0.0;
        const double incl = warp_incl_scan(w) + carry;
        double excl = __shfl_up_sync(kFull, incl, 1);
        if (lane == 0) excl = carry;
        if (target >= 0.0 && sstar < 0) {
            const unsigned hit = __ballot_sync(kFull, s < S2 && w > 0.0 && incl > target);
            if (hit) {
                const int l = __ffs(hit) - 1;
                sstar = base0 + l;
                before = __shfl_sync(kFull, excl, l);
            }
        }
        const unsigned pos = __ballot_sync(kFull, s < S2 && w > 0.0);
        if (pos) {
            const int l = 31 - __clz(pos);
            last_pos = base0 + l;
            // prefix before the last positive segment, for the rounding fallback
            const double bl = __shfl_sync(kFull, excl, l);
            if (target >= 0.0 && sstar < 0) before = bl;
        }
        carry = __shfl_sync(kFull, incl, 31);
    }
    if (target >= 0.0 && sstar < 0) sstar = last_pos;  // rounding left no hit
    return carry;
}

// 2c: the last 2b block of request b draws its token.
template <class Tag>
__device__ void final_sample(const Params &p, int b, ReqInfo info)
{
    __shared__ double sh[kWarps + 1];
    __shared__ double s_target;
    __shared__ int s_seg, s_mode;
    __shared__ int ired[kWarps];
    double *W = p.p2b + static_cast<int64_t>(b) * p.S2;
    const int tid = threadIdx.x;

    if (tid < 32) {
        int dummy;
        double dummy_before;
        const double Z = segment_prefix(W, p.S2, -1.0, dummy, dummy_before);
        if (tid == 0) {
            s_target = Z;
            s_mode = info.mode;
        }
    }
    __syncthreads();
    if (s_mode == kModeResidual && !(s_target > 0.0)) {
        // the residual mass vanished in rounding: draw from target row n
        for (int s = 0; s < p.S2; ++s) {
            double w[kPerThread2];
            const double ts = thread_weights<Tag>(p, info, kModeTargetRow, s, w);
            double tot;
            block_excl_scan(ts, tot, sh);
            if (tid == 0) W[s] = tot;
        }
        __threadfence();
        __syncthreads();
        if (tid < 32) {
            int dummy;
            double dummy_before;
            const double Z = segment_prefix(W, p.S2, -1.0, dummy, dummy_before);
            if (tid == 0) {
                s_target = Z;
                s_mode = kModeTargetRow;
            }
        }
        __syncthreads();
    }
    const int mode = s_mode;
    if (tid < 32) {
        const double target = info.u * s_target;
        int sstar;
        double before;
        segment_prefix(W, p.S2, target, sstar, before);
        if (tid == 0) {
            s_seg = sstar < 0 ? 0 : sstar;
            s_target = target - before;
        }
    }
    __syncthreads();
    const int s2 = s_seg;
    const double tgt = s_target;
    double w[kPerThread2];
    const double ts = thread_weights<Tag>(p, info, mode, s2, w);
    double tot;
    const double excl = block_excl_scan(ts, tot, sh);
    const int base = s2 * kSeg2 + tid * kPerThread2;
    int hit = INT_MAX, last_pos = -1;
    double run = excl;
#pragma unroll
    for (int e = 0; e < kPerThread2; ++e) {
        run += w[e];
        if (w[e] > 0.0) {
            last_pos = base + e;
            if (hit == INT_MAX && run > tgt) hit = base + e;
        }
    }
    hit = block_min(hit, ired);
    int token = hit;
    if (hit == INT_MAX) {
        __syncthreads();
        token = block_max(last_pos, ired);  // rounding left no hit: last positive entry
        if (token < 0) token = 0;
    }
    if (tid == 0) p.out[info.out_index] = token;
}

// 2b: per-segment weight totals; the last block samples.
template <class Tag>
__global__ void __launch_bounds__(kThreads) k_pass2b(const Params p)
{
    __shared__ double sh[kWarps + 1];
    const int b = blockIdx.x / p.S2, s2 = blockIdx.x % p.S2;
    const ReqInfo info = p.req[b];
    if (info.mode == kModeNone) return;  // uniform over the request's blocks
    double w[kPerThread2];
    const double ts = thread_weights<Tag>(p, info, info.mode, s2, w);
    double tot;
    block_excl_scan(ts, tot, sh);
    if (threadIdx.x == 0) p.p2b[static_cast<int64_t>(b) * p.S2 + s2] = tot;
    if (arrive_last(&p.cnt2b[b], static_cast<unsigned>(p.S2))) final_sample<Tag>(p, b, info);
}

}  // namespace sv
