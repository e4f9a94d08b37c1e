// shard.cu -- verification steps for a vocabulary split across ranks.
//
// "Accelerating Sonar through speculation", section "Draft-target
// schedule": the target runs tensor-parallel over a group of ranks (the draft
// on the group's leader).  With the output projection split by vocabulary,
// each rank holds columns [lo, hi) of every logit row.  The verification
// rule ("Speculative decoding explained", section "Draft and verification
// loop"; Leviathan et al.) needs whole-row normalisers and one draw per
// request, so the ranks exchange a few numbers per row:
//   1. spec_shard_row_stats   each rank: per row, the max and the sum of
//                             exp((l - max)/T) over its columns (greedy: the
//                             max and its lowest index), and the logits at the
//                             draft tokens it owns;
//   2. (all-gather)           every rank gets every rank's statistics;
//   3. spec_shard_decide       every rank: the same merge in rank order, the
//                             same accept tests, the same n (greedy:
//                             spec_shard_decide_greedy gives the whole output);
//   4. spec_shard_draw_sums    each rank: fp64 sums of the draw's rows over its
//                             columns -- first the normalisers, then (after an
//                             all-gather of those) the draw weights' mass;
//   5. (all-gather)           the masses;
//   6. spec_shard_draw_pick    the rank whose range of the running mass holds
//                             u * Z draws the token inside its columns;
//   7. (all-reduce max)       the token reaches every rank;
//   8. spec_shard_emit         writes it into the outputs.
// Collectives are the caller's (NCCL through torch.distributed in the
// package); these kernels only compute.  Everything is fp64 where the
// single-GPU path is, and every cross-rank sum runs in rank order, so every
// rank holds bit-identical values.
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "../../include/specverify.h"
#include "sv_common.cuh"
#include "sv_exp64.cuh"
#include "sv_philox.cuh"
#include "sv_verify.cuh"

namespace sv {
namespace {

constexpr int kShardMaxShards = 64;
constexpr int kDrawWords = 6;  // mode, n, target max, draft max, u, spare
constexpr int kShardThreads = 256;

// 2^(j/256), j = 0..255: the table of the fp64 exponential, passed by value.
struct Exp2Tab {
    double v[kExp2Tab];
};

struct ShardRows {
    const void *tl, *dl;
    int64_t stride;
    int B, k, lo, hi;
};

template <class Tag>
__device__ __forceinline__ const char *shard_row(const ShardRows &s, int b, int r)
{
    constexpr int kEsz = sizeof(typename Tag::elem);
    if (r <= s.k)
        return static_cast<const char *>(s.tl) + (static_cast<int64_t>(b) * (s.k + 1) + r) * s.stride * kEsz;
    return static_cast<const char *>(s.dl) + (static_cast<int64_t>(b) * s.k + (r - s.k - 1)) * s.stride * kEsz;
}

// One warp per row: the max (NaN if any NaN) and its lowest index over the
// rank's columns, and (stochastic) the fp64 sum of exp((l - max)/T).  The
// warp of target row j < k also records the logits at draft token j when
// this rank owns it (else NaN).
template <class Tag>
__global__ void __launch_bounds__(kShardThreads) k_shard_stats(ShardRows s, int R, const int32_t *tokens,
                                                               float c, float *rmax, double *rsum,
                                                               int32_t *rarg, float *probe)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    const int lane = threadIdx.x & 31;
    const int64_t g = (static_cast<int64_t>(blockIdx.x) * kShardThreads + threadIdx.x) >> 5;
    if (g >= static_cast<int64_t>(s.B) * R) return;
    const int b = static_cast<int>(g / R), r = static_cast<int>(g % R);
    const char *row = shard_row<Tag>(s, b, r);
    const int Vs = s.hi - s.lo;
    float best = -INFINITY;
    int idx = INT_MAX;
    bool nan = false;
    for (int e0 = lane * kVec; e0 < Vs; e0 += 32 * kVec) {
        uint4 v = ldg_vec(row + static_cast<int64_t>(e0) * kEsz);
        if (e0 + kVec > Vs) v = mask_tail<Tag>(v, Vs - e0);
        const float vm = vec_max<Tag>(v);
        if (!(vm <= best)) {
            if (vm != vm) {
                nan = true;
            } else {
                float x[kVec];
                unpack<Tag>(v, x);
                int first = kVec - 1;
#pragma unroll
                for (int e = kVec - 1; e >= 0; --e)
                    if (x[e] == vm) first = e;
                best = vm;
                idx = e0 + first;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(kFull, best, o);
        const int oi = __shfl_xor_sync(kFull, idx, o);
        argmax_take(best, idx, ov, oi);
    }
    nan = __any_sync(kFull, nan);
    const float M = nan ? __int_as_float(0x7FC00000) : best;
    if (rsum) {
        double sl = 0.0;
        if (!nan && M != -INFINITY) {
            for (int e0 = lane * kVec; e0 < Vs; e0 += 32 * kVec) {
                uint4 v = ldg_vec(row + static_cast<int64_t>(e0) * kEsz);
                if (e0 + kVec > Vs) v = mask_tail<Tag>(v, Vs - e0);
                float x[kVec];
                unpack<Tag>(v, x);
#pragma unroll
                for (int e = 0; e < kVec; ++e)
                    if (x[e] != -INFINITY) sl += static_cast<double>(ex2_approx((x[e] - M) * c));
            }
        }
        const double S = warp_sum(sl);
        if (lane == 0) rsum[g] = nan ? __longlong_as_double(0x7FF8000000000000ll) : S;
    }
    if (lane == 0) {
        rmax[g] = M;
        if (rarg) rarg[g] = (idx == INT_MAX) ? INT_MAX : s.lo + idx;
        if (probe && r < s.k) {
            const int x = __ldg(tokens + static_cast<int64_t>(b) * s.k + r);
            float lt = __int_as_float(0x7FC00000), ld = lt;
            if (x >= s.lo && x < s.hi) {
                lt = load_logit<Tag>(s.tl, (static_cast<int64_t>(b) * (s.k + 1) + r) * s.stride + (x - s.lo));
                ld = load_logit<Tag>(s.dl, (static_cast<int64_t>(b) * s.k + r) * s.stride + (x - s.lo));
            }
            probe[(static_cast<int64_t>(b) * s.k + r) * 2] = lt;
            probe[(static_cast<int64_t>(b) * s.k + r) * 2 + 1] = ld;
        }
    }
}

// Merge row r of request b over the W ranks, in rank order: the max (NaN if
// any rank saw a NaN) and sum_w s_w exp((m_w - M)/T).
__device__ __forceinline__ void merge_shards(const float *rmax, const double *rsum, int W, int B, int R, int b,
                                             int r, double inv_t, float &M, double &S)
{
    const int64_t per = static_cast<int64_t>(B) * R;
    const int64_t at = static_cast<int64_t>(b) * R + r;
    float m = -INFINITY;
    bool nan = false;
    for (int w = 0; w < W; ++w) {
        const float v = rmax[w * per + at];
        nan |= v != v;
        m = fmaxf(m, v);
    }
    double s = 0.0;
    if (!nan && m != -INFINITY)
        for (int w = 0; w < W; ++w) {
            const float v = rmax[w * per + at];
            const double sw = rsum[w * per + at];
            nan |= sw != sw;
            if (v != -INFINITY) s += sw * exp((static_cast<double>(v) - static_cast<double>(m)) * inv_t);
        }
    M = nan ? __int_as_float(0x7FC00000) : m;
    S = nan ? __longlong_as_double(0x7FF8000000000000ll) : s;
}

// One warp per request: the accept tests on the merged statistics, as
// decide_linear does on one GPU.
__global__ void __launch_bounds__(kShardThreads) k_shard_decide(const float *rmax, const double *rsum,
                                                                const float *probe, const int32_t *bounds,
                                                                int W, const int32_t *tokens, int B, int k,
                                                                int V, double inv_t, uint64_t seed,
                                                                uint32_t offset, int32_t *out, int32_t *acc,
                                                                double *draw, int32_t *status)
{
    __shared__ float sm[kShardThreads / 32][2 * SPEC_MAX_K + 1];
    __shared__ double ss[kShardThreads / 32][2 * SPEC_MAX_K + 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = blockIdx.x * (kShardThreads / 32) + warp;
    if (b >= B) return;
    const int R = 2 * k + 1;
    bool bad = false;
    for (int r = lane; r < R; r += 32) {
        float M;
        double S;
        merge_shards(rmax, rsum, W, B, R, b, r, inv_t, M, S);
        sm[warp][r] = M;
        ss[warp][r] = S;
        bad |= !stoch_row_ok(M, S);
    }
    bad = __any_sync(kFull, bad);
    __syncwarp();
    int x = -1;
    bool tok_ok = true;
    double lp = 0.0, lq = 0.0;
    if (lane < k) {
        x = __ldg(tokens + static_cast<int64_t>(b) * k + lane);
        tok_ok = x >= 0 && x < V;
        if (tok_ok) {
            int w = 0;
            while (w + 1 < W && x >= bounds[w + 1]) ++w;
            const float lt = probe[((static_cast<int64_t>(w) * B + b) * k + lane) * 2];
            const float ld = probe[((static_cast<int64_t>(w) * B + b) * k + lane) * 2 + 1];
            lp = (static_cast<double>(lt) - static_cast<double>(sm[warp][lane])) * inv_t - log(ss[warp][lane]);
            lq = (static_cast<double>(ld) - static_cast<double>(sm[warp][k + 1 + lane])) * inv_t -
                 log(ss[warp][k + 1 + lane]);
        }
    }
    const int bits = (__any_sync(kFull, !tok_ok) ? kStToken : 0) | (bad ? kStLogit : 0);
    bool ok = true;
    if (lane < k && !bits) {
        const double u = philox_uniform(seed, static_cast<uint32_t>(b), static_cast<uint32_t>(lane),
                                        kPurposeAccept, offset);
        ok = accept_test(lp, lq, u);
    }
    const unsigned rej = __ballot_sync(kFull, lane < k && !ok);
    const int n = rej ? __ffs(rej) - 1 : k;
    int32_t *o = out + static_cast<int64_t>(b) * (k + 1);
    for (int j = lane; j <= k; j += 32) o[j] = (!bits && j < n) ? x : -1;  // j < n implies j == lane
    if (lane == 0) {
        double *d = draw + static_cast<int64_t>(b) * kDrawWords;
        if (bits) {
            acc[b] = -1;
            report(status, bits);
            d[0] = kModeNone;
            d[1] = d[2] = d[3] = d[4] = d[5] = 0.0;
        } else {
            acc[b] = n;
            d[0] = n < k ? kModeResidual : kModeTargetRow;
            d[1] = n;
            d[2] = sm[warp][n];
            d[3] = n < k ? static_cast<double>(sm[warp][k + 1 + n]) : 0.0;
            d[4] = philox_uniform(seed, static_cast<uint32_t>(b), static_cast<uint32_t>(n), kPurposeSample, offset);
            d[5] = 0.0;
        }
    }
}

// One warp per request: greedy verification from the ranks' (max, lowest
// argmax) per target row, merged in rank order (ties to the lowest index).
__global__ void __launch_bounds__(kShardThreads) k_shard_decide_greedy(const float *rmax, const int32_t *rarg,
                                                                       int W, const int32_t *tokens, int B,
                                                                       int k, int V, int32_t *out,
                                                                       int32_t *acc, int32_t *status)
{
    __shared__ int g_sh[kShardThreads / 32][SPEC_MAX_K + 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = blockIdx.x * (kShardThreads / 32) + warp;
    if (b >= B) return;
    const int R = k + 1;
    const int64_t per = static_cast<int64_t>(B) * R;
    bool nan = false;
    for (int r = lane; r < R; r += 32) {
        float bv = -INFINITY;
        int bi = INT_MAX;
        for (int w = 0; w < W; ++w) {
            const float v = rmax[w * per + static_cast<int64_t>(b) * R + r];
            if (v != v) nan = true;
            else argmax_take(bv, bi, v, rarg[w * per + static_cast<int64_t>(b) * R + r]);
        }
        g_sh[warp][r] = bi == INT_MAX ? 0 : bi;  // an all -inf row: index 0
    }
    nan = __any_sync(kFull, nan);
    __syncwarp();
    int x = -1;
    bool tok_ok = true;
    if (lane < k) {
        x = __ldg(tokens + static_cast<int64_t>(b) * k + lane);
        tok_ok = x >= 0 && x < V;
    }
    const int bits = (__any_sync(kFull, !tok_ok) ? kStToken : 0) | (nan ? kStLogit : 0);
    const unsigned mism = __ballot_sync(kFull, lane < k && x != g_sh[warp][lane < k ? lane : 0]);
    const int n = mism ? __ffs(mism) - 1 : k;
    int32_t *o = out + static_cast<int64_t>(b) * (k + 1);
    for (int j = lane; j <= k; j += 32) o[j] = bits ? -1 : (j < n ? x : (j == n ? g_sh[warp][n] : -1));
    if (lane == 0) {
        acc[b] = bits ? -1 : n;
        report(status, bits);
    }
}

struct DrawInfo {
    int mode, n;
    double mt, md, u;
};

__device__ __forceinline__ DrawInfo load_draw(const double *draw, int b)
{
    const double *d = draw + static_cast<int64_t>(b) * kDrawWords;
    DrawInfo i;
    i.mode = static_cast<int>(d[0]);
    i.n = static_cast<int>(d[1]);
    i.mt = d[2];
    i.md = d[3];
    i.u = d[4];
    return i;
}

// Sum over ranks in rank order of part[w][b][which].
__device__ __forceinline__ double rank_sum(const double *part, int W, int B, int b, int which)
{
    double s = 0.0;
    for (int w = 0; w < W; ++w) s += part[(static_cast<int64_t>(w) * B + b) * 2 + which];
    return s;
}

// The draw weights of one entry: phase 0: (e, f); phase 1: (residual or e,
// e), residual = max(0, e/S_t - f/S_d).
struct DrawWeights {
    const double *tab;
    double nmt, nmd, c64, isp, isq;
    bool residual;
    __device__ __forceinline__ double e(float x) const { return exp2_fp64(fma(static_cast<double>(x), c64, nmt), tab); }
    __device__ __forceinline__ double f(float x) const { return exp2_fp64(fma(static_cast<double>(x), c64, nmd), tab); }
};

// This thread's contiguous columns of the rank's slice: [lo, hi), whole vectors.
template <class Tag>
__device__ __forceinline__ void thread_columns(int Vs, int &lo, int &hi)
{
    constexpr int kVec = Tag::kVec;
    const int per = ((Vs + kShardThreads - 1) / kShardThreads + kVec - 1) / kVec * kVec;
    lo = min(Vs, static_cast<int>(threadIdx.x) * per);
    hi = min(Vs, lo + per);
}

// Visit this thread's columns of the draw rows in index order: f(v, xt, xd).
template <class Tag, class F>
__device__ __forceinline__ void visit_columns(const ShardRows &s, int b, int n, bool two, int lo, int hi, F f)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    const int Vs = s.hi - s.lo;
    const char *trow = shard_row<Tag>(s, b, n);
    const char *drow = two ? shard_row<Tag>(s, b, s.k + 1 + n) : trow;
    for (int e0 = lo; e0 < hi; e0 += kVec) {
        uint4 tv = ldg_vec(trow + static_cast<int64_t>(e0) * kEsz);
        uint4 dv = two ? ldg_vec(drow + static_cast<int64_t>(e0) * kEsz) : tv;
        if (e0 + kVec > Vs) {
            tv = mask_tail<Tag>(tv, Vs - e0);
            dv = mask_tail<Tag>(dv, Vs - e0);
        }
        float xt[kVec], xd[kVec];
        unpack<Tag>(tv, xt);
        unpack<Tag>(dv, xd);
#pragma unroll
        for (int e = 0; e < kVec; ++e)
            if (!f(e0 + e, xt[e], xd[e])) return;
    }
}

// Block sum of per-thread values, warps in order (lane 0's butterfly value):
// the same on every rank for the same inputs.
__device__ __forceinline__ double block_sum(double v, double *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < kShardThreads / 32; ++w) t += scratch[w];
    __syncthreads();
    return t;
}

template <class Tag>
__device__ __forceinline__ DrawWeights make_weights(const DrawInfo &d, double c64, const double *tab,
                                                    const double *norm_part, int W, int B, int b)
{
    DrawWeights w;
    w.tab = tab;
    w.c64 = c64;
    w.nmt = -d.mt * c64;
    w.nmd = -d.md * c64;
    w.residual = d.mode == kModeResidual;
    w.isp = w.isq = 0.0;
    if (norm_part) {
        w.isp = 1.0 / rank_sum(norm_part, W, B, b, 0);
        w.isq = w.residual ? 1.0 / rank_sum(norm_part, W, B, b, 1) : 0.0;
    }
    return w;
}

// One block per request: the rank's fp64 sums of the draw rows.
// norm_part == NULL: (sum e, sum f); else (the draw mass, sum e).
template <class Tag>
__global__ void __launch_bounds__(kShardThreads) k_shard_sums(ShardRows s, const double *draw, double c64,
                                                              const double *norm_part, int W,
                                                              const __grid_constant__ Exp2Tab tabg,
                                                              double *sums)
{
    __shared__ double tab[kExp2Tab];
    __shared__ double scratch[kShardThreads / 32];
    for (int j = threadIdx.x; j < kExp2Tab; j += kShardThreads) tab[j] = tabg.v[j];
    __syncthreads();
    const int b = blockIdx.x;
    const DrawInfo d = load_draw(draw, b);
    double a = 0.0, e2 = 0.0;
    if (d.mode != kModeNone) {
        const DrawWeights w = make_weights<Tag>(d, c64, tab, norm_part, W, s.B, b);
        int lo, hi;
        thread_columns<Tag>(s.hi - s.lo, lo, hi);
        visit_columns<Tag>(s, b, d.n, w.residual, lo, hi, [&](int, float xt, float xd) {
            const double e = w.e(xt);
            if (!norm_part) {
                a += e;
                if (w.residual) e2 += w.f(xd);
            } else {
                if (w.residual) {
                    const double pp = e * w.isp, qq = w.f(xd) * w.isq;
                    a += pp > qq ? pp - qq : 0.0;
                } else {
                    a += e;
                }
                e2 += e;
            }
            return true;
        });
    }
    a = block_sum(a, scratch);
    e2 = block_sum(e2, scratch);
    if (threadIdx.x == 0) {
        sums[static_cast<int64_t>(b) * 2] = a;
        sums[static_cast<int64_t>(b) * 2 + 1] = e2;
    }
}

// One block per request: the rank that owns the running-mass range holding
// u * Z draws inside its columns (thread chunk, then entry); others give -1.
// A residual whose total mass vanished (rounding only) draws from the
// target row instead.
template <class Tag>
__global__ void __launch_bounds__(kShardThreads) k_shard_pick(ShardRows s, const double *draw, double c64,
                                                              const double *norm_part,
                                                              const double *mass_part, int W, int me,
                                                              const __grid_constant__ Exp2Tab tabg,
                                                              int32_t *token)
{
    __shared__ double tab[kExp2Tab];
    __shared__ double tsum[kShardThreads];
    __shared__ int sel;
    __shared__ double sel_before;
    for (int j = threadIdx.x; j < kExp2Tab; j += kShardThreads) tab[j] = tabg.v[j];
    __syncthreads();
    const int b = blockIdx.x;
    const DrawInfo d = load_draw(draw, b);
    if (d.mode == kModeNone) {
        if (threadIdx.x == 0) token[b] = -1;
        return;
    }
    DrawWeights w = make_weights<Tag>(d, c64, tab, norm_part, W, s.B, b);
    int which = 0;
    double Z = rank_sum(mass_part, W, s.B, b, 0);
    if (w.residual && !(Z > 0.0)) {  // the residual vanished in rounding: the target row
        which = 1;
        w.residual = false;
        Z = rank_sum(mass_part, W, s.B, b, 1);
    }
    const double target = d.u * Z;
    double run = 0.0, before = 0.0, last_before = 0.0;
    int owner = -1, last = -1;
    for (int r = 0; r < W; ++r) {
        const double m = mass_part[(static_cast<int64_t>(r) * s.B + b) * 2 + which];
        if (m > 0.0) {
            if (run + m > target) {
                owner = r;
                before = run;
                break;
            }
            last = r;
            last_before = run;
        }
        run += m;
    }
    if (owner < 0) {
        owner = last;
        before = last_before;
    }
    if (owner != me) {
        if (threadIdx.x == 0) token[b] = -1;
        return;
    }
    auto weight = [&](float xt, float xd) {
        const double e = w.e(xt);
        if (!w.residual) return e;
        const double pp = e * w.isp, qq = w.f(xd) * w.isq;
        return pp > qq ? pp - qq : 0.0;
    };
    int lo, hi;
    thread_columns<Tag>(s.hi - s.lo, lo, hi);
    double mine = 0.0;
    visit_columns<Tag>(s, b, d.n, w.residual, lo, hi, [&](int, float xt, float xd) {
        mine += weight(xt, xd);
        return true;
    });
    tsum[threadIdx.x] = mine;
    __syncthreads();
    if (threadIdx.x == 0) {
        const double tl = target - before;
        double r2 = 0.0, lb = 0.0;
        int t = -1, tlast = 0;
        for (int i = 0; i < kShardThreads; ++i) {
            const double v = tsum[i];
            if (v > 0.0) {
                if (r2 + v > tl) {
                    t = i;
                    lb = r2;
                    break;
                }
                tlast = i;
                lb = r2;
            }
            r2 += v;
        }
        sel = t < 0 ? tlast : t;
        sel_before = lb;
    }
    __syncthreads();
    if (static_cast<int>(threadIdx.x) == sel) {
        const double tt = target - before - sel_before;
        double r3 = 0.0;
        int tok = -1, lastp = lo;
        visit_columns<Tag>(s, b, d.n, w.residual, lo, hi, [&](int v, float xt, float xd) {
            const double wv = weight(xt, xd);
            if (wv > 0.0) {
                if (r3 + wv > tt) {
                    tok = v;
                    return false;
                }
                lastp = v;
            }
            r3 += wv;
            return true;
        });
        token[b] = s.lo + (tok < 0 ? lastp : tok);
    }
}

__global__ void k_shard_emit(const int32_t *token, const double *draw, int B, int k, int32_t *out)
{
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const DrawInfo d = load_draw(draw, b);
    if (d.mode != kModeNone) out[static_cast<int64_t>(b) * (k + 1) + d.n] = token[b];
}

// ------------------------------------------------------------ host side
int check_layout(spec_dtype_t dtype, int64_t stride, int lo, int hi)
{
    if (dtype != SPEC_F32 && dtype != SPEC_BF16) return SPEC_EINVAL;
    if (lo < 0 || hi <= lo || stride < hi - lo) return SPEC_EINVAL;
    if ((stride * (dtype == SPEC_BF16 ? 2 : 4)) % 16 != 0) return SPEC_EALIGN;
    return SPEC_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

Exp2Tab exp2_table()
{
    Exp2Tab t;
    for (int j = 0; j < kExp2Tab; ++j) t.v[j] = std::exp2(static_cast<double>(j) / kExp2Tab);
    return t;
}

int launched() { return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ECUDA; }

}  // namespace
}  // namespace sv

using namespace sv;

extern "C" int spec_shard_row_stats(const void *target_logits, const void *draft_logits, spec_dtype_t dtype,
                                    int64_t row_stride, const int32_t *draft_tokens, int batch, int k,
                                    int vocab_lo, int vocab_hi, float temperature, float *row_max,
                                    double *row_sum, int32_t *row_argmax, float *probe,
                                    cudaStream_t stream)
{
    if (batch < 0 || k < 1) return SPEC_EINVAL;
    if (k > SPEC_MAX_K) return SPEC_EUNSUPPORTED;
    const bool stoch = draft_logits != nullptr;
    if (stoch && (!(temperature > 0.f) || !(temperature < INFINITY))) return SPEC_EINVAL;
    int rc = check_layout(dtype, row_stride, vocab_lo, vocab_hi);
    if (rc != SPEC_OK) return rc;
    if (batch == 0) return SPEC_OK;
    if (!target_logits || !row_max || (stoch && (!row_sum || !probe || !draft_tokens)) ||
        (!stoch && !row_argmax))
        return SPEC_EINVAL;
    if (!aligned16(target_logits) || (stoch && !aligned16(draft_logits))) return SPEC_EALIGN;
    ShardRows s{target_logits, draft_logits, row_stride, batch, k, vocab_lo, vocab_hi};
    const int R = stoch ? 2 * k + 1 : k + 1;
    const int64_t warps = static_cast<int64_t>(batch) * R;
    const int64_t blocks = (warps * 32 + kShardThreads - 1) / kShardThreads;
    if (blocks > INT_MAX) return SPEC_EUNSUPPORTED;
    const float c = static_cast<float>(1.4426950408889634074 / static_cast<double>(temperature));
    if (dtype == SPEC_BF16)
        k_shard_stats<Bf16><<<static_cast<unsigned>(blocks), kShardThreads, 0, stream>>>(
            s, R, draft_tokens, c, row_max, stoch ? row_sum : nullptr, row_argmax, stoch ? probe : nullptr);
    else
        k_shard_stats<F32><<<static_cast<unsigned>(blocks), kShardThreads, 0, stream>>>(
            s, R, draft_tokens, c, row_max, stoch ? row_sum : nullptr, row_argmax, stoch ? probe : nullptr);
    return launched();
}

extern "C" int spec_shard_decide(const float *row_max_all, const double *row_sum_all, const float *probe_all,
                                 const int32_t *bounds, int shards, const int32_t *draft_tokens, int batch,
                                 int k, int vocab, float temperature, uint64_t seed, uint32_t offset,
                                 int32_t *out_tokens, int32_t *accepted_len, double *draw, int32_t *status,
                                 cudaStream_t stream)
{
    if (batch < 0 || k < 1 || vocab < 1 || shards < 1) return SPEC_EINVAL;
    if (k > SPEC_MAX_K || shards > kShardMaxShards) return SPEC_EUNSUPPORTED;
    if (!(temperature > 0.f) || !(temperature < INFINITY)) return SPEC_EINVAL;
    if (batch == 0) return SPEC_OK;
    if (!row_max_all || !row_sum_all || !probe_all || !bounds || !draft_tokens || !out_tokens ||
        !accepted_len || !draw)
        return SPEC_EINVAL;
    const int wpb = kShardThreads / 32;
    k_shard_decide<<<(batch + wpb - 1) / wpb, kShardThreads, 0, stream>>>(
        row_max_all, row_sum_all, probe_all, bounds, shards, draft_tokens, batch, k, vocab,
        1.0 / static_cast<double>(temperature), seed, offset, out_tokens, accepted_len, draw, status);
    return launched();
}

extern "C" int spec_shard_decide_greedy(const float *row_max_all, const int32_t *row_argmax_all, int shards,
                                        const int32_t *draft_tokens, int batch, int k, int vocab,
                                        int32_t *out_tokens, int32_t *accepted_len, int32_t *status,
                                        cudaStream_t stream)
{
    if (batch < 0 || k < 1 || vocab < 1 || shards < 1) return SPEC_EINVAL;
    if (k > SPEC_MAX_K || shards > kShardMaxShards) return SPEC_EUNSUPPORTED;
    if (batch == 0) return SPEC_OK;
    if (!row_max_all || !row_argmax_all || !draft_tokens || !out_tokens || !accepted_len) return SPEC_EINVAL;
    const int wpb = kShardThreads / 32;
    k_shard_decide_greedy<<<(batch + wpb - 1) / wpb, kShardThreads, 0, stream>>>(
        row_max_all, row_argmax_all, shards, draft_tokens, batch, k, vocab, out_tokens, accepted_len, status);
    return launched();
}

extern "C" int spec_shard_draw_sums(const void *target_logits, const void *draft_logits, spec_dtype_t dtype,
                                   int64_t row_stride, int batch, int k, int vocab_lo, int vocab_hi,
                                   float temperature, const double *draw, const double *norm_parts,
                                   int shards, double *sums, cudaStream_t stream)
{
    if (batch < 0 || k < 1 || shards < 1) return SPEC_EINVAL;
    if (k > SPEC_MAX_K || shards > kShardMaxShards) return SPEC_EUNSUPPORTED;
    if (!(temperature > 0.f) || !(temperature < INFINITY)) return SPEC_EINVAL;
    int rc = check_layout(dtype, row_stride, vocab_lo, vocab_hi);
    if (rc != SPEC_OK) return rc;
    if (batch == 0) return SPEC_OK;
    if (!target_logits || !draft_logits || !draw || !sums) return SPEC_EINVAL;
    if (!aligned16(target_logits) || !aligned16(draft_logits)) return SPEC_EALIGN;
    const Exp2Tab tab = exp2_table();
    ShardRows s{target_logits, draft_logits, row_stride, batch, k, vocab_lo, vocab_hi};
    const double c64 = 1.4426950408889634074 / static_cast<double>(temperature);
    if (dtype == SPEC_BF16)
        k_shard_sums<Bf16><<<batch, kShardThreads, 0, stream>>>(s, draw, c64, norm_parts, shards, tab, sums);
    else
        k_shard_sums<F32><<<batch, kShardThreads, 0, stream>>>(s, draw, c64, norm_parts, shards, tab, sums);
    return launched();
}

extern "C" int spec_shard_draw_pick(const void *target_logits, const void *draft_logits, spec_dtype_t dtype,
                                   int64_t row_stride, int batch, int k, int vocab_lo, int vocab_hi,
                                   float temperature, const double *draw, const double *norm_parts,
                                   const double *mass_parts, int shards, int shard_index, int32_t *token,
                                   cudaStream_t stream)
{
    if (batch < 0 || k < 1 || shards < 1 || shard_index < 0 || shard_index >= shards) return SPEC_EINVAL;
    if (k > SPEC_MAX_K || shards > kShardMaxShards) return SPEC_EUNSUPPORTED;
    if (!(temperature > 0.f) || !(temperature < INFINITY)) return SPEC_EINVAL;
    int rc = check_layout(dtype, row_stride, vocab_lo, vocab_hi);
    if (rc != SPEC_OK) return rc;
    if (batch == 0) return SPEC_OK;
    if (!target_logits || !draft_logits || !draw || !norm_parts || !mass_parts || !token) return SPEC_EINVAL;
    if (!aligned16(target_logits) || !aligned16(draft_logits)) return SPEC_EALIGN;
    const Exp2Tab tab = exp2_table();
    ShardRows s{target_logits, draft_logits, row_stride, batch, k, vocab_lo, vocab_hi};
    const double c64 = 1.4426950408889634074 / static_cast<double>(temperature);
    if (dtype == SPEC_BF16)
        k_shard_pick<Bf16><<<batch, kShardThreads, 0, stream>>>(s, draw, c64, norm_parts, mass_parts, shards,
                                                                shard_index, tab, token);
    else
        k_shard_pick<F32><<<batch, kShardThreads, 0, stream>>>(s, draw, c64, norm_parts, mass_parts, shards,
                                                               shard_index, tab, token);
    return launched();
}

extern "C" int spec_shard_emit(const int32_t *token, const double *draw, int batch, int k, int32_t *out_tokens,
                              cudaStream_t stream)
{
    if (batch < 0 || k < 1) return SPEC_EINVAL;
    if (k > SPEC_MAX_K) return SPEC_EUNSUPPORTED;
    if (batch == 0) return SPEC_OK;
    if (!token || !draw || !out_tokens) return SPEC_EINVAL;
    k_shard_emit<<<(batch + 255) / 256, 256, 0, stream>>>(token, draw, batch, k, out_tokens);
    return launched();
}
