// sv_decide.cuh -- per-request decide step, run by the last pass-1 block of
// the request.
//
// Linear mode ("Speculative decoding explained", section "Draft and
// verification loop"; Leviathan et al.): draft x_j is accepted when
// u_j * q_j(x_j) < p_j(x_j); n is the first rejected position (k if none).
// Tree mode ("Accelerating Sonar through speculation", section "EAGLE"):
// a node is accepted when its parent is and its own test passes; the deepest
// accepted node (lowest index on ties) ends the emitted path.
#pragma once

#include "sv_common.cuh"
#include "sv_philox.cuh"
#include "sv_stats.cuh"

namespace sv {

constexpr int kMaxNodes = 1024;

// The accept test in the log domain (no underflow): p == 0 rejects,
// q == 0 or p >= q accepts, u == 0 accepts, else log u + log q < log p.
__device__ __forceinline__ bool accept_test(double lp, double lq, double u)
{
    if (lp == -INFINITY) return false;
    if (lq == -INFINITY || lp >= lq) return true;
    if (u == 0.0) return true;
    return log(u) + lq < lp;
}

__device__ __forceinline__ bool stoch_row_ok(const RowStat &st)
{
    return isfinite(st.m) && isfinite(st.s) && st.s > 0.0;
}

// Merge the per-segment partials of every row of request b into
// rowstat[b][r] (one warp per row; fixed summation order).  Rows whose
// `skip` flag is set (draft rows of leaf tree nodes) are left untouched.
template <int MODE>
__device__ void merge_rows(const Params &p, int b, const unsigned char *skip)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int r = warp; r < p.R; r += kWarps) {
        if (skip && skip[r]) continue;
        const float2 *part = p.rowpart + (static_cast<int64_t>(b) * p.R + r) * p.S;
        RowStat st;
        st.s = 0.0;
        st.idx = 0;
        if (MODE == kTreeGreedy) {
            float bv = -INFINITY;
            int bi = INT_MAX;
            bool nan = false;
            for (int sg = lane; sg < p.S; sg += 32) {
                const float2 v = __ldcg(part + sg);
                if (v.x != v.x) nan = true;
                else argmax_take(bv, bi, v.x, __float_as_int(v.y));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(kFull, bv, o);
                const int oi = __shfl_xor_sync(kFull, bi, o);
                argmax_take(bv, bi, ov, oi);
            }
            nan = __any_sync(kFull, nan);
            st.m = nan ? __int_as_float(0x7FC00000) : bv;
            st.idx = (bi == INT_MAX) ? 0 : bi;  // an all -inf row: index 0
        } else {
            float M = -INFINITY;
            for (int sg = lane; sg < p.S; sg += 32) M = max_nan(M, __ldcg(part + sg).x);
            M = warp_max_nan(M);
            double S = 0.0;
            for (int sg = lane; sg < p.S; sg += 32) {
                const float2 v = __ldcg(part + sg);
                if (v.x != -INFINITY)
                    S += static_cast<double>(v.y) *
                         exp((static_cast<double>(v.x) - static_cast<double>(M)) * p.inv_t);
            }
            st.m = M;
            st.s = warp_sum(S);
        }
        if (lane == 0) p.rowstat[static_cast<int64_t>(b) * p.R + r] = st;
    }
    __syncthreads();
}

// ------------------------------------------------------------------ linear
template <class Tag>
__device__ void decide_linear(const Params &p, int b)
{
    merge_rows<kLinear>(p, b, nullptr);
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const int k = p.k, R = p.R;
    const RowStat *rs = p.rowstat + static_cast<int64_t>(b) * R;

    bool bad_row = false;
    for (int r = lane; r < R; r += 32) bad_row |= !stoch_row_ok(rs[r]);
    bad_row = __any_sync(kFull, bad_row);

    int x = -1;
    bool tok_ok = true;
    if (lane < k) {
        x = __ldg(p.tokens + static_cast<int64_t>(b) * k + lane);
        tok_ok = (x >= 0 && x < p.V);
    }
    const bool tok_bad = __any_sync(kFull, !tok_ok);
    const int bits = (tok_bad ? kStToken : 0) | (bad_row ? kStLogit : 0);

    bool acc = true;
    float lpf = __int_as_float(0x7FC00000), lqf = lpf;
    if (lane < k && !bits) {
        const RowStat ts = rs[lane], ds = rs[k + 1 + lane];
        const float lt = load_logit<Tag>(p.tl, (static_cast<int64_t>(b) * (k + 1) + lane) * p.stride + x);
        const float ld = load_logit<Tag>(p.dl, (static_cast<int64_t>(b) * k + lane) * p.stride + x);
        const double lp = (static_cast<double>(lt) - static_cast<double>(ts.m)) * p.inv_t - log(ts.s);
        const double lq = (static_cast<double>(ld) - static_cast<double>(ds.m)) * p.inv_t - log(ds.s);
        const double u = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(lane),
                                        kPurposeAccept, p.offset);
        acc = accept_test(lp, lq, u);
        lpf = static_cast<float>(lp);
        lqf = static_cast<float>(lq);
    }
    const unsigned rej = __ballot_sync(kFull, lane < k && !acc);
    const int n = rej ? __ffs(rej) - 1 : k;

    int32_t *out = p.out + static_cast<int64_t>(b) * (k + 1);
    if (lane < k) {
        if (p.dbg_lp) p.dbg_lp[static_cast<int64_t>(b) * k + lane] = lpf;
        if (p.dbg_lq) p.dbg_lq[static_cast<int64_t>(b) * k + lane] = lqf;
    }
    for (int j = lane; j <= k; j += 32) out[j] = (!bits && j < n) ? x : -1;  // j < n implies j == lane
    if (lane == 0) {
        ReqInfo info;
        info.t_off = 0;
        info.d_off = 0;
        info.u = 0.0;
        info.inv_sp = 0.0;
        info.inv_sq = 0.0;
        info.mt = 0.f;
        info.md = 0.f;
        info.out_index = 0;
        if (bits) {
            info.mode = kModeNone;
            p.acc[b] = -1;
            report(p.status, bits);
        } else {
            p.acc[b] = n;
            info.mode = (n < k) ? kModeResidual : kModeTargetRow;
            info.t_off = (static_cast<int64_t>(b) * (k + 1) + n) * p.stride;
            info.mt = rs[n].m;
            if (n < k) {
                info.d_off = (static_cast<int64_t>(b) * k + n) * p.stride;
                info.md = rs[k + 1 + n].m;
            }
            info.u = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(n),
                                    kPurposeSample, p.offset);
            info.out_index = b * (k + 1) + n;
        }
        p.req[b] = info;
    }
}

// -------------------------------------------------------------------- tree
template <class Tag, int MODE>
__device__ void decide_tree(const Params &p, int b)
{
    __shared__ short depth[kMaxNodes];
    __shared__ unsigned char has_child[kMaxNodes];
    __shared__ unsigned char skip[2 * kMaxNodes];
    __shared__ unsigned char test_ok[kMaxNodes];
    __shared__ unsigned char accepted[kMaxNodes];
    __shared__ int s_err;

    const int N = p.N, R = p.R, tid = threadIdx.x;
    const int32_t *pa = p.parents + static_cast<int64_t>(b) * N;
    const int32_t *tk = p.tokens + static_cast<int64_t>(b) * N;
    if (tid == 0) s_err = 0;
    for (int i = tid; i < N; i += kThreads) has_child[i] = 0;
    __syncthreads();
    int err = 0;
    for (int i = tid; i < N; i += kThreads) {
        const int par = __ldg(pa + i);
        if (i == 0) {
            if (par != -1) err |= kStTree;
        } else if (par < 0 || par >= i) {
            err |= kStTree;
        } else {
            has_child[par] = 1;
            const int t = __ldg(tk + i);
            if (t < 0 || t >= p.V) err |= kStToken;
        }
    }
    if (err) atomicOr(&s_err, err);
    __syncthreads();
    if (tid == 0 && !(s_err & kStTree)) {
        depth[0] = 0;
        int e = 0;
        for (int i = 1; i < N; ++i) {
            const int d = depth[__ldg(pa + i)] + 1;
            depth[i] = static_cast<short>(d);
            if (d > p.max_depth) e = kStTree;
        }
        s_err |= e;
    }
    for (int r = tid; r < R; r += kThreads) skip[r] = (r >= N) ? !has_child[r - N] : 0;
    __syncthreads();

    merge_rows<MODE>(p, b, skip);
    const RowStat *rs = p.rowstat + static_cast<int64_t>(b) * R;

    // rows the mode reads must be usable
    int bad = 0;
    for (int r = tid; r < R; r += kThreads) {
        if (skip[r]) continue;
        const RowStat st = rs[r];
        if (MODE == kTreeGreedy ? (st.m != st.m) : !stoch_row_ok(st)) bad = kStLogit;
    }
    if (bad) atomicOr(&s_err, bad);
    __syncthreads();
    const int bits = s_err;

    if (!bits) {
        for (int i = 1 + tid; i < N; i += kThreads) {
            const int par = __ldg(pa + i), t = __ldg(tk + i);
            bool ok;
            if (MODE == kTreeGreedy) {
                ok = (t == rs[par].idx);
            } else {
                const RowStat ts = rs[par], ds = rs[N + par];
                const int64_t off = (static_cast<int64_t>(b) * N + par) * p.stride + t;
                const double lp = (static_cast<double>(load_logit<Tag>(p.tl, off)) -
                                   static_cast<double>(ts.m)) * p.inv_t - log(ts.s);
                const double lq = (static_cast<double>(load_logit<Tag>(p.dl, off)) -
                                   static_cast<double>(ds.m)) * p.inv_t - log(ds.s);
                const double u = philox_uniform(p.seed, static_cast<uint32_t>(b),
                                                static_cast<uint32_t>(i - 1), kPurposeAccept,
                                                p.offset);
                ok = accept_test(lp, lq, u);
            }
            test_ok[i] = ok;
        }
    }
    __syncthreads();

    if (tid != 0) return;
    const int W = p.max_depth + 1;
    int32_t *out = p.out + static_cast<int64_t>(b) * W;
    int32_t *path = p.path ? p.path + static_cast<int64_t>(b) * W : nullptr;
    for (int j = 0; j < W; ++j) {
        out[j] = -1;
        if (path) path[j] = -1;
    }
    ReqInfo info;
    info.t_off = 0;
    info.d_off = 0;
    info.u = 0.0;
    info.inv_sp = 0.0;
    info.inv_sq = 0.0;
    info.mt = 0.f;
    info.md = 0.f;
    info.mode = kModeNone;
    info.out_index = 0;
    if (bits) {
        p.acc[b] = -1;
        report(p.status, bits);
        p.req[b] = info;
        return;
    }
    accepted[0] = 1;
    int d = 0;
    for (int i = 1; i < N; ++i) {
        const unsigned char a = accepted[__ldg(pa + i)] && test_ok[i];
        accepted[i] = a;
        if (a && depth[i] > depth[d]) d = i;
    }
    const int D = depth[d];
    for (int node = d; node != 0; node = __ldg(pa + node)) {
        out[depth[node] - 1] = __ldg(tk + node);
        if (path) path[depth[node]] = node;
    }
    if (path) path[0] = 0;
    p.acc[b] = D;
    if (MODE == kTreeGreedy) {
        out[D] = rs[d].idx;
    } else {
        info.mode = kModeTargetRow;
        info.t_off = (static_cast<int64_t>(b) * N + d) * p.stride;
        info.mt = rs[d].m;
        info.u = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(d),
                                kPurposeSample, p.offset);
        info.out_index = b * W + D;
    }
    p.req[b] = info;
}

}  // namespace sv
