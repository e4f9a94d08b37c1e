// sv_engine.cuh -- persistent verification engine (linear stochastic,
// tree stochastic, tree greedy).
//
// One kernel launch; every warp is an independent worker.
//
//  * Pass 1 (items of `seg` entries of one logit row, request-major order):
//    one streaming read of every row, moved by asynchronous copies into a
//    per-warp shared-memory ring kRing batches ahead of use.  Stochastic
//    modes reduce an item to (max, sum exp((l - max)/T)), three quarters of
//    the exponentials on the special-function unit and one quarter on the
//    FMA pipe; greedy trees reduce to (max, lowest argmax).  "Accelerating
//    Sonar through speculation", section "Target-Draft": acceptance compares
//    the full draft and target distributions, hence whole-vocabulary
//    normalisers.  The warp that completes the last item of a row merges the
//    row; the warp that merges the last row of a request runs the request's
//    decide step ("Speculative decoding explained", section "Draft and
//    verification loop"; section "EAGLE" of the Sonar post for trees) and
//    publishes its pass-2 work.
//  * Pass 2 (items of kSeg2 entries of the row, or row pair, the final draw
//    needs): fp64 weights.  For the residual norm(max(0, p_n - q_n)) one
//    pass yields both normalisers and the segment sums: an entry whose sign
//    of p - q is already decided by the fp32 ratio bounds goes into a
//    linear sum, the few undecided ones are marked in a bitmap and resolved
//    exactly once the fp64 normalisers are known.  Per-lane partial sums are
//    kept, so the warp that completes the last pass-2 item of a request
//    draws the token by inverse CDF (segment prefix, lane-chunk prefix,
//    entry) without recomputing the chosen segment.
//
// Warps [0, kP2Warps) of every block serve pass 2 from the start; the other
// warps stream pass 1 and join pass 2 when no pass-1 item is left.  Pass-1
// items are claimed with fetch-and-add; pass-2 items are claimed the same
// way as tickets in request order, and a ticket holder waits (bounded) until
// its request is decided.  A warp waits only while it holds no pass-1 item,
// and decide steps run on pass-1 workers, which never wait, so every ticket
// becomes serviceable.  On an expired wait the warp sets
// SPEC_STATUS_TIMEOUT and exits.  The asynchronous-copy waits are hardware
// waits on the thread's own copies.
#pragma once

#include "sv_common.cuh"
#include "sv_exp64.cuh"
#include "sv_philox.cuh"

namespace sv {

constexpr int kMaxNodes = 1024;
constexpr int kMaxLinearRows = 2 * 32 + 1;
// The fp32 normalisers of pass 1 are within a few 1e-6 of the fp64 ones;
// entries whose ratio e/f lies within this relative margin of the fp32
// estimate of S_t/S_d are resolved exactly after pass 2.
constexpr double kRhoMargin = 3e-5;
constexpr unsigned kIdleLimit = 1u << 21;  // polls of a waiting ticket holder (~ seconds)
constexpr int kAmbList = 64;               // undecided entries gathered per round
constexpr int kP2Warps = 2;                // pass-2 workers per block from the start
constexpr int kRing = 4;                   // pass-1 batches in flight per warp
constexpr int kSlot = 4 * 32;              // uint4 per ring slot (one warp batch)
constexpr unsigned kNoItem = 0xFFFFFFFFu;

// Dynamic shared memory of one engine block: one region per warp, the
// pass-1 ring of a pass-1 worker and afterwards its pass-2 staging area.
constexpr int kWarpRegion = kSlot * kRing;  // uint4 (8 KB)
constexpr size_t kRingBytes = sizeof(uint4) * kWarpRegion * kWarps;

template <class Tag>
struct Pass1Shape {
    static constexpr int kBatch = 32 * 4 * Tag::kVec;  // entries per warp batch
};

template <int MODE>
struct WarpScratch;
template <>
struct WarpScratch<kLinear> {
    double s[kMaxLinearRows];
    float m[kMaxLinearRows];
    int amb[kAmbList];
};
template <>
struct WarpScratch<kTreeStochastic> {
    short depth[kMaxNodes];
    unsigned char flag[kMaxNodes];  // 1 has child, 2 test passed, 4 accepted
    int amb[kAmbList];
};
template <>
struct WarpScratch<kTreeGreedy> {
    short depth[kMaxNodes];
    unsigned char flag[kMaxNodes];
    int amb[kAmbList];
};

// ------------------------------------------------------------ small helpers
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

__device__ __forceinline__ ReqInfo load_req(const ReqInfo *r)
{
    ReqInfo q;
    q.t_off = __ldcg(&r->t_off);
    q.d_off = __ldcg(&r->d_off);
    q.u = __ldcg(&r->u);
    q.rho_lo = __ldcg(&r->rho_lo);
    q.rho_hi = __ldcg(&r->rho_hi);
    q.mt = __ldcg(&r->mt);
    q.md = __ldcg(&r->md);
    q.mode = __ldcg(&r->mode);
    q.out_index = __ldcg(&r->out_index);
    return q;
}

__device__ __forceinline__ void store_req(ReqInfo *r, const ReqInfo &q)
{
    __stcg(&r->t_off, q.t_off);
    __stcg(&r->d_off, q.d_off);
    __stcg(&r->u, q.u);
    __stcg(&r->rho_lo, q.rho_lo);
    __stcg(&r->rho_hi, q.rho_hi);
    __stcg(&r->mt, q.mt);
    __stcg(&r->md, q.md);
    __stcg(&r->mode, q.mode);
    __stcg(&r->out_index, q.out_index);
}

__device__ __forceinline__ ReqInfo empty_req()
{
    ReqInfo q;
    q.t_off = 0;
    q.d_off = 0;
    q.u = 0.0;
    q.rho_lo = 0.0;
    q.rho_hi = 0.0;
    q.mt = 0.f;
    q.md = 0.f;
    q.mode = kModeNone;
    q.out_index = 0;
    return q;
}

// double4 through L2 as two double2 halves.
__device__ __forceinline__ double4 ldcg_d4(const double4 *p)
{
    const double2 a = __ldcg(reinterpret_cast<const double2 *>(p));
    const double2 b = __ldcg(reinterpret_cast<const double2 *>(p) + 1);
    return make_double4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void stcg_d4(double4 *p, double4 v)
{
    __stcg(reinterpret_cast<double2 *>(p), make_double2(v.x, v.y));
    __stcg(reinterpret_cast<double2 *>(p) + 1, make_double2(v.z, v.w));
}

// Exact fp64 value of one stored logit (integer widening, no conversion unit).
template <class Tag>
__device__ __forceinline__ double logit_f64(const uint4 &v, int e);
template <>
__device__ __forceinline__ double logit_f64<Bf16>(const uint4 &v, int e)
{
    const uint32_t w = (e >> 1) == 0 ? v.x : (e >> 1) == 1 ? v.y : (e >> 1) == 2 ? v.z : v.w;
    return bf16_to_f64((e & 1) ? (w >> 16) : (w & 0xFFFFu));
}
template <>
__device__ __forceinline__ double logit_f64<F32>(const uint4 &v, int e)
{
    const uint32_t w = e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
    return f32_to_f64(__uint_as_float(w));
}

template <class Tag>
__device__ __forceinline__ double logit_f64_at(const void *base, int64_t index)
{
    return f32_to_f64(load_logit<Tag>(base, index));
}

// Mark request b decided and move the decided frontier as far as it goes.
// Lane 0 only.  Bounded by B steps; never waits.
__device__ __forceinline__ void publish(const Params &p, int b)
{
    __threadfence();
    atomicExch(&p.decided[b], 1u);
    __threadfence();
    unsigned f = ld_volatile(&p.ctr->frontier);
    while (f < static_cast<unsigned>(p.B) && ld_volatile(&p.decided[f])) {
        const unsigned old = atomicCAS(&p.ctr->frontier, f, f + 1u);
        f = (old == f) ? f + 1u : old;
    }
}

__device__ __forceinline__ void request_done(const Params &p)
{
    __threadfence();
    atomicAdd(&p.ctr->finalized, 1u);
}

// The accept test in the log domain (no underflow): p == 0 rejects,
// q == 0 or p >= q accepts, u == 0 accepts, else log u + log q < log p.
__device__ __forceinline__ bool accept_test(double lp, double lq, double u)
{
    if (lp == -INFINITY) return false;
    if (lq == -INFINITY || lp >= lq) return true;
    if (u == 0.0) return true;
    return log(u) + lq < lp;
}

__device__ __forceinline__ bool stoch_row_ok(float m, double s)
{
    return isfinite(m) && isfinite(s) && s > 0.0;
}

// Release / acquire fences at GPU scope (lighter than a full sequentially
// consistent fence; enough to pass a partial result through a counter).
__device__ __forceinline__ void fence_acq_rel() { asm volatile("fence.acq_rel.gpu;\n" ::: "memory"); }

// Lane-0 "last arrival" on a counter: true (in every lane) for the warp
// that brings `counter` to `total`.  The warp's prior writes are made
// visible first; the last arriver sees everyone's.
__device__ __forceinline__ bool arrive(unsigned *counter, unsigned total)
{
    unsigned last = 0;
    if ((threadIdx.x & 31) == 0) {
        fence_acq_rel();
        last = (atomicAdd(counter, 1u) == total - 1u) ? 1u : 0u;
        if (last) fence_acq_rel();
    }
    return __shfl_sync(kFull, last, 0) != 0;
}

// The same arrival split in two: the counter update is issued now and its
// result read later, so the warp does not wait for the atomic's round trip.
struct Arrival {
    unsigned *counter;
    unsigned total;
    unsigned old;  // lane 0: the counter value before our increment
    bool pending;
};
__device__ __forceinline__ void arrive_issue(Arrival &a, unsigned *counter, unsigned total)
{
    a.counter = counter;
    a.total = total;
    a.pending = true;
    if ((threadIdx.x & 31) == 0) {
        fence_acq_rel();
        a.old = atomicAdd(counter, 1u);
    }
}
__device__ __forceinline__ bool arrive_result(Arrival &a)
{
    a.pending = false;
    unsigned last = 0;
    if ((threadIdx.x & 31) == 0) {
        last = (a.old == a.total - 1u) ? 1u : 0u;
        if (last) fence_acq_rel();
    }
    return __shfl_sync(kFull, last, 0) != 0;
}

__device__ __forceinline__ RowStat load_rowstat(const RowStat *r)
{
    RowStat st;
    st.m = __ldcg(&r->m);
    st.idx = __ldcg(&r->idx);
    st.s = __ldcg(&r->s);
    return st;
}

// ------------------------------------------------------------- row merge
// Merge the S pass-1 partials of row r of request b into rowstat[b][r].
// Stochastic rows: (max, sum exp((l - max)/T)), the partial sums rescaled
// on the FMA pipe and accumulated in fp64.  Greedy rows: (max, lowest
// argmax).  Whole warp; fixed order, so deterministic.
template <int MODE>
__device__ __forceinline__ void merge_row(const Params &p, int b, int r)
{
    const int lane = threadIdx.x & 31;
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
            else if (v.x != -INFINITY) argmax_take(bv, bi, v.x, __float_as_int(v.y));
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
        float m = -INFINITY;
        double s = 0.0;
        bool nan = false;
        for (int sg = lane; sg < p.S; sg += 32) {
            const float2 v = __ldcg(part + sg);
            if (v.x != v.x || v.y != v.y) {
                nan = true;
            } else if (v.x > m) {
                s = s * f32_to_f64(ex2_fma((m - v.x) * p.c)) + f32_to_f64(v.y);
                m = v.x;
            } else if (v.x != -INFINITY) {
                s += f32_to_f64(v.y) * f32_to_f64(ex2_fma((v.x - m) * p.c));
            }
        }
        const float M = warp_max_nan(m);
        const double sr = (m == -INFINITY) ? 0.0 : s * f32_to_f64(ex2_fma((m - M) * p.c));
        nan = __any_sync(kFull, nan);
        st.m = nan ? __int_as_float(0x7FC00000) : M;
        st.s = nan ? __longlong_as_double(0x7FF8000000000000ll) : warp_sum(sr);
    }
    if (lane == 0) {
        RowStat *dst = p.rowstat + static_cast<int64_t>(b) * p.R + r;
        __stcg(&dst->m, st.m);
        __stcg(&dst->idx, st.idx);
        __stcg(&dst->s, st.s);
    }
}

// ------------------------------------------------------------------ decide
template <class Tag>
__device__ __forceinline__ void decide_linear(const Params &p, int b, WarpScratch<kLinear> &sh)
{
    const int lane = threadIdx.x & 31;
    const int k = p.k, R = p.R;
    for (int r = lane; r < R; r += 32) {
        const RowStat st = load_rowstat(p.rowstat + static_cast<int64_t>(b) * R + r);
        sh.m[r] = st.m;
        sh.s[r] = st.s;
    }
    __syncwarp();

    bool bad_row = false;
    for (int r = lane; r < R; r += 32) bad_row |= !stoch_row_ok(sh.m[r], sh.s[r]);
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
        const double lt = logit_f64_at<Tag>(p.tl, (static_cast<int64_t>(b) * (k + 1) + lane) * p.stride + x);
        const double ld = logit_f64_at<Tag>(p.dl, (static_cast<int64_t>(b) * k + lane) * p.stride + x);
        const double lp = (lt - static_cast<double>(sh.m[lane])) * p.inv_t - log(sh.s[lane]);
        const double lq = (ld - static_cast<double>(sh.m[k + 1 + lane])) * p.inv_t - log(sh.s[k + 1 + lane]);
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
        ReqInfo info = empty_req();
        if (bits) {
            p.acc[b] = -1;
            report(p.status, bits);
        } else {
            p.acc[b] = n;
            info.mode = (n < k) ? kModeResidual : kModeTargetRow;
            info.t_off = (static_cast<int64_t>(b) * (k + 1) + n) * p.stride;
            info.mt = sh.m[n];
            if (n < k) {
                info.d_off = (static_cast<int64_t>(b) * k + n) * p.stride;
                info.md = sh.m[k + 1 + n];
                const double rho0 = sh.s[n] / sh.s[k + 1 + n];
                info.rho_lo = rho0 * (1.0 - kRhoMargin);
                info.rho_hi = rho0 * (1.0 + kRhoMargin);
            }
            info.u = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(n),
                                    kPurposeSample, p.offset);
            info.out_index = b * (k + 1) + n;
        }
        store_req(p.req + b, info);
        publish(p, b);
        if (bits) request_done(p);
    }
}

// Does tree node `node` of request b have a child?  Warp-wide.
__device__ __forceinline__ bool node_has_child(const Params &p, int b, int node)
{
    const int32_t *pa = p.parents + static_cast<int64_t>(b) * p.N;
    bool found = false;
    for (int j = node + 1 + static_cast<int>(threadIdx.x & 31); j < p.N; j += 32)
        found |= (__ldg(pa + j) == node);
    return __any_sync(kFull, found);
}

template <class Tag, int MODE>
__device__ __forceinline__ void decide_tree(const Params &p, int b, WarpScratch<MODE> &sh)
{
    const int lane = threadIdx.x & 31;
    const int N = p.N, R = p.R;
    const int32_t *pa = p.parents + static_cast<int64_t>(b) * N;
    const int32_t *tk = p.tokens + static_cast<int64_t>(b) * N;
    for (int i = lane; i < N; i += 32) sh.flag[i] = 0;
    __syncwarp();
    int err = 0;
    for (int i = lane; i < N; i += 32) {
        const int par = __ldg(pa + i);
        if (i == 0) {
            if (par != -1) err |= kStTree;
        } else if (par < 0 || par >= i) {
            err |= kStTree;
        } else {
            sh.flag[par] = 1;  // benign race: every writer stores 1
            const int t = __ldg(tk + i);
            if (t < 0 || t >= p.V) err |= kStToken;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) err |= __shfl_xor_sync(kFull, err, o);
    __syncwarp();
    if (lane == 0 && !(err & kStTree)) {
        sh.depth[0] = 0;
        for (int i = 1; i < N; ++i) {
            const int d = sh.depth[__ldg(pa + i)] + 1;
            sh.depth[i] = static_cast<short>(d);
            if (d > p.max_depth) err |= kStTree;
        }
    }
    err = __shfl_sync(kFull, err, 0);
    __syncwarp();

    // rows the mode reads must be usable: every target row, and the draft
    // rows of nodes with children
    const RowStat *rs = p.rowstat + static_cast<int64_t>(b) * R;
    bool bad = false;
    for (int r = lane; r < R; r += 32) {
        if (r >= N && !(sh.flag[r - N] & 1)) continue;
        const RowStat st = load_rowstat(rs + r);
        bad |= (MODE == kTreeGreedy) ? (st.m != st.m) : !stoch_row_ok(st.m, st.s);
    }
    if (__any_sync(kFull, bad)) err |= kStLogit;

    if (!err) {
        for (int i = 1 + lane; i < N; i += 32) {
            const int par = __ldg(pa + i), t = __ldg(tk + i);
            bool ok;
            if (MODE == kTreeGreedy) {
                ok = (t == __ldcg(&rs[par].idx));
            } else {
                const RowStat ts = load_rowstat(rs + par), ds = load_rowstat(rs + N + par);
                const int64_t off = (static_cast<int64_t>(b) * N + par) * p.stride + t;
                const double lp = (logit_f64_at<Tag>(p.tl, off) - static_cast<double>(ts.m)) * p.inv_t - log(ts.s);
                const double lq = (logit_f64_at<Tag>(p.dl, off) - static_cast<double>(ds.m)) * p.inv_t - log(ds.s);
                const double u = philox_uniform(p.seed, static_cast<uint32_t>(b),
                                                static_cast<uint32_t>(i - 1), kPurposeAccept, p.offset);
                ok = accept_test(lp, lq, u);
            }
            if (ok) sh.flag[i] |= 2;
        }
    }
    __syncwarp();
    if (lane != 0) return;

    const int W = p.max_depth + 1;
    int32_t *out = p.out + static_cast<int64_t>(b) * W;
    int32_t *path = p.path ? p.path + static_cast<int64_t>(b) * W : nullptr;
    for (int j = 0; j < W; ++j) {
        out[j] = -1;
        if (path) path[j] = -1;
    }
    ReqInfo info = empty_req();
    if (err) {
        p.acc[b] = -1;
        report(p.status, err);
        store_req(p.req + b, info);
        publish(p, b);
        request_done(p);
        return;
    }
    sh.flag[0] |= 4;
    int d = 0;
    for (int i = 1; i < N; ++i) {
        const bool a = (sh.flag[__ldg(pa + i)] & 4) && (sh.flag[i] & 2);
        if (a) {
            sh.flag[i] |= 4;
            if (sh.depth[i] > sh.depth[d]) d = i;
        }
    }
    const int D = sh.depth[d];
    for (int node = d; node != 0; node = __ldg(pa + node)) {
        out[sh.depth[node] - 1] = __ldg(tk + node);
        if (path) path[sh.depth[node]] = node;
    }
    if (path) path[0] = 0;
    p.acc[b] = D;
    if (MODE == kTreeGreedy) {
        out[D] = __ldcg(&rs[d].idx);
        store_req(p.req + b, info);
        publish(p, b);
        request_done(p);
    } else {
        info.mode = kModeTargetRow;
        info.t_off = (static_cast<int64_t>(b) * N + d) * p.stride;
        info.mt = __ldcg(&rs[d].m);
        info.u = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(d),
                                kPurposeSample, p.offset);
        info.out_index = b * W + D;
        store_req(p.req + b, info);
        publish(p, b);
    }
}

// ------------------------------------------------------------------ pass 1
// One pass-1 item: row, entry range and whether the row is read at all
// (draft rows of leaf tree nodes are not).
struct Item1 {
    const char *row;
    int b, r, s;
    int e_begin, e_end;
    bool active;
};

template <class Tag, int MODE>
__device__ __forceinline__ Item1 item1(const Params &p, unsigned item)
{
    constexpr int kEsz = sizeof(typename Tag::elem);
    Item1 it;
    it.b = static_cast<int>(fdiv(item, p.div_req));
    const unsigned rem = item - static_cast<unsigned>(it.b) * p.div_req.d;
    it.r = static_cast<int>(fdiv(rem, p.div_s));
    it.s = static_cast<int>(rem - static_cast<unsigned>(it.r) * p.div_s.d);
    it.e_begin = it.s * p.seg;
    it.e_end = min(p.V, it.e_begin + p.seg);
    it.active = true;
    const void *base;
    int64_t row;
    const int b = it.b, r = it.r;
    if (MODE == kLinear) {
        if (r <= p.k) {
            base = p.tl;
            row = static_cast<int64_t>(b) * (p.k + 1) + r;
        } else {
            base = p.dl;
            row = static_cast<int64_t>(b) * p.k + (r - p.k - 1);
        }
    } else if (r < p.N) {
        base = p.tl;
        row = static_cast<int64_t>(b) * p.N + r;
    } else {
        base = p.dl;
        row = static_cast<int64_t>(b) * p.N + (r - p.N);
        it.active = node_has_child(p, b, r - p.N);
    }
    it.row = static_cast<const char *>(base) + row * p.stride * kEsz;
    return it;
}

__device__ __forceinline__ void commit_copies() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

template <int N>
__device__ __forceinline__ void wait_copies()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Asynchronous copy of this lane's 4 vectors of one batch into its parts
// of a ring slot (vectors at or past e_end are not copied).
template <class Tag>
__device__ __forceinline__ void issue_batch(const Item1 &it, int batch, uint4 *slot)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    const int lane = threadIdx.x & 31;
    if (!it.active) return;
    const int base = it.e_begin + batch * Pass1Shape<Tag>::kBatch;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int e0 = base + (u * 32 + lane) * kVec;
        if (e0 < it.e_end) {
            const char *src = it.row + static_cast<int64_t>(e0) * kEsz;
            const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(slot + u * 32 + lane));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
        }
    }
}

// Per-lane running state of the item being reduced.
struct Acc1 {
    float m, sum;  // stochastic
    float best;    // greedy
    int idx;
    bool nan;
};

__device__ __forceinline__ void acc_reset(Acc1 &a)
{
    a.m = -INFINITY;
    a.sum = 0.f;
    a.best = -INFINITY;
    a.idx = INT_MAX;
    a.nan = false;
}

// Fold one batch (this lane's 4 vectors from the ring slot) into the lane state.
template <class Tag, int MODE>
__device__ __forceinline__ void fold_batch(const Params &p, const Item1 &it, int batch,
                                           const uint4 *slot, Acc1 &a)
{
    constexpr int kVec = Tag::kVec;
    const int lane = threadIdx.x & 31;
    if (!it.active) return;
    const int base = it.e_begin + batch * Pass1Shape<Tag>::kBatch;
    uint4 raw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int e0 = base + (u * 32 + lane) * kVec;
        if (e0 < it.e_end) {
            raw[u] = slot[u * 32 + lane];
            if (e0 + kVec > it.e_end) raw[u] = mask_tail<Tag>(raw[u], it.e_end - e0);
        } else {
            raw[u] = make_uint4(Tag::kNegInfWord, Tag::kNegInfWord, Tag::kNegInfWord, Tag::kNegInfWord);
        }
    }
    if (MODE == kTreeGreedy) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float x[kVec];
            unpack<Tag>(raw[u], x);
            const int e0 = base + (u * 32 + lane) * kVec;
#pragma unroll
            for (int e = 0; e < kVec; ++e) {
                a.nan |= (x[e] != x[e]);
                if (x[e] > a.best) {
                    a.best = x[e];
                    a.idx = e0 + e;
                }
            }
        }
    } else {
        const float c = p.c;
        float bm = -INFINITY;
#pragma unroll
        for (int u = 0; u < 4; ++u) bm = max_nan(bm, vec_max<Tag>(raw[u]));
        if (bm != bm) {
            a.nan = true;
        } else if (bm > a.m) {
            a.sum *= ex2_fma((a.m - bm) * c);
            a.m = bm;
        }
        if (a.m != -INFINITY) {
            // three vectors on the special-function unit, one on the FMA pipe
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float x[kVec];
                unpack<Tag>(raw[u], x);
#pragma unroll
                for (int e = 0; e < kVec; ++e)
                    a.sum += (u == 3) ? ex2_fma((x[e] - a.m) * c) : ex2_approx((x[e] - a.m) * c);
            }
        }
    }
}

// Finish a pass-1 item: warp-reduce, store the partial and issue its
// arrival on the row counter (resolved one item later, see settle_item).
template <class Tag, int MODE>
__device__ __forceinline__ void finish_item(const Params &p, const Item1 &it, const Acc1 &a,
                                            Arrival &arr)
{
    const int lane = threadIdx.x & 31;
    if (it.active) {
        float2 part;
        if (MODE == kTreeGreedy) {
            float best = a.best;
            int idx = a.idx;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(kFull, best, o);
                const int oi = __shfl_xor_sync(kFull, idx, o);
                argmax_take(best, idx, ov, oi);
            }
            const bool nan = __any_sync(kFull, a.nan);
            part = make_float2(nan ? __int_as_float(0x7FC00000) : best, __int_as_float(idx));
        } else {
            const float M = warp_max_nan(a.m);
            float sr = (a.m == -INFINITY) ? 0.f : a.sum * ex2_fma((a.m - M) * p.c);
            sr = warp_sum(sr);
            const bool nan = __any_sync(kFull, a.nan);
            part = make_float2(nan ? __int_as_float(0x7FC00000) : M, nan ? __int_as_float(0x7FC00000) : sr);
        }
        if (lane == 0) __stcg(p.rowpart + (static_cast<int64_t>(it.b) * p.R + it.r) * p.S + it.s, part);
    }
    arrive_issue(arr, &p.row_done[static_cast<int64_t>(it.b) * p.R + it.r], static_cast<unsigned>(p.S));
}

// Resolve a pending row arrival: the warp that completed a row merges it;
// the warp that merged the last row of a request decides.
template <class Tag, int MODE>
__device__ __forceinline__ void settle_item(const Params &p, const Item1 &it, Arrival &arr,
                                            WarpScratch<MODE> &sh)
{
    if (!arr.pending) return;
    if (arrive_result(arr)) {
        if (it.active) merge_row<MODE>(p, it.b, it.r);
        if (arrive(&p.a_done[it.b], static_cast<unsigned>(p.R))) {
            if constexpr (MODE == kLinear) decide_linear<Tag>(p, it.b, sh);
            else decide_tree<Tag, MODE>(p, it.b, sh);
        }
    }
}

// The pass-1 worker: one continuous stream of batches through a kRing-slot
// ring.  The producer side claims items one ahead (the claim for the item
// after next is in flight while the current one is copied), so copies run
// ahead across item boundaries.  Slot metadata stays in registers: the
// consumer loop is unrolled over the slots.
template <class Tag, int MODE>
__device__ __forceinline__ void pass1_worker(const Params &p, uint4 *ring, WarpScratch<MODE> &sh)
{
    const int lane = threadIdx.x & 31;
    const int nb = p.seg / Pass1Shape<Tag>::kBatch;

    unsigned c0 = 0, c1 = 0;
    if (lane == 0) {
        c0 = atomicAdd(&p.ctr->a_next, 1u);
        c1 = atomicAdd(&p.ctr->a_next, 1u);
    }
    c0 = __shfl_sync(kFull, c0, 0);
    unsigned claim = c1;  // lane 0: the id of the item after the producer's
    bool claim_ready = true;

    unsigned prod_id = c0;
    Item1 prod_it;
    if (prod_id < p.nA) prod_it = item1<Tag, MODE>(p, prod_id);
    else prod_id = kNoItem;
    int prod_b = 0;

    unsigned meta_id[kRing];
    int meta_b[kRing];

    auto produce = [&](int q) {
        if (prod_id != kNoItem) {
            issue_batch<Tag>(prod_it, prod_b, ring + q * kSlot);
            meta_id[q] = prod_id;
            meta_b[q] = prod_b;
            if (++prod_b == nb) {
                prod_b = 0;
                unsigned nid = __shfl_sync(kFull, claim, 0);
                (void)claim_ready;
                if (nid < p.nA) {
                    prod_id = nid;
                    prod_it = item1<Tag, MODE>(p, nid);
                    if (lane == 0) claim = atomicAdd(&p.ctr->a_next, 1u);
                } else {
                    prod_id = kNoItem;
                }
            }
        } else {
            meta_id[q] = kNoItem;
            meta_b[q] = 0;
        }
        commit_copies();
    };

#pragma unroll
    for (int q = 0; q < kRing; ++q) produce(q);

    unsigned cons_id = kNoItem;
    Item1 cons_it, done_it;
    Acc1 acc;
    acc_reset(acc);
    Arrival arr;
    arr.pending = false;
    bool done = false;
#pragma unroll 1
    while (!done) {
#pragma unroll
        for (int q = 0; q < kRing; ++q) {
            if (!done) {
                wait_copies<kRing - 1>();
                const unsigned id = meta_id[q];
                if (id == kNoItem) {
                    done = true;
                } else {
                    if (id != cons_id) {
                        cons_id = id;
                        cons_it = item1<Tag, MODE>(p, id);
                        acc_reset(acc);
                    }
                    fold_batch<Tag, MODE>(p, cons_it, meta_b[q], ring + q * kSlot, acc);
                    if (meta_b[q] == nb - 1) {
                        settle_item<Tag, MODE>(p, done_it, arr, sh);  // the previous item
                        finish_item<Tag, MODE>(p, cons_it, acc, arr);
                        done_it = cons_it;
                    }
                    produce(q);
                }
            }
        }
    }
    settle_item<Tag, MODE>(p, done_it, arr, sh);
    wait_copies<0>();
}

// ------------------------------------------------------------------ pass 2
struct Exp64 {
    double e, f;
};

// This lane's kLane2 contiguous entries of segment s2, staged into the
// warp's shared-memory region with asynchronous copies in 64-byte chunks
// per row and lane, two chunks in flight (the next chunk's copies run while
// the current one is evaluated), four entries at a time so that their
// exponentials overlap.  Calls `fn(index, x)` for every entry (entries at
// or past V give e = f = 0); warp-collective.  Each lane reads back only
// the vectors it copied.
template <class Tag, bool kResidual, class Fn>
__device__ __forceinline__ void for_lane_entries(const Params &p, const ReqInfo &info, int s2,
                                                 const Exp2Table &tab, uint4 *stage, Fn fn)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    constexpr int kCH = 64 / kEsz;      // entries per chunk (32 bf16, 16 fp32)
    constexpr int kNC = kLane2 / kCH;   // chunks per lane
    constexpr int kNVC = kCH / kVec;    // vectors per chunk and row (4)
    constexpr int kG = 4;
    const int lane = threadIdx.x & 31;
    const int base = s2 * kSeg2 + lane * kLane2;
    const char *trow = static_cast<const char *>(p.tl) + info.t_off * kEsz;
    const char *drow = static_cast<const char *>(p.dl) + info.d_off * kEsz;
    const double mt = static_cast<double>(info.mt), md = static_cast<double>(info.md);

    auto stage_chunk = [&](int c, int buf) {
#pragma unroll
        for (int v = 0; v < kNVC; ++v) {
            const int e0 = base + c * kCH + v * kVec;
            if (e0 < p.V) {
                const unsigned dt = static_cast<unsigned>(
                    __cvta_generic_to_shared(stage + ((buf * 2 + 0) * kNVC + v) * 32 + lane));
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dt),
                             "l"(trow + static_cast<int64_t>(e0) * kEsz) : "memory");
                if (kResidual) {
                    const unsigned dd = static_cast<unsigned>(
                        __cvta_generic_to_shared(stage + ((buf * 2 + 1) * kNVC + v) * 32 + lane));
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dd),
                                 "l"(drow + static_cast<int64_t>(e0) * kEsz) : "memory");
                }
            }
        }
        commit_copies();
    };

    stage_chunk(0, 0);
    if (kNC > 1) stage_chunk(1, 1);
    // a compact loop over groups of four entries keeps the hot code small
    constexpr int kGroupsPerChunk = kCH / kG;
#pragma unroll 1
    for (int c = 0; c < kNC; ++c) {
        if (c + 1 < kNC) wait_copies<1>();
        else wait_copies<0>();
        const int buf = c & 1;
#pragma unroll 1
        for (int gi = 0; gi < kGroupsPerChunk; ++gi) {
            const int e0 = base + c * kCH + gi * kG;
            const int v = (gi * kG) / kVec, sub = (gi * kG) % kVec;  // vector and first entry in it
            const uint4 tv = stage[((buf * 2 + 0) * kNVC + v) * 32 + lane];
            const uint4 dv = kResidual ? stage[((buf * 2 + 1) * kNVC + v) * 32 + lane] : make_uint4(0, 0, 0, 0);
            Exp64 x[kG];
#pragma unroll
            for (int e = 0; e < kG; ++e) {
                const bool valid = e0 + e < p.V;
                const double zt = valid ? (logit_f64<Tag>(tv, sub + e) - mt) * p.c64 : -INFINITY;
                x[e].e = exp2_fp64(zt, tab);
                x[e].f = 0.0;
                if (kResidual) {
                    const double zd = valid ? (logit_f64<Tag>(dv, sub + e) - md) * p.c64 : -INFINITY;
                    x[e].f = exp2_fp64(zd, tab);
                }
            }
#pragma unroll
            for (int e = 0; e < kG; ++e) fn(e0 + e, x[e]);
        }
        if (c + 2 < kNC) stage_chunk(c + 2, buf);
    }
}

// Exact weight of one entry.  residual: max(0, e/S_t - f/S_d); else e.
__device__ __forceinline__ double entry_weight(int mode, double inv_sp, double inv_sq, const Exp64 &x)
{
    if (mode == kModeResidual) {
        const double pp = x.e * inv_sp, qq = x.f * inv_sq;
        return pp > qq ? pp - qq : 0.0;
    }
    return x.e;
}

// Segment prefix over W[0..S2): with target < 0 returns the total Z;
// otherwise also finds the first segment with positive weight whose
// inclusive prefix exceeds target, and the prefix before it.  Warp-wide,
// fixed association order (the two calls see identical prefixes).
__device__ __forceinline__ double segment_prefix(const double *W, int S2, double target,
                                                 int &sstar, double &before)
{
    const int lane = threadIdx.x & 31;
    double carry = 0.0;
    sstar = -1;
    before = 0.0;
    int last_pos = -1;
    double last_before = 0.0;
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
            last_before = __shfl_sync(kFull, excl, l);
        }
        carry = __shfl_sync(kFull, incl, 31);
    }
    if (target >= 0.0 && sstar < 0) {  // rounding left no hit: the last positive segment
        sstar = last_pos;
        before = last_before;
    }
    return carry;
}

// Exact residual weight of one marked entry per lane (idx < 0: none).
// Warp-collective.
template <class Tag>
__device__ __forceinline__ double marked_weight(const Params &p, const ReqInfo &info, int idx,
                                                double inv_sp, double inv_sq, const Exp2Table &tab)
{
    double zt = -INFINITY, zd = -INFINITY;
    if (idx >= 0) {
        zt = (logit_f64_at<Tag>(p.tl, info.t_off + idx) - static_cast<double>(info.mt)) * p.c64;
        zd = (logit_f64_at<Tag>(p.dl, info.d_off + idx) - static_cast<double>(info.md)) * p.c64;
    }
    Exp64 x;
    x.e = exp2_fp64(zt, tab);
    x.f = exp2_fp64(zd, tab);
    return idx >= 0 ? entry_weight(kModeResidual, inv_sp, inv_sq, x) : 0.0;
}

// 2c: the warp that completes the last pass-2 item of request b draws its
// token.
template <class Tag>
__device__ __forceinline__ void finalize(const Params &p, int b, const ReqInfo &info,
                                      const Exp2Table &tab, int *amb_list, uint4 *stage)
{
    const int lane = threadIdx.x & 31;
    const int S2 = p.S2;
    const double4 *part = p.p2part + static_cast<int64_t>(b) * S2;
    const int *namb = p.p2amb + static_cast<int64_t>(b) * S2;
    const unsigned *bits = p.ambbits + static_cast<int64_t>(b) * p.W32;
    double *W = p.p2w + static_cast<int64_t>(b) * S2;
    int mode = info.mode;
    double inv_sp = 1.0, inv_sq = 1.0;
    bool exact_all = false;

    if (mode == kModeResidual) {
        double Sp = 0.0, Sq = 0.0;
        for (int s = lane; s < S2; s += 32) {
            const double4 v = ldcg_d4(part + s);
            Sp += v.x;
            Sq += v.y;
        }
        Sp = warp_sum(Sp);
        Sq = warp_sum(Sq);
        inv_sp = 1.0 / Sp;
        inv_sq = 1.0 / Sq;
        const double rho = Sp / Sq;
        exact_all = !(rho >= info.rho_lo && rho <= info.rho_hi);
        // decided entries: closed form per segment
        for (int s = lane; s < S2; s += 32) {
            const double4 v = ldcg_d4(part + s);
            const double w = v.z * inv_sp - v.w * inv_sq;
            __stcg(W + s, w > 0.0 ? w : 0.0);
        }
        __threadfence_block();
        __syncwarp();
        // undecided entries: exactly, per segment that has any
        for (int base0 = 0; base0 < S2; base0 += 32) {
            const int s = base0 + lane;
            const bool need = s < S2 && (exact_all || __ldcg(namb + s) > 0);
            unsigned todo = __ballot_sync(kFull, need);
            while (todo) {
                const int l = __ffs(todo) - 1;
                todo &= todo - 1;
                const int sg = base0 + l;
                const int nseg = exact_all ? kSeg2 : __ldcg(namb + sg);
                double add = 0.0;
                if (exact_all || nseg > kAmbList) {
                    for_lane_entries<Tag, true>(p, info, sg, tab, stage, [&](int, const Exp64 &x) {
                        add += entry_weight(kModeResidual, inv_sp, inv_sq, x);
                    });
                    add = warp_sum(add);
                    if (lane == 0) __stcg(W + sg, add);
                } else {
                    // gather the marked entries in increasing index order
                    const int word = (sg * kSeg2 + lane * kLane2) >> 5;
                    const unsigned b0 = word < p.W32 ? __ldcg(bits + word) : 0u;
                    const unsigned b1 = word + 1 < p.W32 ? __ldcg(bits + word + 1) : 0u;
                    const int cnt = __popc(b0) + __popc(b1);
                    int pos = cnt;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int n2 = __shfl_up_sync(kFull, pos, o);
                        if (lane >= o) pos += n2;
                    }
                    pos -= cnt;  // exclusive prefix
                    const int ebase = sg * kSeg2 + lane * kLane2;
                    unsigned m0 = b0, m1 = b1;
                    while (m0) {
                        const int bit = __ffs(m0) - 1;
                        m0 &= m0 - 1;
                        if (pos < kAmbList) amb_list[pos] = ebase + bit;
                        ++pos;
                    }
                    while (m1) {
                        const int bit = __ffs(m1) - 1;
                        m1 &= m1 - 1;
                        if (pos < kAmbList) amb_list[pos] = ebase + 32 + bit;
                        ++pos;
                    }
                    __syncwarp();
                    double w = marked_weight<Tag>(p, info, lane < nseg ? amb_list[lane] : -1,
                                                  inv_sp, inv_sq, tab);
                    if (nseg > 32)
                        w += marked_weight<Tag>(p, info, lane + 32 < nseg ? amb_list[lane + 32] : -1,
                                                inv_sp, inv_sq, tab);
                    add = warp_sum(w);
                    if (lane == 0) __stcg(W + sg, __ldcg(W + sg) + add);
                    __syncwarp();
                }
            }
        }
        __threadfence_block();
        __syncwarp();
        int d0;
        double d1;
        const double Z = segment_prefix(W, S2, -1.0, d0, d1);
        if (!(Z > 0.0)) {
            // residual mass vanished in rounding: draw from target row n
            mode = kModeTargetRow;
            exact_all = false;
            for (int s = lane; s < S2; s += 32) __stcg(W + s, ldcg_d4(part + s).x);
            __threadfence_block();
            __syncwarp();
        }
    } else {
        for (int s = lane; s < S2; s += 32) __stcg(W + s, ldcg_d4(part + s).x);
        __threadfence_block();
        __syncwarp();
    }

    int dummy;
    double dummy_before;
    const double Z = segment_prefix(W, S2, -1.0, dummy, dummy_before);
    const double target = info.u * Z;
    int sstar;
    double before;
    segment_prefix(W, S2, target, sstar, before);
    if (sstar < 0) sstar = 0;
    const double tseg = target - before;

    // lane chunks of the chosen segment, from the pass-2 per-lane partials
    double lane_sum;
    {
        const double2 pl = __ldcg(p.p2lane + (static_cast<int64_t>(b) * S2 + sstar) * 32 + lane);
        if (mode == kModeResidual) {
            if (exact_all) {
                lane_sum = 0.0;
                for_lane_entries<Tag, true>(p, info, sstar, tab, stage, [&](int, const Exp64 &x) {
                    lane_sum += entry_weight(kModeResidual, inv_sp, inv_sq, x);
                });
            } else {
                const double w = pl.x * inv_sp - pl.y * inv_sq;
                lane_sum = w > 0.0 ? w : 0.0;
                // this lane's marked entries, one per round
                const int word = (sstar * kSeg2 + lane * kLane2) >> 5;
                unsigned m0 = word < p.W32 ? __ldcg(bits + word) : 0u;
                unsigned m1 = word + 1 < p.W32 ? __ldcg(bits + word + 1) : 0u;
                const int ebase = sstar * kSeg2 + lane * kLane2;
                int rounds = __popc(m0) + __popc(m1);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) rounds = max(rounds, __shfl_xor_sync(kFull, rounds, o));
                for (int q = 0; q < rounds; ++q) {
                    int idx = -1;
                    if (m0) {
                        idx = ebase + __ffs(m0) - 1;
                        m0 &= m0 - 1;
                    } else if (m1) {
                        idx = ebase + 32 + __ffs(m1) - 1;
                        m1 &= m1 - 1;
                    }
                    lane_sum += marked_weight<Tag>(p, info, idx, inv_sp, inv_sq, tab);
                }
            }
        } else {
            lane_sum = pl.x;
        }
    }
    const double incl = warp_incl_scan(lane_sum);
    double excl = __shfl_up_sync(kFull, incl, 1);
    if (lane == 0) excl = 0.0;
    const unsigned hit = __ballot_sync(kFull, lane_sum > 0.0 && incl > tseg);
    int cl;
    if (hit) {
        cl = __ffs(hit) - 1;
    } else {
        const unsigned pos = __ballot_sync(kFull, lane_sum > 0.0);
        cl = pos ? 31 - __clz(pos) : 0;
    }
    const double tchunk = tseg - __shfl_sync(kFull, excl, cl);

    // entries of chunk cl: two per lane
    const int cbase = sstar * kSeg2 + cl * kLane2 + 2 * lane;
    double w2[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int idx = cbase + q;
        const bool valid = idx < p.V;
        double zt = -INFINITY, zd = -INFINITY;
        if (valid) {
            zt = (logit_f64_at<Tag>(p.tl, info.t_off + idx) - static_cast<double>(info.mt)) * p.c64;
            if (mode == kModeResidual)
                zd = (logit_f64_at<Tag>(p.dl, info.d_off + idx) - static_cast<double>(info.md)) * p.c64;
        }
        Exp64 x;
        x.e = exp2_fp64(zt, tab);
        x.f = exp2_fp64(zd, tab);
        w2[q] = valid ? entry_weight(mode, inv_sp, inv_sq, x) : 0.0;
    }
    const double psum = w2[0] + w2[1];
    const double pincl = warp_incl_scan(psum);
    double pexcl = __shfl_up_sync(kFull, pincl, 1);
    if (lane == 0) pexcl = 0.0;
    int cand = INT_MAX, lastpos = -1;
    double run = pexcl;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        run += w2[q];
        if (w2[q] > 0.0) {
            lastpos = cbase + q;
            if (cand == INT_MAX && run > tchunk) cand = cbase + q;
        }
    }
    cand = warp_min(cand);
    int token = cand;
    if (cand == INT_MAX) {
        token = warp_max(lastpos);
        if (token < 0) token = sstar * kSeg2 + cl * kLane2;
    }
    if (lane == 0) {
        p.out[info.out_index] = token;
        request_done(p);
    }
}

template <class Tag, int MODE>
__device__ __forceinline__ void p2_item(const Params &p, unsigned item, const Exp2Table &tab,
                                     WarpScratch<MODE> &sh, uint4 *stage)
{
    const int lane = threadIdx.x & 31;
    const int b = static_cast<int>(fdiv(item, p.div_s2));
    const int s2 = static_cast<int>(item - static_cast<unsigned>(b) * static_cast<unsigned>(p.S2));
    __threadfence();
    const ReqInfo info = load_req(p.req + b);
    if (info.mode == kModeNone) return;
    double E = 0.0, F = 0.0, A = 0.0, Bq = 0.0;
    int namb = 0;
    unsigned w0 = 0, w1 = 0;
    const int base = s2 * kSeg2 + lane * kLane2;
    if (info.mode == kModeResidual) {
        const double lo = info.rho_lo, hi = info.rho_hi;
        for_lane_entries<Tag, true>(p, info, s2, tab, stage, [&](int idx, const Exp64 &x) {
            E += x.e;
            F += x.f;
            if (x.e > hi * x.f) {
                A += x.e;
                Bq += x.f;
            } else if (x.e > lo * x.f) {
                const int bit = idx - base;
                if (bit < 32) w0 |= 1u << bit;
                else w1 |= 1u << (bit - 32);
                ++namb;
            }
        });
        const int word = base >> 5;
        unsigned *bits = p.ambbits + static_cast<int64_t>(b) * p.W32;
        if (word < p.W32) __stcg(bits + word, w0);
        if (word + 1 < p.W32) __stcg(bits + word + 1, w1);
    } else {
        for_lane_entries<Tag, false>(p, info, s2, tab, stage, [&](int, const Exp64 &x) { E += x.e; });
        A = E;
    }
    // per-lane partials (decided residual part, or the lane's weight sum)
    __stcg(p.p2lane + (static_cast<int64_t>(b) * p.S2 + s2) * 32 + lane, make_double2(A, Bq));
    E = warp_sum(E);
    F = warp_sum(F);
    A = warp_sum(A);
    Bq = warp_sum(Bq);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) namb += __shfl_xor_sync(kFull, namb, o);
    if (lane == 0) {
        const int64_t at = static_cast<int64_t>(b) * p.S2 + s2;
        stcg_d4(p.p2part + at, make_double4(E, F, A, Bq));
        __stcg(p.p2amb + at, namb);
    }
    if (arrive(&p.p2_done[b], static_cast<unsigned>(p.S2))) finalize<Tag>(p, b, info, tab, sh.amb, stage);
}

// ------------------------------------------------------------------ engine
template <class Tag, int MODE>
__global__ void __launch_bounds__(kThreads, 2) k_engine(const __grid_constant__ Params p)
{
    __shared__ WarpScratch<MODE> scratch[kWarps];
    extern __shared__ uint4 rings[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    WarpScratch<MODE> &sh = scratch[warp];
    Exp2Table tab;
    tab.lo = p.exp2tab[lane];
    tab.hi = p.exp2tab[lane + 32];

    uint4 *region = rings + warp * kWarpRegion;
    if (warp >= kP2Warps) pass1_worker<Tag, MODE>(p, region, sh);
    if (p.nP == 0) return;
    for (;;) {
        unsigned t = 0;
        if (lane == 0) t = atomicAdd(&p.ctr->p_head, 1u);
        t = __shfl_sync(kFull, t, 0);
        if (t >= p.nP) break;
        const unsigned need = fdiv(t, p.div_s2) + 1u;  // requests [0, need) decided
        int ok = 1;
        if (lane == 0) {
            unsigned spins = 0;
            unsigned ns = 32;
            while (ld_volatile(&p.ctr->frontier) < need) {
                if (++spins > kIdleLimit) {
                    ok = 0;
                    report(p.status, kStTimeout);
                    break;
                }
                __nanosleep(ns);
                ns = ns < 1024 ? ns * 2 : 1024;
            }
        }
        ok = __shfl_sync(kFull, ok, 0);
        if (!ok) break;
        p2_item<Tag, MODE>(p, t, tab, sh, region);
    }
}

}  // namespace sv
