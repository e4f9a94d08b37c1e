// sv_verify.cuh -- the steps of stochastic and tree verification, and the
// four-kernel path of the tree modes (the linear mode runs the same steps
// in one kernel, sv_fused.cuh).
//
//  * Pass 1 (k_pass1): one streaming read of every row that a mode needs,
//    in items of 2048 bf16 (1024 fp32) entries of one row taken by warps in
//    static round robin and copied by asynchronous copies into a per-warp
//    shared-memory ring ahead of use.  Stochastic modes reduce an item to
//    (max, sum exp((l - max)/T)) with one special-function exponential per
//    entry; greedy trees reduce to (max, lowest argmax).  "Accelerating
//    Sonar through speculation", section "Target-Draft": acceptance
//    compares the full draft and target distributions, hence
//    whole-vocabulary normalisers.
//  * Decide (k_decide): one block per request merges its rows' partials
//    and runs the decide step ("Speculative decoding explained", section
//    "Draft and verification loop"; section "EAGLE" of the Sonar post for
//    trees).
//  * Pass 2 (k_pass2): items of kSeg2 entries of the row, or row pair, that
//    the final draw needs, in fp64.  For the residual norm(max(0, p_n - q_n))
//    one pass yields both normalisers and the segment sums: an entry whose
//    sign of p - q is already certain from its fp32 logits goes into a
//    linear sum, the few undecided ones are marked in a bitmap and resolved
//    exactly once the fp64 normalisers are known.  Per-lane partial sums
//    are kept for the draw.
//  * Finalize (k_finalize): one warp per request draws the token by inverse
//    CDF (segment, lane chunk, entry).
//
// Each kernel is a programmatic dependent of the one before: its blocks are
// scheduled as the previous grid's retire and start work once that grid
// has completed and its writes are visible.  The only waits are hardware
// waits (own asynchronous copies, the grid dependency).
#pragma once

#include <cooperative_groups.h>

#include "sv_common.cuh"
#include "sv_exp64.cuh"
#include "sv_philox.cuh"

namespace sv {

constexpr int kMaxNodes = 1024;
// The fp32 normalisers of pass 1 are within a few 1e-6 of the fp64 ones.
// An entry whose log2(e/f) lies within kLog2Margin (plus its own fp32
// rounding bound) of log2 of the pass-1 estimate of S_t/S_d is resolved
// exactly after pass 2; the exact ratio must then lie within 2^(+-kLog2Margin)
// of the estimate, else every entry is recomputed exactly.
constexpr double kLog2Margin = 4.3e-5;  // ~ log2(1 + 3e-5)
// Pass-2 staging: a lane's kLane2 entries of the row (and of the draft row),
// two buffers per warp (the next item is copied while one is reduced).
template <class Tag>
struct StageShape {
    static constexpr int kNV = kLane2 / Tag::kVec;  // vectors per lane and row
    static constexpr int kPerBuf = 2 * kNV * 32;    // uint4 per buffer
    static constexpr int kPerWarp = 2 * kPerBuf;
    static constexpr size_t kBytes = sizeof(uint4) * kPerWarp * kWarps;
};
// Segment weights of a finalize step live in shared memory up to this many
// segments per request (vocabularies up to kMaxS2Shared * kSeg2), else in
// the workspace.
constexpr int kMaxS2Shared = 1024;

// Shared memory of a decide block beside the row statistics (trees).
struct TreeScratch {
    int par[kMaxNodes];             // parents as given (checked in tree_prepare)
    int tok[kMaxNodes];
    short depth[kMaxNodes];
    unsigned char flag[kMaxNodes];  // 1 has child, 2 test passed
    int err;                        // status bits of the request
    int key;                        // deepest accepted node: depth << 11 | (kMaxNodes - 1 - node)
};
// The accept and sample uniforms of a stochastic tree's nodes.
struct TreeUniforms {
    double ua[kMaxNodes], us[kMaxNodes];
};
// The logits a stochastic tree's node tests read (target and draft row of
// the parent at the node's token), fetched before pass 1 completes.
struct TreeProbe {
    float lt[kMaxNodes], ld[kMaxNodes];
};

// ------------------------------------------------------------ small helpers

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
    q.kc = __ldcg(&r->kc);
    q.tcls = __ldcg(&r->tcls);
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
    __stcg(&r->kc, q.kc);
    __stcg(&r->tcls, q.tcls);
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
    q.kc = 0.f;
    q.tcls = 0.f;
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

template <class Tag>
__device__ __forceinline__ double logit_f64_at(const void *base, int64_t index)
{
    return f32_to_f64(load_logit<Tag>(base, index));
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

// ------------------------------------------------------------------ pass 1
// Items: one batch of one row, kVecL vectors of kVec entries per lane;
// a request's rows are [0, R) (linear: target rows 0..k, then draft rows
// k+1..2k; tree: target rows 0..N-1, then draft rows N..2N-1).  An item
// reduces to a partial (max, sum exp((l - max)/T)) or, for greedy trees,
// (max, lowest argmax), stored at rowpart[b][r][s].
template <class Tag>
struct Pass1Shape {
    static constexpr int kVecL = 8;                       // vectors per lane per item
    static constexpr int kItem = 32 * kVecL * Tag::kVec;  // entries per item
    static constexpr int kSlot = 32 * kVecL;              // uint4 per ring slot
};
constexpr int kRing1 = 3;  // ring slots per warp: one reduced, two in flight
constexpr size_t kRingBytes = sizeof(uint4) * kRing1 * 32 * 8 * kWarps;
constexpr unsigned kNoItem = 0xFFFFFFFFu;

struct Item1 {
    const char *row;
    int b, r, s;
    int e_begin, e_end;
    bool active;
};


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
__device__ __forceinline__ Item1 item1(const Params &p, unsigned item, bool check_active = true)
{
    constexpr int kEsz = sizeof(typename Tag::elem);
    Item1 it;
    it.b = static_cast<int>(fdiv(item, p.div_req));
    const unsigned rem = item - static_cast<unsigned>(it.b) * p.div_req.d;
    it.r = static_cast<int>(fdiv(rem, p.div_s));
    it.s = static_cast<int>(rem - static_cast<unsigned>(it.r) * p.div_s.d);
    it.e_begin = it.s * Pass1Shape<Tag>::kItem;
    it.e_end = min(p.V, it.e_begin + Pass1Shape<Tag>::kItem);
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
        if (check_active) it.active = node_has_child(p, b, r - p.N);
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

// Asynchronous copy of this lane's vectors of an item into a ring slot
// (vectors at or past e_end are not copied).
template <class Tag>
__device__ __forceinline__ void issue_item(const Item1 &it, uint4 *slot)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    const int lane = threadIdx.x & 31;
    if (!it.active) return;
    const char *src = it.row + static_cast<int64_t>(it.e_begin + lane * kVec) * kEsz;
    const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(slot + lane));
    if (it.e_begin + Pass1Shape<Tag>::kItem <= it.e_end) {
#pragma unroll
        for (int v = 0; v < Pass1Shape<Tag>::kVecL; ++v)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst + v * 512),
                         "l"(src + v * 32 * kVec * kEsz) : "memory");
        return;
    }
#pragma unroll
    for (int v = 0; v < Pass1Shape<Tag>::kVecL; ++v) {
        const int e0 = it.e_begin + (v * 32 + lane) * kVec;
        if (e0 < it.e_end)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst + v * 512),
                         "l"(src + v * 32 * kVec * kEsz) : "memory");
    }
}

// NaN-propagating max of this lane's vectors of an item.
template <class Tag>
__device__ __forceinline__ float lane_max(const uint4 (&raw)[Pass1Shape<Tag>::kVecL]);
template <>
__device__ __forceinline__ float lane_max<Bf16>(const uint4 (&raw)[Pass1Shape<Bf16>::kVecL])
{
    constexpr int kV = Pass1Shape<Bf16>::kVecL;
    __nv_bfloat162 m[kV];
#pragma unroll
    for (int v = 0; v < kV; ++v) {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw[v].x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&raw[v].y);
        const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162 *>(&raw[v].z);
        const __nv_bfloat162 d = *reinterpret_cast<const __nv_bfloat162 *>(&raw[v].w);
        m[v] = __hmax2_nan(__hmax2_nan(a, b), __hmax2_nan(c, d));
    }
#pragma unroll
    for (int w = kV / 2; w > 0; w >>= 1)
#pragma unroll
        for (int v = 0; v < w; ++v) m[v] = __hmax2_nan(m[v], m[v + w]);
    return max_nan(__low2float(m[0]), __high2float(m[0]));
}
template <>
__device__ __forceinline__ float lane_max<F32>(const uint4 (&raw)[Pass1Shape<F32>::kVecL])
{
    constexpr int kV = Pass1Shape<F32>::kVecL;
    float m[kV];
#pragma unroll
    for (int v = 0; v < kV; ++v) m[v] = vec_max<F32>(raw[v]);
#pragma unroll
    for (int w = kV / 2; w > 0; w >>= 1)
#pragma unroll
        for (int v = 0; v < w; ++v) m[v] = max_nan(m[v], m[v + w]);
    return m[0];
}

// Reduce one staged item (item id `item`, segment s of its row) and store
// its partial at rowpart[item] (= rowpart[b][r][s]).  Stochastic: each
// lane takes its own max m, then sums 2^(x c - fl(m c)): one FMA and one
// special-function exponential per entry, four independent sums; the lane
// sums are corrected by 2^(fl(m c) - m c) (the FMA residual gives the
// difference exactly) and rescaled to the warp max.
template <class Tag, int MODE>
__device__ __forceinline__ void reduce_item1(const Params &p, unsigned item, int s, const uint4 *slot)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kV = Pass1Shape<Tag>::kVecL;
    const int lane = threadIdx.x & 31;
    const int e_begin = s * Pass1Shape<Tag>::kItem;
    uint4 raw[kV];
    if (e_begin + Pass1Shape<Tag>::kItem <= p.V) {
#pragma unroll
        for (int v = 0; v < kV; ++v) raw[v] = slot[v * 32 + lane];
    } else {  // the ragged end of a row
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            const int e0 = e_begin + (v * 32 + lane) * kVec;
            raw[v] = e0 < p.V ? mask_tail<Tag>(slot[v * 32 + lane], p.V - e0)
                              : make_uint4(Tag::kNegInfWord, Tag::kNegInfWord, Tag::kNegInfWord,
                                           Tag::kNegInfWord);
        }
    }
    float2 part;
    if (MODE == kTreeGreedy) {
        // the item's max from packed maxima (NaN if any entry is NaN), then
        // the lowest index holding it: entry e of lane l's vector v is entry
        // (v * 32 + l) * kVec + e of the item, so the first vector round
        // with a hit, its lowest lane and that lane's first entry give it
        const float M = warp_max_nan(lane_max<Tag>(raw));
        int idx = INT_MAX;
        bool found = !(M == M && M != -INFINITY);  // NaN or all -inf: no search
        // fully unrolled with a warp-uniform guard (no break), so that raw[]
        // stays in registers
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            if (found) continue;
            const unsigned hit = __ballot_sync(kFull, vec_max<Tag>(raw[v]) == M);
            if (hit) {
                const int w = __ffs(hit) - 1;
                int first = 0;
                if (lane == w) {
                    float x[kVec];
                    unpack<Tag>(raw[v], x);
                    first = kVec - 1;
#pragma unroll
                    for (int e = kVec - 1; e >= 0; --e)
                        if (x[e] == M) first = e;
                }
                first = __shfl_sync(kFull, first, w);
                idx = e_begin + (v * 32 + w) * kVec + first;
                found = true;
            }
        }
        part = make_float2(M, __int_as_float(idx));
    } else {
        const float c = p.c;
        const float m = lane_max<Tag>(raw);
        const float mc = (m == -INFINITY) ? 0.f : m * c;  // all -inf: every term is 0
        const float nmc = -mc;
        // entries in pairs through the packed fp32x2 FMA and add: entry e
        // goes to sum e & 3 in index order, as four scalar sums would
        const unsigned long long c2 = f2_pack(c, c), n2 = f2_pack(nmc, nmc);
        unsigned long long acc2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            float x[kVec];
            unpack<Tag>(raw[v], x);
#pragma unroll
            for (int e = 0; e < kVec; e += 2) {
                float z0, z1;
                f2_unpack(f2_fma(f2_pack(x[e], x[e + 1]), c2, n2), z0, z1);
                acc2[(e >> 1) & 1] = f2_add(acc2[(e >> 1) & 1], f2_pack(ex2_approx(z0), ex2_approx(z1)));
            }
        }
        float acc[4];
        f2_unpack(acc2[0], acc[0], acc[1]);
        f2_unpack(acc2[1], acc[2], acc[3]);
        const float lsum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        const float M = warp_max_nan(m);
        float sr = 0.f;
        if (m != -INFINITY) {
            const float d = -fmaf(m, c, nmc);  // fl(m c) - m c, exactly
            sr = lsum * ex2_approx((m - M) * c) * fmaf(d, 0.693147180559945309f, 1.0f);
        }
        sr = warp_sum(sr);
        part = make_float2(M, sr);
    }
    if (lane == 0 && !p.diag_no_partials) __stcg(p.rowpart + item, part);
}

// The pass-1 worker.  Items [0, nAs) are taken in static round robin (warp
// w of W takes w, w + W, ...: items are equal, so this balances them
// without a shared counter); the rest, in chunks of kDynChunk consecutive
// items from a counter (a_claim, all ones at the start of a call), claimed
// one chunk ahead just before the warp needs it, so that the SMs that run
// faster take more of the tail.  Items are copied into a kRing1-slot ring
// kRing1 - 1 items ahead of their reduction; lane q holds the item of slot
// q (kNoItem: the sequence ended) and whether it is read at all (tree
// draft rows of leaves are not), so the loop body exists once with a
// rotating slot index.
constexpr unsigned kDynChunk = 4;
template <class Tag, int MODE>
__device__ __forceinline__ void pass1_stream(const Params &p, uint4 *ring, unsigned w, unsigned W)
{
    constexpr int kSlot = Pass1Shape<Tag>::kSlot;
    const int lane = threadIdx.x & 31;
    unsigned st = w;                  // next static item
    unsigned dyn = 0, dyn_end = 0;    // current claimed chunk
    unsigned claim = 0;               // lane 0: the chunk claimed ahead
    bool claimed = false, done = false;
    auto claim_ahead = [&]() {
        if (lane == 0) claim = atomicAdd(p.a_claim, 1u) + 1u;  // the counter starts at all ones
        claimed = true;
    };
    auto next_item = [&]() -> unsigned {
        if (st < p.nAs) {
            const unsigned it = st;
            st += W;
            if (st >= p.nAs) claim_ahead();  // the next item comes from a claim
            return it;
        }
        if (dyn == dyn_end) {
            if (!claimed) claim_ahead();
            const unsigned c = __shfl_sync(kFull, claim, 0);
            claimed = false;
            const unsigned first = p.nAs + kDynChunk * c;
            if (c >= (p.nA - p.nAs + kDynChunk - 1) / kDynChunk || first >= p.nA) {
                done = true;
                return kNoItem;
            }
            dyn = first;
            dyn_end = min(first + kDynChunk, p.nA);
            claim_ahead();
        }
        return dyn++;
    };
    unsigned meta = kNoItem;
    bool act = true;
    auto refill = [&](int q) {
        const unsigned it = done ? kNoItem : next_item();
        bool a = false;
        if (it != kNoItem) {
            const Item1 i1 = item1<Tag, MODE>(p, it, MODE != kLinear);
            issue_item<Tag>(i1, ring + q * kSlot);
            a = i1.active;
        }
        if (lane == q) {
            meta = it;
            act = a;
        }
        commit_copies();
    };
#pragma unroll 1
    for (int q = 0; q < kRing1; ++q) refill(q);
    int q = 0;
#pragma unroll 1
    for (;;) {
        wait_copies<kRing1 - 1>();
        const unsigned it = __shfl_sync(kFull, meta, q);
        if (it == kNoItem) break;
        if (MODE == kLinear || __shfl_sync(kFull, act ? 1 : 0, q)) {
            const int s = static_cast<int>(it - fdiv(it, p.div_s) * static_cast<unsigned>(p.S));
            reduce_item1<Tag, MODE>(p, it, s, ring + q * kSlot);
        }
        refill(q);
        q = (q + 1 == kRing1) ? 0 : q + 1;
    }
    wait_copies<0>();
}

// ------------------------------------------------------------- row merge
// Merged statistics of a request's rows, in the decide block's shared
// memory: max (NaN if a NaN was read), sum exp((l - max)/T) (stochastic)
// or lowest argmax (greedy).
struct RowStats {
    double *s;
    float *m;
    int *idx;
};

// Merge the S pass-1 partials of row r of request b.  Stochastic rows: the
// partial sums rescaled on the FMA pipe and accumulated in fp64.  Greedy
// rows: (max, lowest argmax).  One warp; fixed order, so deterministic.
template <int MODE>
__device__ __forceinline__ void merge_row(const Params &p, int b, int r, RowStats rs,
                                          const float2 *staged = nullptr, int rbase = 0)
{
    const int lane = threadIdx.x & 31;
    // the row's partials: in global memory, or staged in shared memory
    // (rows from rbase on)
    const float2 *part = staged ? staged + static_cast<int64_t>(r - rbase) * p.S
                                : p.rowpart + (static_cast<int64_t>(b) * p.R + r) * p.S;
    if (MODE == kTreeGreedy) {
        float bv = -INFINITY;
        int bi = INT_MAX;
        bool nan = false;
        for (int sg = lane; sg < p.S; sg += 32) {
            const float2 v = staged ? part[sg] : __ldcg(part + sg);
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
        if (lane == 0) {
            rs.m[r] = nan ? __int_as_float(0x7FC00000) : bv;
            rs.idx[r] = (bi == INT_MAX) ? 0 : bi;  // an all -inf row: index 0
            rs.s[r] = 0.0;
        }
    } else {
        float m = -INFINITY;
        double s = 0.0;
        bool nan = false;
        for (int sg = lane; sg < p.S; sg += 32) {
            const float2 v = staged ? part[sg] : __ldcg(part + sg);
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
        const double S = warp_sum(sr);
        if (lane == 0) {
            rs.m[r] = nan ? __int_as_float(0x7FC00000) : M;
            rs.s[r] = nan ? __longlong_as_double(0x7FF8000000000000ll) : S;
        }
    }
}

// ------------------------------------------------------------------ decide
// Lane j < k of warp 0 has read the draft token x_j and the target and
// draft logits at x_j (inputs, so read before pass 1 completes).
struct DraftProbe {
    int x;
    float lt, ld;
};

template <class Tag>
__device__ __forceinline__ DraftProbe probe_drafts(const Params &p, int b)
{
    const int lane = threadIdx.x & 31;
    DraftProbe d;
    d.x = -1;
    d.lt = d.ld = 0.f;
    if (b < p.B && lane < p.k) {
        d.x = __ldg(p.tokens + static_cast<int64_t>(b) * p.k + lane);
        if (d.x >= 0 && d.x < p.V) {
            d.lt = load_logit<Tag>(p.tl, (static_cast<int64_t>(b) * (p.k + 1) + lane) * p.stride + d.x);
            d.ld = load_logit<Tag>(p.dl, (static_cast<int64_t>(b) * p.k + lane) * p.stride + d.x);
        }
    }
    return d;
}

template <class Tag>
__device__ __forceinline__ void decide_linear(const Params &p, int b, RowStats sh, const DraftProbe &pr)
{
    const int lane = threadIdx.x & 31;
    const int k = p.k, R = p.R;

    bool bad_row = false;
    for (int r = lane; r < R; r += 32) bad_row |= !stoch_row_ok(sh.m[r], sh.s[r]);
    bad_row = __any_sync(kFull, bad_row);
    int x = -1;
    bool tok_ok = true;
    if (lane < k) {
        x = pr.x;
        tok_ok = (x >= 0 && x < p.V);
    }
    const bool tok_bad = __any_sync(kFull, !tok_ok);
    const int bits = (tok_bad ? kStToken : 0) | (bad_row ? kStLogit : 0);

    bool acc = true;
    float lpf = __int_as_float(0x7FC00000), lqf = lpf;
    if (lane < k && !bits) {
        const double lt = f32_to_f64(pr.lt);
        const double ld = f32_to_f64(pr.ld);
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
                info.rho_lo = rho0 * exp2(-kLog2Margin);
                info.rho_hi = rho0 * exp2(kLog2Margin);
                const double kc = (static_cast<double>(info.mt) - static_cast<double>(info.md)) * p.c64 + log2(rho0);
                info.kc = static_cast<float>(kc);
                // |dz - true| <= 2^-21 (|dz| + |kc|) (fp32 roundings, with a
                // factor-2 margin): dz > tcls implies a true value above
                // kLog2Margin; rounded up
                constexpr double k21 = 4.76837158203125e-7;
                info.tcls = static_cast<float>((kLog2Margin + k21 * fabs(kc)) / (1.0 - k21) * (1.0 + 1e-6));
            }
            info.u = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(n),
                                    kPurposeSample, p.offset);
            info.out_index = b * (k + 1) + n;
        }
        store_req(p.req + b, info);
    }
}


constexpr int kDecideThreads = 1024;

// The tree decide step of request b, in two parts run by every thread of
// the decide block.
//
// tree_prepare reads only inputs, so it runs before pass 1 completes: the
// parents and tokens (into shared memory), the structural checks (root,
// parents before children, tokens in range), which nodes have children,
// every node's depth (a walk up its parents, at most max_depth + 1 steps;
// a node still short of the root is too deep), and for stochastic trees
// the logits each node test reads and the Philox uniforms of every test
// and of every possible draw.
template <class Tag, int MODE>
__device__ __forceinline__ void tree_prepare(const Params &p, int b, TreeScratch &ts, TreeProbe &tp,
                                             TreeUniforms &tu)
{
    constexpr int kT = kDecideThreads;
    const int N = p.N, tid = threadIdx.x;
    const int32_t *pa = p.parents + static_cast<int64_t>(b) * N;
    const int32_t *tk = p.tokens + static_cast<int64_t>(b) * N;
    if (tid == 0) {
        ts.err = 0;
        ts.key = 0;
    }
    for (int i = tid; i < N; i += kT) {
        ts.par[i] = __ldg(pa + i);
        ts.tok[i] = __ldg(tk + i);
        ts.flag[i] = 0;
    }
    __syncthreads();
    int err = 0;
    for (int i = tid; i < N; i += kT) {
        const int par = ts.par[i], t = ts.tok[i];
        if (i == 0) {
            if (par != -1) err |= kStTree;
        } else if (par < 0 || par >= i) {
            err |= kStTree;
        } else {
            ts.flag[par] = 1;  // every writer stores 1
            if (t < 0 || t >= p.V) err |= kStToken;
        }
        if (MODE == kTreeStochastic) {
            float lt = 0.f, ld = 0.f;
            if (i > 0 && par >= 0 && par < i && t >= 0 && t < p.V) {
                const int64_t off = (static_cast<int64_t>(b) * N + par) * p.stride + t;
                lt = load_logit<Tag>(p.tl, off);
                ld = load_logit<Tag>(p.dl, off);
            }
            tp.lt[i] = lt;
            tp.ld[i] = ld;
            if (i > 0)
                tu.ua[i] = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(i - 1),
                                          kPurposeAccept, p.offset);
            tu.us[i] = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(i),
                                      kPurposeSample, p.offset);
        }
    }
    if (err) atomicOr(&ts.err, err);
    __syncthreads();
    if (!(ts.err & kStTree)) {
        for (int i = tid; i < N; i += kT) {
            int j = i, d = 0;
            while (j != 0 && d <= p.max_depth) {
                j = ts.par[j];
                ++d;
            }
            const bool ok = (j == 0);
            ts.depth[i] = static_cast<short>(ok ? d : -1);
            if (!ok) atomicOr(&ts.err, kStTree);
        }
    }
    __syncthreads();
}

// tree_decide runs once the rows are merged: the row checks (every target
// row, and the draft rows of nodes with children), the node tests (a thread
// per node; greedy: the token is the parent's argmax; stochastic: the
// acceptance test), acceptance (a node is accepted when every node on its
// path passed its test: a walk up at most max_depth parents), the deepest
// accepted node (ties to the lowest index), and the outputs.
template <class Tag, int MODE>
__device__ __forceinline__ void tree_decide(const Params &p, int b, RowStats rs, TreeScratch &ts,
                                            const TreeProbe &tp, const TreeUniforms &tu)
{
    constexpr int kT = kDecideThreads;
    const int N = p.N, R = p.R, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    bool bad = false;
    for (int r = tid; r < R; r += kT) {
        if (r >= N && !(ts.flag[r - N] & 1)) continue;
        bad |= (MODE == kTreeGreedy) ? (rs.m[r] != rs.m[r]) : !stoch_row_ok(rs.m[r], rs.s[r]);
    }
    if (bad) atomicOr(&ts.err, kStLogit);
    __syncthreads();
    const int err = ts.err;
    if (!err) {
        for (int i = 1 + tid; i < N; i += kT) {
            const int par = ts.par[i];
            bool ok;
            if (MODE == kTreeGreedy) {
                ok = (ts.tok[i] == rs.idx[par]);
            } else {
                const double lp =
                    (f32_to_f64(tp.lt[i]) - static_cast<double>(rs.m[par])) * p.inv_t - log(rs.s[par]);
                const double lq =
                    (f32_to_f64(tp.ld[i]) - static_cast<double>(rs.m[N + par])) * p.inv_t - log(rs.s[N + par]);
                ok = accept_test(lp, lq, tu.ua[i]);
            }
            if (ok) ts.flag[i] |= 2;
        }
        __syncthreads();
        int key = 0;
        for (int i = tid; i < N; i += kT) {
            bool acc = true;
            for (int j = i; j != 0; j = ts.par[j]) acc &= (ts.flag[j] & 2) != 0;
            if (acc) key = max(key, (static_cast<int>(ts.depth[i]) << 11) | (kMaxNodes - 1 - i));
        }
        key = warp_max(key);
        if (lane == 0 && key) atomicMax(&ts.key, key);
        __syncthreads();
    }
    if (warp != 0) return;
    const int W = p.max_depth + 1;
    int32_t *out = p.out + static_cast<int64_t>(b) * W;
    int32_t *path = p.path ? p.path + static_cast<int64_t>(b) * W : nullptr;
    for (int j = lane; j < W; j += 32) {
        out[j] = -1;
        if (path) path[j] = -1;
    }
    __syncwarp();
    if (lane != 0) return;
    ReqInfo info = empty_req();
    if (err) {
        p.acc[b] = -1;
        report(p.status, err);
        store_req(p.req + b, info);
        return;
    }
    const int d = kMaxNodes - 1 - (ts.key & 2047);
    const int D = ts.depth[d];
    for (int node = d; node != 0; node = ts.par[node]) {
        out[ts.depth[node] - 1] = ts.tok[node];
        if (path) path[ts.depth[node]] = node;
    }
    if (path) path[0] = 0;
    p.acc[b] = D;
    if (MODE == kTreeGreedy) {
        out[D] = rs.idx[d];
    } else {
        info.mode = kModeTargetRow;
        info.t_off = (static_cast<int64_t>(b) * N + d) * p.stride;
        info.mt = rs.m[d];
        info.u = tu.us[d];
        info.out_index = b * W + D;
    }
    store_req(p.req + b, info);
}

// ------------------------------------------------------------------ pass 2
// Items of kSeg2 entries of the row (or row pair) a request draws from; a
// lane owns kLane2 contiguous entries of its item.

// The part of ReqInfo a pass-2 item needs, read as three 16-byte loads.
struct ItemInfo {
    int64_t t_off, d_off;
    float mt, md, kc, tcls;
    int mode;
};

__device__ __forceinline__ ItemInfo load_item_info(const Params &p, int b)
{
    static_assert(sizeof(ReqInfo) == 64, "ReqInfo is read as four 16-byte words");
    const uint4 *q = reinterpret_cast<const uint4 *>(p.req + b);
    const uint4 w0 = __ldcg(q), w2 = __ldcg(q + 2), w3 = __ldcg(q + 3);
    ItemInfo it;
    it.t_off = static_cast<int64_t>((static_cast<uint64_t>(w0.y) << 32) | w0.x);
    it.d_off = static_cast<int64_t>((static_cast<uint64_t>(w0.w) << 32) | w0.z);
    it.mt = __uint_as_float(w2.z);
    it.md = __uint_as_float(w2.w);
    it.mode = static_cast<int>(w3.x);
    it.kc = __uint_as_float(w3.z);
    it.tcls = __uint_as_float(w3.w);
    return it;
}

// The exponent of one entry, 2^z = exp((l - m)/T): z = l c - m c with one
// rounding (the rounding of m c shifts every z of a row alike and cancels
// in every normalised quantity).  Every fp64 weight of a row uses this.
__device__ __forceinline__ double neg_mc(const Params &p, float m) { return -(static_cast<double>(m) * p.c64); }
__device__ __forceinline__ double entry_z(const Params &p, float l, double nmc)
{
    return fma(static_cast<double>(l), p.c64, nmc);
}

// Stage this lane's vectors of item (s2) of the row (and draft row) into
// buf with asynchronous copies (one group is committed by the caller).
template <class Tag, bool kResidual>
__device__ __forceinline__ void stage_item(const Params &p, const ItemInfo &it, int s2, uint4 *buf)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    constexpr int kNV = StageShape<Tag>::kNV;
    const int lane = threadIdx.x & 31;
    const int base = s2 * kSeg2 + lane * kLane2;
    const char *trow = static_cast<const char *>(p.tl) + it.t_off * kEsz;
    const char *drow = static_cast<const char *>(p.dl) + it.d_off * kEsz;
#pragma unroll
    for (int v = 0; v < kNV; ++v) {
        const int e0 = base + v * kVec;
        if (e0 < p.V) {
            const unsigned dt = static_cast<unsigned>(__cvta_generic_to_shared(buf + v * 32 + lane));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dt),
                         "l"(trow + static_cast<int64_t>(e0) * kEsz) : "memory");
            if (kResidual) {
                const unsigned dd = static_cast<unsigned>(__cvta_generic_to_shared(buf + (kNV + v) * 32 + lane));
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dd),
                             "l"(drow + static_cast<int64_t>(e0) * kEsz) : "memory");
            }
        }
    }
}

// Per-lane sums of one item.  E, F: all e and f; A, B: e and f over the
// entries with p > q certain; amb: the entries whose sign is not certain.
struct P2Acc {
    double E, F, A, B;
    unsigned amb;  // bit i: entry base + i
};

// Reduce this lane's staged entries.  Residual: the sign of
// e/S_t - f/S_d is read from the fp32 logits: dz = (l_t - l_d) c - kc is
// log2(e/f) - log2(rho0) within 2^-21 (|dz| + |kc|), so dz > tcls makes
// e/f > rho0 2^kLog2Margin certain, |dz| <= tcls marks the entry.
template <class Tag, bool kResidual>
__device__ __forceinline__ P2Acc reduce_item(const Params &p, const ItemInfo &it, int s2, const uint4 *buf,
                                             const double *tab)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kNV = StageShape<Tag>::kNV;
    const int lane = threadIdx.x & 31;
    const int base = s2 * kSeg2 + lane * kLane2;
    const double nmt = neg_mc(p, it.mt), nmd = neg_mc(p, it.md);
    const float c = p.c, kc = it.kc, tc = it.tcls;
    P2Acc a;
    a.E = a.F = a.A = a.B = 0.0;
    a.amb = 0u;
#pragma unroll
    for (int v = 0; v < kNV; ++v) {
        const int e0 = base + v * kVec;
        uint4 tv = buf[v * 32 + lane];
        uint4 dv = kResidual ? buf[(kNV + v) * 32 + lane] : make_uint4(0, 0, 0, 0);
        if (e0 + kVec > p.V) {  // the ragged end of the row (nothing staged past V)
            tv = mask_tail<Tag>(tv, p.V - e0);
            if (kResidual) dv = mask_tail<Tag>(dv, p.V - e0);
        }
        float xt[kVec], xd[kVec];
        unpack<Tag>(tv, xt);
        if (kResidual) unpack<Tag>(dv, xd);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            const double et = exp2_fp64(entry_z(p, xt[e], nmt), tab);
            a.E += et;
            if (kResidual) {
                const double ef = exp2_fp64(entry_z(p, xd[e], nmd), tab);
                a.F += ef;
                const float dz = fmaf(xt[e] - xd[e], c, -kc);
                const double on = dz > tc ? 1.0 : 0.0;
                a.A = fma(on, et, a.A);
                a.B = fma(on, ef, a.B);
                a.amb |= fabsf(dz) <= tc ? (1u << (v * kVec + e)) : 0u;
            }
        }
    }
    if (!kResidual) a.A = a.E;
    return a;
}

// Exact weight of entry idx: residual max(0, e/S_t - f/S_d); else e.
template <class Tag>
__device__ __forceinline__ double exact_weight(const Params &p, const ReqInfo &info, bool residual, int idx,
                                               double isp, double isq, const double *tab)
{
    const double et = exp2_fp64(entry_z(p, load_logit<Tag>(p.tl, info.t_off + idx), neg_mc(p, info.mt)), tab);
    if (!residual) return et;
    const double ef = exp2_fp64(entry_z(p, load_logit<Tag>(p.dl, info.d_off + idx), neg_mc(p, info.md)), tab);
    const double pp = et * isp, qq = ef * isq;
    return pp > qq ? pp - qq : 0.0;
}

// Exact weights, summed in index order, of this lane's kLane2 entries
// [lo, lo + kLane2) (lo a multiple of kLane2), read as whole vectors.
template <class Tag>
__device__ __forceinline__ double lane_exact_sum(const Params &p, const ReqInfo &info, bool residual, int lo,
                                                 double isp, double isq, const double *tab)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    constexpr int kNV = kLane2 / kVec;
    const char *trow = static_cast<const char *>(p.tl) + info.t_off * kEsz;
    const char *drow = static_cast<const char *>(p.dl) + info.d_off * kEsz;
    const double nmt = neg_mc(p, info.mt), nmd = neg_mc(p, info.md);
    uint4 tv[kNV], dv[kNV];
#pragma unroll
    for (int v = 0; v < kNV; ++v) {
        const int e0 = lo + v * kVec;
        const bool in = e0 < p.V;
        tv[v] = in ? __ldcg(reinterpret_cast<const uint4 *>(trow + static_cast<int64_t>(e0) * kEsz)) : make_uint4(0, 0, 0, 0);
        dv[v] = (in && residual) ? __ldcg(reinterpret_cast<const uint4 *>(drow + static_cast<int64_t>(e0) * kEsz))
                                 : make_uint4(0, 0, 0, 0);
    }
    double w = 0.0;
#pragma unroll
    for (int v = 0; v < kNV; ++v) {
        const int e0 = lo + v * kVec;
        if (e0 + kVec > p.V) {
            tv[v] = mask_tail<Tag>(tv[v], p.V - e0);
            dv[v] = mask_tail<Tag>(dv[v], p.V - e0);
        }
        float xt[kVec], xd[kVec];
        unpack<Tag>(tv[v], xt);
        unpack<Tag>(dv[v], xd);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            const double et = exp2_fp64(entry_z(p, xt[e], nmt), tab);
            if (residual) {
                const double ef = exp2_fp64(entry_z(p, xd[e], nmd), tab);
                const double pp = et * isp, qq = ef * isq;
                w += pp > qq ? pp - qq : 0.0;
            } else {
                w += et;
            }
        }
    }
    return w;
}


// Exact weights, summed in index order, of the marked entries among the
// n32 bitmap words starting at word w0 (n32 = 16: a whole segment, read as
// four 16-byte loads; n32 = 1: one word, keeping the bits of [lo, lo+16)).
// Four entries at a time: their logits are loaded together.  One lane.
template <class Tag, int kWords>
__device__ __forceinline__ double marked_sum(const Params &p, const ReqInfo &info, const unsigned *bits,
                                             int w0, unsigned keep, double isp, double isq, const double *tab)
{
    unsigned m[kWords];
    if constexpr (kWords > 1) {
        static_assert(kWords % 4 == 0, "whole 16-byte words");
        const uint4 *q = reinterpret_cast<const uint4 *>(bits + w0);
#pragma unroll
        for (int i = 0; i < kWords / 4; ++i) {
            const uint4 u = __ldcg(q + i);
            m[4 * i] = u.x;
            m[4 * i + 1] = u.y;
            m[4 * i + 2] = u.z;
            m[4 * i + 3] = u.w;
        }
    } else {
        m[0] = __ldcg(bits + w0) & keep;
    }
    const double nmt = neg_mc(p, info.mt), nmd = neg_mc(p, info.md);
    double w = 0.0;
    for (;;) {
        int idx[4] = {-1, -1, -1, -1};
        int n = 0;
#pragma unroll
        for (int i = 0; i < kWords; ++i) {
            while (m[i] && n < 4) {
                const int v = ((w0 + i) << 5) + __ffs(m[i]) - 1;
                m[i] &= m[i] - 1;
                idx[0] = n == 0 ? v : idx[0];
                idx[1] = n == 1 ? v : idx[1];
                idx[2] = n == 2 ? v : idx[2];
                idx[3] = n == 3 ? v : idx[3];
                ++n;
            }
        }
        if (n == 0) break;
        float lt[4], ld[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            lt[j] = idx[j] >= 0 ? load_logit<Tag>(p.tl, info.t_off + idx[j]) : -INFINITY;
            ld[j] = idx[j] >= 0 ? load_logit<Tag>(p.dl, info.d_off + idx[j]) : -INFINITY;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const double pp = exp2_fp64(entry_z(p, lt[j], nmt), tab) * isp;
            const double qq = exp2_fp64(entry_z(p, ld[j], nmd), tab) * isq;
            w += pp > qq ? pp - qq : 0.0;
        }
        if (n < 4) break;
    }
    return w;
}

// Inclusive warp scan of doubles (fixed association order).
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

// Inverse CDF over n weights W[0..n) (this warp's scratch): the first
// index with positive weight whose inclusive prefix exceeds target, and the
// prefix before it; if rounding leaves none, the last index with positive
// weight (-1 if none).  Lane l owns the contiguous block
// [l per, (l+1) per): block sums, one warp scan, then one lane walks its
// block.  Z receives the total.  Warp-wide, fixed association order.
__device__ __forceinline__ int icdf_blocked(const double *W, int n, double u, double &before, double &Z)
{
    const int lane = threadIdx.x & 31;
    const int per = (n + 31) / 32;
    const int lo = min(n, lane * per), hi = min(n, lo + per);
    double bsum = 0.0;
    int blast = -1;
    for (int s = lo; s < hi; ++s) {
        const double w = W[s];
        bsum += w;
        if (w > 0.0) blast = s;
    }
    const double incl = warp_incl_scan(bsum);
    double excl = __shfl_up_sync(kFull, incl, 1);
    if (lane == 0) excl = 0.0;
    Z = __shfl_sync(kFull, incl, 31);
    const double target = u * Z;
    const unsigned hit = __ballot_sync(kFull, bsum > 0.0 && incl > target);
    if (hit) {
        const int L = __ffs(hit) - 1;
        int found = -1;
        double fb = 0.0;
        if (lane == L) {
            double run = excl;
            int lastp = -1;
            double lastb = 0.0;
            for (int s = lo; s < hi; ++s) {
                const double w = W[s];
                const double nxt = run + w;
                if (w > 0.0) {
                    lastp = s;
                    lastb = run;
                    if (nxt > target) {
                        found = s;
                        fb = run;
                        break;
                    }
                }
                run = nxt;
            }
            if (found < 0) {  // the block sum and the walk round differently
                found = lastp;
                fb = lastb;
            }
        }
        before = __shfl_sync(kFull, fb, L);
        return __shfl_sync(kFull, found, L);
    }
    const unsigned pos = __ballot_sync(kFull, blast >= 0);
    if (!pos) {
        before = 0.0;
        return -1;
    }
    const int L = 31 - __clz(pos);
    // the prefix before the last positive entry of block L
    double pre = 0.0;
    if (lane == L) {
        pre = excl;
        for (int s = lo; s < blast; ++s) pre += W[s];
    }
    before = __shfl_sync(kFull, pre, L);
    return __shfl_sync(kFull, blast, L);
}

// Draw the token of request b by inverse CDF: segment weights (closed form
// from the decided sums plus the exact weights of the marked entries), then
// the lane chunk of the chosen segment (the items' per-lane sums), then its
// entries (exact weights, one per lane).  One warp; W, B: S2 doubles of
// scratch each.  The sums of all segments are read in one round.
template <class Tag>
__device__ __forceinline__ void finalize(const Params &p, int b, const double *tab, double *W, double *B)
{
    constexpr int kU = 8;
    const int lane = threadIdx.x & 31;
    const int S2 = p.S2;
    const ReqInfo info = load_req(p.req + b);
    const double4 *part = p.p2part + static_cast<int64_t>(b) * S2;
    const int *namb = p.p2amb + static_cast<int64_t>(b) * S2;
    const unsigned *bits = p.ambbits + static_cast<int64_t>(b) * p.W32;
    double Sp = 0.0, Sq = 0.0;
    unsigned marked = 0u;  // bit j: segment 32 j + lane (mod 1024) holds marked entries
    for (int s0 = 0; s0 < S2; s0 += 32 * kU) {
        double4 pv[kU];
        int na[kU];
#pragma unroll
        for (int j = 0; j < kU; ++j) {
            const int s = s0 + j * 32 + lane;
            pv[j] = s < S2 ? ldcg_d4(part + s) : make_double4(0.0, 0.0, 0.0, 0.0);
            na[j] = s < S2 ? __ldcg(namb + s) : 0;
        }
#pragma unroll
        for (int j = 0; j < kU; ++j) {
            const int s = s0 + j * 32 + lane;
            if (s < S2) {
                Sp += pv[j].x;
                Sq += pv[j].y;
                W[s] = pv[j].z;
                B[s] = pv[j].w;
                if (na[j] > 0) marked |= 1u << ((s >> 5) & 31);
            }
        }
    }
    bool residual = info.mode == kModeResidual;
    bool exact_lanes = false;
    double isp = 1.0, isq = 1.0;
    if (residual) {
        Sp = warp_sum(Sp);
        Sq = warp_sum(Sq);
        isp = 1.0 / Sp;
        isq = 1.0 / Sq;
        const double rho = Sp / Sq;
        __syncwarp();
        if (!(rho >= info.rho_lo && rho <= info.rho_hi)) {
            exact_lanes = true;
            // the pass-1 estimate missed: every weight exactly, a segment at a time
            for (int s = 0; s < S2; ++s) {
                const double w =
                    warp_sum(lane_exact_sum<Tag>(p, info, true, s * kSeg2 + lane * kLane2, isp, isq, tab));
                if (lane == 0) W[s] = w;
            }
        } else {
            for (int s = lane; s < S2; s += 32) {
                const double w = W[s] * isp - B[s] * isq;
                W[s] = w > 0.0 ? w : 0.0;
            }
            // this lane's segments that hold marked entries
            while (marked) {
                const int j = __ffs(marked) - 1;
                marked &= marked - 1;
                for (int s = j * 32 + lane; s < S2; s += 32 * 32)
                    if (__ldcg(namb + s) > 0)
                        W[s] += marked_sum<Tag, kSeg2 / 32>(p, info, bits, s * (kSeg2 / 32), 0u, isp, isq, tab);
            }
        }
        __syncwarp();
        double z = 0.0;
        for (int s = lane; s < S2; s += 32) z += W[s];
        if (!(warp_sum(z) > 0.0)) {  // residual mass vanished in rounding: draw from target row n
            residual = false;
            exact_lanes = true;  // the items' lane sums are residual sums
            __syncwarp();
            for (int s = lane; s < S2; s += 32) W[s] = ldcg_d4(part + s).x;
        }
    }
    __syncwarp();
    double before, Z;
    int sstar = icdf_blocked(W, S2, info.u, before, Z);
    if (sstar < 0) sstar = 0;
    const double tseg = info.u * Z - before;

    // lane chunks of the chosen segment: the items' per-lane sums of the
    // decided entries plus the exact weights of the lane's marked entries
    // (every entry exactly when the pass-1 estimate missed or the residual
    // vanished)
    const int clo = sstar * kSeg2 + lane * kLane2;
    double lane_w;
    if (exact_lanes) {
        lane_w = lane_exact_sum<Tag>(p, info, residual, clo, isp, isq, tab);
    } else {
        const double2 pl = __ldcg(p.p2lane + (static_cast<int64_t>(b) * S2 + sstar) * 32 + lane);
        if (residual) {
            const double w = pl.x * isp - pl.y * isq;
            lane_w = w > 0.0 ? w : 0.0;
            if (__ldcg(namb + sstar) > 0) {
                // this lane's entries: the bits of [clo, clo + kLane2) of word clo / 32
                static_assert(kLane2 == 16 || kLane2 == 32, "a lane's entries lie in one bitmap word");
                const unsigned keep = kLane2 == 32 ? 0xFFFFFFFFu : ((clo & 31) ? 0xFFFF0000u : 0x0000FFFFu);
                lane_w += marked_sum<Tag, 1>(p, info, bits, clo >> 5, keep, isp, isq, tab);
            }
        } else {
            lane_w = pl.x;
        }
    }
    const double incl = warp_incl_scan(lane_w);
    double excl = __shfl_up_sync(kFull, incl, 1);
    if (lane == 0) excl = 0.0;
    const unsigned hit = __ballot_sync(kFull, lane_w > 0.0 && incl > tseg);
    int cl;
    if (hit) {
        cl = __ffs(hit) - 1;
    } else {
        const unsigned pos = __ballot_sync(kFull, lane_w > 0.0);
        cl = pos ? 31 - __clz(pos) : 0;
    }
    const double tchunk = tseg - __shfl_sync(kFull, excl, cl);

    // entries of chunk cl, one per lane
    const int cbase = sstar * kSeg2 + cl * kLane2;
    const int idx = cbase + lane;
    const bool valid = lane < kLane2 && idx < p.V;
    const double w1 = valid ? exact_weight<Tag>(p, info, residual, idx, isp, isq, tab) : 0.0;
    const double pincl = warp_incl_scan(w1);
    const unsigned ehit = __ballot_sync(kFull, w1 > 0.0 && pincl > tchunk);
    int token;
    if (ehit) {
        token = cbase + __ffs(ehit) - 1;
    } else {
        const unsigned pos = __ballot_sync(kFull, w1 > 0.0);
        token = pos ? cbase + 31 - __clz(pos) : cbase;
    }
    if (lane == 0) p.out[info.out_index] = token;
}

// One pass-2 item: reduce, then publish the sums, the per-lane partials
// and the marked entries.
template <class Tag, bool kResidual>
__device__ __forceinline__ void p2_item(const Params &p, int b, int s2, const ItemInfo &it, const uint4 *buf,
                                        const double *tab)
{
    const int lane = threadIdx.x & 31;
    const P2Acc a = reduce_item<Tag, kResidual>(p, it, s2, buf, tab);
    const int64_t at = static_cast<int64_t>(b) * p.S2 + s2;
    __stcg(p.p2lane + at * 32 + lane, make_double2(a.A, a.B));
    int namb = 0;
    if (kResidual) {
        const int word = (s2 * kSeg2 + lane * kLane2) >> 5;
        if constexpr (kLane2 == 32) {
            __stcg(p.ambbits + static_cast<int64_t>(b) * p.W32 + word, a.amb);
        } else {
            // two lanes' 16-entry masks form one bitmap word
            static_assert(kLane2 == 16, "one or two lanes per bitmap word");
            const unsigned other = __shfl_down_sync(kFull, a.amb, 1);
            if (!(lane & 1)) __stcg(p.ambbits + static_cast<int64_t>(b) * p.W32 + word, a.amb | (other << 16));
        }
        namb = __popc(a.amb);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) namb += __shfl_xor_sync(kFull, namb, o);
    }
    const double E = warp_sum(a.E), F = warp_sum(a.F), A = warp_sum(a.A), B = warp_sum(a.B);
    if (lane == 0) {
        stcg_d4(p.p2part + at, make_double4(E, F, A, B));
        __stcg(p.p2amb + at, namb);
    }
}

// ----------------------------------------------------------------- kernels
// Pass 1: every warp streams pass-1 items.
template <class Tag, int MODE, int kMinBlocks>
__global__ void __launch_bounds__(kThreads, kMinBlocks) k_pass1(const __grid_constant__ Params p)
{
    extern __shared__ uint4 rings[];
    // every pass-1 block is resident by now: the decide grid may be
    // scheduled onto the SMs that pass-1 blocks free
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    const int warp = threadIdx.x >> 5;
    pass1_stream<Tag, MODE>(p, rings + warp * kRing1 * Pass1Shape<Tag>::kSlot,
                            blockIdx.x * kWarps + warp, gridDim.x * kWarps);
}

// Decide: one block per request merges its rows (a warp per row) into
// shared memory, then runs the decide step (linear: warp 0; trees: the
// whole block, with the input-only part done before pass 1 completes).
// partials a decide block stages in shared memory (beyond that it reads them
// through L2): 12288 x 8 B = 96 KB
constexpr int kDecideStageMax = 12288;
template <class Tag, int MODE>
__global__ void __launch_bounds__(kDecideThreads) k_decide(const __grid_constant__ Params p)
{
    namespace cg = cooperative_groups;
    constexpr int kDW = kDecideThreads / 32;
    extern __shared__ double rowmem[];
    __shared__ TreeScratch ts;
    __shared__ TreeProbe tp;
    __shared__ TreeUniforms tu;
    // a request is decided by a cluster of G blocks (G = 1 without a
    // cluster launch): block `rank` merges rows [r0, r1) into the row
    // statistics of the cluster's rank-0 block (distributed shared memory),
    // which then runs the decide step
    cg::cluster_group cluster = cg::this_cluster();
    const int G = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int cid = blockIdx.x / G, ncl = gridDim.x / G;
    const int RG = (p.R + G - 1) / G;
    const int r0 = min(p.R, rank * RG), r1 = min(p.R, r0 + RG);
    const int warp = threadIdx.x >> 5;
    RowStats rs;  // this block's row statistics (rank 0: the request's)
    rs.s = rowmem;
    rs.m = reinterpret_cast<float *>(rowmem + p.R);
    rs.idx = reinterpret_cast<int *>(rs.m + p.R);
    RowStats rs0;  // rank 0's
    rs0.s = cluster.map_shared_rank(rs.s, 0);
    rs0.m = cluster.map_shared_rank(rs.m, 0);
    rs0.idx = cluster.map_shared_rank(rs.idx, 0);
    const bool stage_parts = (r1 - r0) * p.S <= kDecideStageMax;
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    DraftProbe pr;
    if (MODE == kLinear && warp == 0) pr = probe_drafts<Tag>(p, cid);
    // trees: everything that reads only inputs, before pass 1 completes
    if (MODE != kLinear && cid < p.B) tree_prepare<Tag, MODE>(p, cid, ts, tp, tu);
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    for (int b = cid; b < p.B; b += ncl) {
        // the block's rows' partials, staged in shared memory by every
        // thread at once (one round of independent loads) when they fit,
        // then merged a warp per row (the draft rows of nodes without
        // children are not read)
        float2 *stg = stage_parts ? reinterpret_cast<float2 *>(rs.idx + p.R) : nullptr;
        if (stage_parts) {
            const float2 *src = p.rowpart + (static_cast<int64_t>(b) * p.R + r0) * p.S;
            const int n = (r1 - r0) * p.S;
            for (int i = threadIdx.x; i < n; i += kDecideThreads) stg[i] = __ldcg(src + i);
            __syncthreads();
        }
        for (int r = r0 + warp; r < r1; r += kDW) {
            if (MODE != kLinear && r >= p.N && !(ts.flag[r - p.N] & 1)) continue;
            merge_row<MODE>(p, b, r, rs0, stg, r0);
        }
        cluster.sync();  // every row's statistics are in rank 0
        if (rank == 0) {
            if constexpr (MODE == kLinear) {
                if (warp == 0) {
                    decide_linear<Tag>(p, b, rs, pr);
                    pr = probe_drafts<Tag>(p, b + ncl);
                }
            } else {
                tree_decide<Tag, MODE>(p, b, rs, ts, tp, tu);
            }
        }
        __syncthreads();
        if (MODE != kLinear && b + ncl < p.B) tree_prepare<Tag, MODE>(p, b + ncl, ts, tp, tu);
        cluster.sync();  // rank 0 is done with the statistics before they are rewritten
    }
}

// Pass 2: (request, segment) items, two ahead: while item i is reduced,
// item i+1 is being copied and the request record of item i+2 is read.
template <class Tag, int MODE>
__global__ void __launch_bounds__(kThreads, 3) k_pass2(const __grid_constant__ Params p)
{
    extern __shared__ uint4 dyn[];
    __shared__ double tab[kExp2Tab];
    const int warp = threadIdx.x >> 5;
    for (int j = threadIdx.x; j < kExp2Tab; j += kThreads) tab[j] = p.exp2tab[j];
    __syncthreads();
    uint4 *stage = dyn + warp * StageShape<Tag>::kPerWarp;
    // the finalize grid may be scheduled as blocks of this one retire
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    // hardware wait: pass 1 complete and its writes visible
    asm volatile("griddepcontrol.wait;\n" ::: "memory");

    const unsigned W = gridDim.x * kWarps;
    auto req_of = [&](unsigned t) { return static_cast<int>(fdiv(t, p.div_s2)); };
    auto info_of = [&](unsigned t) {
        ItemInfo it;
        if (t < p.nP) {
            it = load_item_info(p, req_of(t));
        } else {
            it.mode = kModeNone;
            it.t_off = it.d_off = 0;
            it.mt = it.md = it.kc = it.tcls = 0.f;
        }
        return it;
    };
    auto stage_of = [&](unsigned t, const ItemInfo &it, uint4 *buf) {
        if (t >= p.nP) return;
        const int s2 = static_cast<int>(t - static_cast<unsigned>(req_of(t)) * static_cast<unsigned>(p.S2));
        if (it.mode == kModeResidual) stage_item<Tag, true>(p, it, s2, buf);
        else if (it.mode == kModeTargetRow) stage_item<Tag, false>(p, it, s2, buf);
    };

    // warp w of W takes items w, w + W, ... (a static round robin over
    // request-major items mixes requests evenly)
    unsigned t_cur = blockIdx.x * kWarps + warp;
    unsigned t_nxt = t_cur + W;
    ItemInfo i_cur = info_of(t_cur);
    ItemInfo i_nxt = info_of(t_nxt);
    stage_of(t_cur, i_cur, stage);
    commit_copies();
    int buf = 0;
#pragma unroll 1
    while (t_cur < p.nP) {
        stage_of(t_nxt, i_nxt, stage + (buf ^ 1) * StageShape<Tag>::kPerBuf);
        commit_copies();
        const unsigned t_nn = t_nxt + W;
        const ItemInfo i_nn = info_of(t_nn);  // loads in flight during the reduction
        wait_copies<1>();
        const int b = req_of(t_cur);
        const int s2 = static_cast<int>(t_cur - static_cast<unsigned>(b) * static_cast<unsigned>(p.S2));
        const uint4 *cur = stage + buf * StageShape<Tag>::kPerBuf;
        if (i_cur.mode == kModeResidual) p2_item<Tag, true>(p, b, s2, i_cur, cur, tab);
        else if (i_cur.mode == kModeTargetRow) p2_item<Tag, false>(p, b, s2, i_cur, cur, tab);
        t_cur = t_nxt;
        i_cur = i_nxt;
        t_nxt = t_nn;
        i_nxt = i_nn;
        buf ^= 1;
    }
    wait_copies<0>();
}

// Finalize: one warp per request draws its token once every pass-2 item
// has completed (a programmatic dependent of the pass-2 grid).
template <class Tag, int MODE>
__global__ void __launch_bounds__(kThreads) k_finalize(const __grid_constant__ Params p)
{
    extern __shared__ double wdyn[];
    __shared__ double tab[kExp2Tab];
    const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int j = threadIdx.x; j < kExp2Tab; j += blockDim.x) tab[j] = p.exp2tab[j];
    __syncthreads();
    const bool w_shared = p.S2 <= kMaxS2Shared;
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    for (int b = blockIdx.x * nw + warp; b < p.B; b += gridDim.x * nw) {
        if (__ldcg(&p.req[b].mode) == kModeNone) continue;
        double *W = w_shared ? wdyn + 2 * warp * p.S2 : p.p2w + 2 * static_cast<int64_t>(b) * p.S2;
        finalize<Tag>(p, b, tab, W, W + p.S2);
    }
}

}  // namespace sv
