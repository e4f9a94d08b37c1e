// sv_fused.cuh -- linear stochastic verification as one persistent kernel.
//
// The same steps as the four-kernel path (sv_verify.cuh), overlapped:
// while pass 1 streams the rows of later requests, the decide steps and
// the fp64 pass-2 items of earlier requests run beside it, so the
// special-function, FMA and fp64 pipes and the memory system work at the
// same time and no step waits for a whole grid.
//
//  * Warps [0, kStreamers) of each block stream pass-1 items as k_pass1
//    does (static round robin, no fences), the last part of them in
//    chunks claimed from a counter, so faster SMs take more.  Before the
//    kernel every partial holds kPartEmpty, a bit pattern the reduction
//    never stores, so a partial that differs from it is complete.
//  * The other warps, and every streamer once its pass-1 items are done,
//    take tasks from a shared counter: first the B decide tasks (each starts
//    as early as possible), then the B * S2 pass-2 items in request order.
//    The decide task polls the
//    request's partials (uncached loads, bounded) until none is empty,
//    merges its rows, decides ("Speculative decoding explained", section
//    "Draft and verification loop") and publishes decided[b].  A pass-2
//    item waits (bounded) for decided[b], is reduced, and arrives on the
//    request's counter; the warp that completes the last draws the token.
//    An expired wait sets SPEC_STATUS_TIMEOUT and the warp leaves.
//
// Progress: streamers wait on nothing; a decide task waits only on
// streamers; an item waits only on its request's decide task, which was
// claimed earlier by a running warp.  The grid is one resident wave, and
// the launch is cooperative, so a grid that cannot be resident at once
// fails to launch instead of leaving a wait to expire.
#pragma once

#include "sv_verify.cuh"

namespace sv {

constexpr int kStreamers = 6;        // pass-1 warps per block
constexpr int kRegion = 3 * 256;     // uint4 per warp (12 KB): pass-1 ring, later task scratch
static_assert(kRing1 * 32 * 8 <= kRegion, "the pass-1 ring fits a warp region");
constexpr size_t kFusedSmem = sizeof(uint4) * kRegion * kWarps;
constexpr unsigned kWaitPolls = 1u << 20;  // ~1 s of polling at <= 1 us per poll (Params::poll_limit)
// An empty partial / counter word: all bits set (one memset per call).  A
// stored partial's max is never this NaN: NaN maxima are canonical.
constexpr unsigned kPartEmpty = 0xFFFFFFFFu;

// Polling reads: fetched again on every call (never from a stale L1 line)
// and free to overlap with each other; 8-byte reads are single-copy atomic,
// so a partial is seen either empty or complete.
__device__ __forceinline__ unsigned long long ld_poll64(const void *p)
{
    return __ldcv(reinterpret_cast<const unsigned long long *>(p));
}
__device__ __forceinline__ unsigned ld_poll32(const unsigned *p) { return __ldcv(p); }
// A flag read with acquire semantics: this thread's later reads see what the
// writer stored before its release (a fence, then the flag).
__device__ __forceinline__ unsigned ld_acquire32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void backoff(unsigned &ns)
{
    __nanosleep(ns);
    ns = ns < 1024 ? 2 * ns : 1024;
}

// Merge one row's S partials (one lane), in two passes so that the terms
// are independent: the row max first, then the sum in fp64 of each partial
// rescaled to it by a special-function exponential (relative error ~2^-22,
// below the pass-1 sums' own).
template <class Load>
__device__ __forceinline__ void merge_row_lane(const Params &p, Load part, float &M, double &S)
{
    float m = -INFINITY;
    bool nan = false;
#pragma unroll 4
    for (int j = 0; j < p.S; ++j) {
        const float2 v = part(j);
        nan |= (v.x != v.x) || (v.y != v.y);
        m = fmaxf(m, v.x);
    }
    double s = 0.0;
    if (m != -INFINITY) {
#pragma unroll 4
        for (int j = 0; j < p.S; ++j) {
            const float2 v = part(j);
            if (v.x != -INFINITY) s += static_cast<double>(v.y * ex2_approx((v.x - m) * p.c));
        }
    }
    M = nan ? __int_as_float(0x7FC00000) : m;
    S = nan ? __longlong_as_double(0x7FF8000000000000ll) : s;
}

// The decide task of request b: wait until all its pass-1 partials are
// stored, merge its rows (a lane per row), decide, publish.  scr: the
// warp's region; R*S partials are staged there when they fit, else
// re-read through L2.  False when the wait expired.
template <class Tag>
__device__ __forceinline__ bool decide_task(const Params &p, int b, uint4 *scr)
{
    const int lane = threadIdx.x & 31;
    const DraftProbe pr = probe_drafts<Tag>(p, b);  // inputs: read while pass 1 runs
    const int n = p.R * p.S;
    const float2 *part = p.rowpart + static_cast<int64_t>(b) * n;
    float2 *stg = reinterpret_cast<float2 *>(scr);
    const bool staged = static_cast<size_t>(n) * sizeof(float2) + sizeof(double) * 2 * 65 <=
                        sizeof(uint4) * kRegion;
    bool done = false;
    unsigned ns = 64, it = 0;
    // the request's last partial first, one word per poll (items are taken
    // in increasing order, so it is among the last of the request's to be
    // stored); then every partial until all are stored
    for (; it < p.poll_limit; ++it) {
        unsigned seen = 0;
        if (lane == 0) seen = static_cast<unsigned>(ld_poll64(part + n - 1)) != kPartEmpty;
        if (__shfl_sync(kFull, seen, 0)) break;
        backoff(ns);
    }
    ns = 64;
    for (; it < p.poll_limit; ++it) {
        bool all = true;
        for (int i = lane; i < n; i += 32) {
            const unsigned long long v = ld_poll64(part + i);
            all &= static_cast<unsigned>(v) != kPartEmpty;
            if (staged) stg[i] = make_float2(__uint_as_float(static_cast<unsigned>(v)),
                                             __uint_as_float(static_cast<unsigned>(v >> 32)));
        }
        if (__all_sync(kFull, all)) {
            done = true;
            break;
        }
        backoff(ns);
    }
    if (!done) {
        // the request is given up: its outputs read -1
        for (int j = lane; j <= p.k; j += 32) p.out[static_cast<int64_t>(b) * (p.k + 1) + j] = -1;
        if (lane == 0) {
            p.acc[b] = -1;
            report(p.status, kStTimeout);
        }
        return false;
    }
    __syncwarp();
    double *ds = reinterpret_cast<double *>(scr + kRegion) - 65;
    float *dm = reinterpret_cast<float *>(ds) - 65;
    for (int r = lane; r < p.R; r += 32) {
        float M;
        double S;
        if (staged) {
            merge_row_lane(p, [&](int j) { return stg[r * p.S + j]; }, M, S);
        } else {
            // not staged: the values are final now; read them through L2
            merge_row_lane(p, [&](int j) { return __ldcg(part + r * p.S + j); }, M, S);
        }
        dm[r] = M;
        ds[r] = S;
    }
    __syncwarp();
    RowStats rs;
    rs.s = ds;
    rs.m = dm;
    rs.idx = nullptr;
    decide_linear<Tag>(p, b, rs, pr);
    __syncwarp();
    if (lane == 0) {
        __threadfence();
        atomicExch(&p.decided[b], 1u);
    }
    return true;
}

// Request b's decision, published?  Every lane reads the flag with acquire
// semantics, so the request record read afterwards is the published one.
__device__ __forceinline__ bool is_decided(const Params &p, int b)
{
    return __all_sync(kFull, ld_acquire32(&p.decided[b]) == 1u);
}

// Wait (bounded) until request b is decided.  False on expiry.
__device__ __forceinline__ bool wait_decided(const Params &p, int b)
{
    unsigned ns = 32;
    for (unsigned i = 0; i < p.poll_limit; ++i) {
        if (is_decided(p, b)) return true;
        backoff(ns);
    }
    if ((threadIdx.x & 31) == 0) report(p.status, kStTimeout);
    return false;
}

// The task worker.  Tasks come in request order from one shared counter
// (which starts at kPartEmpty, so a claim returns the task id minus one):
// first the B decide tasks, then the B * S2 pass-2 items.  A decide task is
// claimed only by a free warp, so it starts at once and no item waits on a
// decide that waits on that item's warp.  Once a warp's claim is an item,
// every decide has been claimed, and the warp claims one item ahead: the
// next item is staged (if its request is decided by then) while the
// current one is reduced.
template <class Tag>
__device__ __forceinline__ void fused_tasks(const Params &p, uint4 *region, const double *tab)
{
    constexpr int kBuf = StageShape<Tag>::kPerBuf;
    const int lane = threadIdx.x & 31;
    // two staging buffers, then the finalize scratch
    static_assert(2 * kBuf <= kRegion, "two staging buffers fit a warp region");
    double *W_sh = reinterpret_cast<double *>(region + 2 * kBuf);
    const bool w_shared = 2 * static_cast<size_t>(p.S2) * sizeof(double) <=
                          sizeof(uint4) * static_cast<size_t>(kRegion - 2 * kBuf);
    const unsigned nB = static_cast<unsigned>(p.B);
    const unsigned ntask = nB * (static_cast<unsigned>(p.S2) + 1u);
    auto claim = [&]() {
        unsigned t = 0;
        if (lane == 0) t = atomicAdd(p.p2claim, 1u) + 1u;
        return __shfl_sync(kFull, t, 0);
    };
    unsigned cur = claim();
#pragma unroll 1
    while (cur < nB) {
        if (!decide_task<Tag>(p, static_cast<int>(cur), region)) return;
        cur = claim();
    }
    if (cur >= ntask) return;

    // a held item: request, segment, record; staged = its copies are issued
    // (one committed group per staged item)
    struct Held {
        int b, s2;
        ItemInfo it;
        bool staged;
    };
    auto locate = [&](unsigned t) {
        Held h;
        const unsigned item = t - nB;
        h.b = static_cast<int>(fdiv(item, p.div_s2));
        h.s2 = static_cast<int>(item - static_cast<unsigned>(h.b) * static_cast<unsigned>(p.S2));
        h.it.mode = kModeNone;
        h.staged = false;
        return h;
    };
    auto stage = [&](Held &h, uint4 *buf) {
        h.it = load_item_info(p, h.b);
        if (h.it.mode == kModeResidual) stage_item<Tag, true>(p, h.it, h.s2, buf);
        else if (h.it.mode == kModeTargetRow) stage_item<Tag, false>(p, h.it, h.s2, buf);
        commit_copies();
        h.staged = true;
    };
    Held c = locate(cur);
    if (!wait_decided(p, c.b)) return;
    stage(c, region);
    int bc = 0;
#pragma unroll 1
    for (;;) {
        const unsigned nt = claim();
        const bool more = nt < ntask;
        Held n = more ? locate(nt) : c;
        if (more && is_decided(p, n.b)) stage(n, region + (bc ^ 1) * kBuf);
        const bool ahead = more && n.staged;
        if (ahead) wait_copies<1>();
        else wait_copies<0>();
        const uint4 *buf = region + bc * kBuf;
        if (c.it.mode == kModeResidual || c.it.mode == kModeTargetRow) {
            if (c.it.mode == kModeResidual) p2_item<Tag, true>(p, c.b, c.s2, c.it, buf, tab);
            else p2_item<Tag, false>(p, c.b, c.s2, c.it, buf, tab);
            // no copy in flight across the fence (a fence waits for them)
            if (ahead) wait_copies<0>();
            __threadfence();  // every lane's stores of the item precede its arrival
            __syncwarp();
            unsigned o = 0;
            if (lane == 0) {
                o = atomicAdd(&p.p2cnt[c.b], 1u) + 1u;  // the counter starts at kPartEmpty
                if (o == static_cast<unsigned>(p.S2) - 1u) __threadfence();
            }
            if (__shfl_sync(kFull, o == static_cast<unsigned>(p.S2) - 1u ? 1 : 0, 0)) {
                double *W = w_shared ? W_sh : p.p2w + 2 * static_cast<int64_t>(c.b) * p.S2;
                finalize<Tag>(p, c.b, tab, W, W + p.S2);
            }
        }
        if (!more) break;
        if (!n.staged) {
            if (!wait_decided(p, n.b)) break;
            stage(n, region + (bc ^ 1) * kBuf);
        }
        c = n;
        bc ^= 1;
    }
    wait_copies<0>();
}

template <class Tag>
__global__ void __launch_bounds__(kThreads, 2) k_fused(const __grid_constant__ Params p)
{
    extern __shared__ uint4 fdyn[];
    __shared__ double tab[kExp2Tab];
    for (int j = threadIdx.x; j < kExp2Tab; j += kThreads) tab[j] = p.exp2tab[j];
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    uint4 *region = fdyn + warp * kRegion;
    if (warp < kStreamers)
        pass1_stream<Tag, kLinear>(p, region, blockIdx.x * kStreamers + warp, gridDim.x * kStreamers);
    fused_tasks<Tag>(p, region, tab);
}

}  // namespace sv
