// sv_fused.cuh -- linear stochastic verification as one persistent kernel.
//
// The same steps as the four-kernel path (sv_verify.cuh), overlapped:
// while pass 1 streams the rows of later requests, the decide steps and
// the fp64 pass-2 items of earlier requests run beside it, so the
// special-function, FMA and fp64 pipes and the memory system work at the
// same time and no step waits for a whole grid.
//
//  * The kernel is launched cooperatively (every block resident at once,
//    or the launch fails).  It first clears its own counters and sets every
//    pass-1 partial to kPartEmpty (a bit pattern the reduction never
//    stores) and every output to -1, then passes one grid-wide barrier;
//    the streamers' first copies are already in flight across it.
//  * Warps [0, kStreamers) of each block stream pass-1 items as k_pass1
//    does (static round robin, no fences), the last part of them in
//    chunks claimed from a counter, so faster SMs take more.  A partial
//    that differs from kPartEmpty is complete.
//  * Each stored partial is also counted on its row (rowdone, a relaxed
//    atomic without a fence: the count may become visible before the
//    partial, so a reader checks the partials themselves).
//  * The other warps, and every streamer once its pass-1 items are done,
//    first take the B decide tasks from a counter (each starts as early as
//    possible).  A decide task polls its request's R row counts (one word
//    per lane, bounded) until every row is counted complete, reads the
//    partials (re-reading any still empty), merges each row across the warp,
//    decides ("Speculative decoding explained", section "Draft and
//    verification loop") and publishes decided[b].
//  * Then they take pass-2 tickets from one counter, in request order: a
//    ticket is a chunk of a request's items (segments of the row or row pair
//    of its final draw).  A worker keeps two tickets in flight: the next
//    one's rows are copied into shared memory while the current one is
//    reduced in fp64, published, and counted with one fence and one atomic;
//    the warp that completes a request's last item draws its token.  An
//    expired wait sets SPEC_STATUS_TIMEOUT and the warp leaves.
//
// Progress: streamers wait on nothing; a decide task waits only on
// streamers; a pass-2 worker waits only on decide tasks, which are claimed
// (and so running) before any warp takes a ticket.
#pragma once

#include <cooperative_groups.h>

#include "sv_verify.cuh"

namespace sv {

constexpr int kStreamers = 6;        // pass-1 warps per block
constexpr int kFusedRing = 3;        // ring slots of a streamer (kFusedRing - 1 items in flight)
constexpr int kRegion = 640;         // uint4 (10 KB): a task warp's scratch
// a streamer's region holds its ring, and later (when it takes tasks) the
// task scratch
constexpr int kRegionS = kFusedRing * 256 > kRegion ? kFusedRing * 256 : kRegion;
static_assert(256 == 32 * 8, "a ring slot is one pass-1 item (256 uint4)");
constexpr size_t kFusedSmem = sizeof(uint4) * (kRegionS * kStreamers + kRegion * (kWarps - kStreamers));
constexpr unsigned kWaitPolls = 1u << 20;  // ~1 s of polling at <= 1 us per poll
// pass-2 items per ticket: two 2 KB segments (bf16), one 4 KB segment (fp32)
constexpr int kP2ChunkBf16 = 2;
constexpr int kP2ChunkF32 = 1;
template <class Tag>
constexpr int p2_chunk() { return Tag::kVec == 8 ? kP2ChunkBf16 : kP2ChunkF32; }
// An empty partial: all bits set.  A stored partial's max is never this
// NaN: NaN maxima are canonical.
constexpr unsigned kPartEmpty = 0xFFFFFFFFu;

// Polling reads: fetched again on every call (never from a stale L1 line)
// and free to overlap with each other; 8-byte reads are single-copy atomic,
// so a partial is seen either empty or complete.
__device__ __forceinline__ unsigned long long ld_poll64(const void *p)
{
    return __ldcv(reinterpret_cast<const unsigned long long *>(p));
}
__device__ __forceinline__ unsigned ld_poll32(const unsigned *p) { return __ldcv(p); }

__device__ __forceinline__ void backoff(unsigned &ns, unsigned cap = 1024)
{
    __nanosleep(ns);
    ns = ns < cap ? 2 * ns : cap;
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

// Before the grid-wide barrier: counters to 0, pass-1 partials to
// kPartEmpty, outputs to -1 (what a request keeps if a wait expires).
__device__ __forceinline__ void fused_init(const Params &p)
{
    const unsigned tid = blockIdx.x * blockDim.x + threadIdx.x;
    const unsigned nth = gridDim.x * blockDim.x;
    for (unsigned i = tid; i < p.ncounters; i += nth) p.p2cnt[i] = 0u;
    uint2 *part = reinterpret_cast<uint2 *>(p.rowpart);
    for (unsigned i = tid; i < p.nA; i += nth) part[i] = make_uint2(kPartEmpty, kPartEmpty);
    const unsigned nout = static_cast<unsigned>(p.B) * static_cast<unsigned>(p.k + 1);
    for (unsigned i = tid; i < nout; i += nth) p.out[i] = -1;
    for (unsigned i = tid; i < static_cast<unsigned>(p.B); i += nth) p.acc[i] = -1;
}

// The streamer of the fused kernel.  Items [0, nAs) are taken in static
// round robin (as in pass1_stream); the rest, in chunks of kDynChunk
// consecutive items from a shared counter, claimed one chunk ahead just
// before the warp needs it, so the SMs that run faster take more of the
// tail.  Lane q holds the item id of slot q (kNoItem: the sequence ended).
// The ring is first filled with static items only, before the grid-wide
// barrier (no counter may be touched before it); then the barrier.
constexpr unsigned kDynChunk = 4;
template <class Tag>
__device__ __forceinline__ void fused_stream(const Params &p, uint4 *ring, unsigned w, unsigned W,
                                             bool streamer)
{
    constexpr int kSlot = Pass1Shape<Tag>::kSlot;
    const int lane = threadIdx.x & 31;
    unsigned st = w;                  // next static item
    unsigned dyn = 0, dyn_end = 0;    // current claimed chunk
    unsigned claim = 0;               // lane 0: the chunk claimed ahead
    bool claimed = false, done = false;
    auto claim_ahead = [&]() {
        if (lane == 0) claim = atomicAdd(p.a_claim, 1u);
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
    auto refill = [&](int q) {
        const unsigned it = done ? kNoItem : next_item();
        if (it != kNoItem) issue_item<Tag>(item1<Tag, kLinear>(p, it, false), ring + q * kSlot);
        if (lane == q) meta = it;
        commit_copies();
    };
    // prologue: static items only (a static item whose successor would be
    // claimed stops the prologue before that claim)
    int filled = 0;
    if (streamer) {
#pragma unroll 1
        for (; filled < kFusedRing && st < p.nAs && st + W < p.nAs; ++filled) refill(filled);
    }
    cooperative_groups::this_grid().sync();
    if (!streamer) return;
#pragma unroll 1
    for (; filled < kFusedRing; ++filled) refill(filled);
    int q = 0;
#pragma unroll 1
    for (;;) {
        wait_copies<kFusedRing - 1>();
        const unsigned it = __shfl_sync(kFull, meta, q);
        if (it == kNoItem) break;
        const int s = static_cast<int>(it - fdiv(it, p.div_s) * static_cast<unsigned>(p.S));
        reduce_item1<Tag, kLinear>(p, it, s, ring + q * kSlot);
        if (lane == 0) atomicAdd(p.rowdone + fdiv(it, p.div_s), 1u);  // no fence: a hint only
        refill(q);
        q = (q + 1 == kFusedRing) ? 0 : q + 1;
    }
    wait_copies<0>();
}

// The decide task of request b: wait until every row of the request is
// counted complete, then until every partial is stored (the counts carry no
// fence, so a partial still empty is read again), merge each row across the
// warp, decide, publish.  scr: the warp's region (the partials are staged
// there when they fit, else read again through L2).  False when a wait
// expired.
template <class Tag>
__device__ __forceinline__ bool decide_task(const Params &p, int b, uint4 *scr)
{
    const int lane = threadIdx.x & 31;
    const DraftProbe pr = probe_drafts<Tag>(p, b);  // inputs: read while pass 1 runs
    const int n = p.R * p.S;
    const float2 *part = p.rowpart + static_cast<int64_t>(b) * n;
    const unsigned *cnt = p.rowdone + static_cast<int64_t>(b) * p.R;
    float2 *stg = reinterpret_cast<float2 *>(scr);
    const bool staged = static_cast<size_t>(n) * sizeof(float2) + sizeof(double) * 2 * 65 <=
                        sizeof(uint4) * kRegion;
    bool done = false;
    unsigned it = 0, ns = 64;
    for (; it < p.poll_limit; ++it) {
        bool all = true;
        for (int r = lane; r < p.R; r += 32) all &= ld_poll32(cnt + r) >= static_cast<unsigned>(p.S);
        if (__all_sync(kFull, all)) {
            done = true;
            break;
        }
        backoff(ns, 1024);
    }
    // every partial counted: read them all, again only those still empty
    bool have = false;
    if (done) {
        bool first = true;  // the first round reads every partial
        for (; it < p.poll_limit; ++it) {
            bool all = true;
            for (int i = lane; i < n; i += 32) {
                if (staged && !first && __float_as_uint(stg[i].x) != kPartEmpty) continue;
                const unsigned long long v = ld_poll64(part + i);
                all &= static_cast<unsigned>(v) != kPartEmpty;
                if (staged)
                    stg[i] = make_float2(__uint_as_float(static_cast<unsigned>(v)),
                                         __uint_as_float(static_cast<unsigned>(v >> 32)));
            }
            first = false;
            if (__all_sync(kFull, all)) break;
            __nanosleep(64);
        }
        have = it < p.poll_limit;
    }
    if (!have) {
        if (lane == 0) report(p.status, kStTimeout);
        return false;
    }
    __syncwarp();
    // a lane per row (its partials from shared memory; no shuffles, so the
    // chain stays short on a warp that shares its scheduler with streamers)
    double *ds = reinterpret_cast<double *>(scr + kRegion) - 65;
    float *dm = reinterpret_cast<float *>(ds) - 65;
    for (int r = lane; r < p.R; r += 32) {
        float M;
        double S;
        if (staged) merge_row_lane(p, [&](int j) { return stg[r * p.S + j]; }, M, S);
        else merge_row_lane(p, [&](int j) { return __ldcg(part + r * p.S + j); }, M, S);
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

// Wait (lane 0 polls, bounded) until request b is decided; then a fence
// orders the request record's reads after the flag.  False on expiry.
__device__ __forceinline__ bool wait_decided(const Params &p, int b)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0) {
        unsigned ns = 32;
        for (unsigned i = 0; i < p.poll_limit; ++i) {
            if (ld_poll32(&p.decided[b]) == 1u) {
                ok = 1;
                break;
            }
            backoff(ns, 512);
        }
        if (ok) __threadfence();
        else report(p.status, kStTimeout);
    }
    return __shfl_sync(kFull, ok, 0) != 0;
}

// A pass-2 ticket: items [c0, c1) of request b.
struct Ticket {
    int b, c0, c1;
    ItemInfo it;
    bool valid;  // a ticket of the call (past the last: the worker is done)
    bool work;   // the request draws a token (else its tickets are empty)
};

// Take the next ticket, wait until its request is decided and read its
// record (unless it is the request of `prev`), and start the copies of its
// rows into buf (one commit group, empty when there is nothing to copy).
// False when a wait expired.
template <class Tag>
__device__ __forceinline__ bool take_ticket(const Params &p, Ticket &t, const Ticket &prev, uint4 *buf,
                                            unsigned &ahead)
{
    constexpr int kCh = p2_chunk<Tag>();
    const int lane = threadIdx.x & 31;
    // the ticket number was claimed one ticket ahead (lane 0), so the
    // atomic's round trip overlaps the work in between
    unsigned x = __shfl_sync(kFull, ahead, 0);
    if (lane == 0) ahead = atomicAdd(p.p2ticket, 1u);
    const unsigned cpr = p.div_cpr.d;
    t.valid = x < static_cast<unsigned>(p.B) * cpr;
    t.work = false;
    if (t.valid) {
        t.b = static_cast<int>(fdiv(x, p.div_cpr));
        const int c = static_cast<int>(x - static_cast<unsigned>(t.b) * cpr);
        t.c0 = c * kCh;
        t.c1 = min(t.c0 + kCh, p.S2);
        if (prev.valid && prev.b == t.b) {
            t.it = prev.it;
        } else {
            if (!wait_decided(p, t.b)) {
                commit_copies();
                return false;
            }
            t.it = load_item_info(p, t.b);
        }
        t.work = t.it.mode == kModeResidual || t.it.mode == kModeTargetRow;
        if (t.work)
            for (int s2 = t.c0; s2 < t.c1; ++s2) {
                uint4 *sb = buf + (s2 - t.c0) * StageShape<Tag>::kPerBuf;
                if (t.it.mode == kModeResidual) stage_item<Tag, true>(p, t.it, s2, sb);
                else stage_item<Tag, false>(p, t.it, s2, sb);
            }
    }
    commit_copies();
    return true;
}

// Reduce and publish a staged ticket, count its items with one fence and
// one atomic; true when it completed its request (the caller then draws).
template <class Tag>
__device__ __forceinline__ bool finish_ticket(const Params &p, const Ticket &t, const uint4 *buf,
                                              const double *tab)
{
    const int lane = threadIdx.x & 31;
    const bool residual = t.it.mode == kModeResidual;
    for (int s2 = t.c0; s2 < t.c1; ++s2) {
        const uint4 *sb = buf + (s2 - t.c0) * StageShape<Tag>::kPerBuf;
        if (residual) p2_item<Tag, true>(p, t.b, s2, t.it, sb, tab);
        else p2_item<Tag, false>(p, t.b, s2, t.it, sb, tab);
    }
    __threadfence();  // every lane's stores of the ticket precede its count
    __syncwarp();
    unsigned o = 0;
    const unsigned nc = static_cast<unsigned>(t.c1 - t.c0);
    if (lane == 0) {
        o = atomicAdd(&p.p2cnt[t.b], nc) + nc;
        if (o == static_cast<unsigned>(p.S2)) __threadfence();
    }
    return __shfl_sync(kFull, o == static_cast<unsigned>(p.S2) ? 1 : 0, 0) != 0;
}

// The task worker: decide tasks first (claimed from a counter), then pass-2
// tickets, two in flight.
template <class Tag>
__device__ __forceinline__ void fused_tasks(const Params &p, uint4 *region, const double *tab)
{
    const int lane = threadIdx.x & 31;
    constexpr int kBuf = p2_chunk<Tag>() * StageShape<Tag>::kPerBuf;  // uint4 per ticket
    static_assert(2 * kBuf <= kRegion, "two tickets' staging fit a warp region");
    double *W_sh = reinterpret_cast<double *>(region + 2 * kBuf);
    const bool w_shared = 2 * static_cast<size_t>(p.S2) * sizeof(double) <=
                          sizeof(uint4) * static_cast<size_t>(kRegion - 2 * kBuf);
    const unsigned B = static_cast<unsigned>(p.B);
    // decide tasks: a task is claimed only by a free warp, which starts it
    // at once, so no pass-2 worker waits on a decide that nobody runs
#pragma unroll 1
    for (;;) {
        unsigned t = 0;
        if (lane == 0) t = atomicAdd(p.p2claim, 1u);
        t = __shfl_sync(kFull, t, 0);
        if (t >= B) break;
        if (!decide_task<Tag>(p, static_cast<int>(t), region)) return;
    }
    // pass 2: tickets in request order, the next one copied while the
    // current one is reduced
    Ticket none;
    none.valid = false;
    Ticket cur, nxt;
    int q = 0;
    unsigned ahead = 0;
    if (lane == 0) ahead = atomicAdd(p.p2ticket, 1u);
    if (!take_ticket<Tag>(p, cur, none, region, ahead)) return;
#pragma unroll 1
    while (cur.valid) {
        if (!take_ticket<Tag>(p, nxt, cur, region + (q ^ 1) * kBuf, ahead)) {
            wait_copies<0>();
            return;
        }
        wait_copies<1>();  // the current ticket's copies have landed
        if (cur.work && finish_ticket<Tag>(p, cur, region + q * kBuf, tab)) {
            double *W = w_shared ? W_sh : p.p2w + 2 * static_cast<int64_t>(cur.b) * p.S2;
            finalize<Tag>(p, cur.b, tab, W, W + p.S2);
        }
        cur = nxt;
        q ^= 1;
    }
    wait_copies<0>();
}

template <class Tag>
__global__ void __launch_bounds__(kThreads, 2) k_fused(const __grid_constant__ Params p)
{
    extern __shared__ uint4 fdyn[];
    __shared__ double tab[kExp2Tab];
    for (int j = threadIdx.x; j < kExp2Tab; j += kThreads) tab[j] = p.exp2tab[j];
    fused_init(p);
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    uint4 *region = warp < kStreamers ? fdyn + warp * kRegionS
                                      : fdyn + kStreamers * kRegionS + (warp - kStreamers) * kRegion;
    // every warp reaches the grid-wide barrier inside fused_stream
    fused_stream<Tag>(p, region, blockIdx.x * kStreamers + warp, gridDim.x * kStreamers, warp < kStreamers);
    fused_tasks<Tag>(p, region, tab);
}

}  // namespace sv
