// sv_walk.cuh -- greedy verification that reads only the rows it needs.
//
// "Accelerating Sonar through speculation", sections "Target-Draft" and
// "EAGLE": a draft node is kept when its parent is kept and its token is the
// target's top token after the parent; the output is the deepest kept path
// plus the top token after its last node.  Only the rows of kept nodes (and
// the root) can influence that output, so this kernel walks the tree from
// the root and reduces exactly those rows: a linear chain of k drafts stops
// at the first mismatch (n + 1 of the k + 1 rows), a tree reads one row per
// kept node.  The price is a dependent step per level.
//
// One thread-block cluster of CL blocks runs a queue of pending rows for
// the requests it owns (requests cid, cid + ncl, ...; up to A at a time).
// A round takes up to kWalkRows pending rows; every block reduces its slice
// of each row to (max, lowest argmax, NaN seen) and, after one cluster
// barrier, every block merges all CL partials through distributed shared
// memory.  All blocks keep identical copies of the queue and request state:
// every update is computed from the same inputs, and where several threads
// update one record they do it with order-free atomics (OR, max), so no
// second barrier is needed to broadcast it.  The children of a processed
// node whose token equals the row's argmax join the queue; a request is
// done when none of its rows is pending, and rank 0 writes its outputs.
// The bookkeeping between rounds is one warp wide (a lane per request slot).
//
// Node records (parent, token, depth) of the requests in flight are cached
// in shared memory when a request is admitted; depths come from pointer
// jumping (log2 N rounds).  A linear chain is the tree parent(i) = i - 1,
// token(i) = draft i - 1 over the k + 1 target rows of the request.
#pragma once

#include <cooperative_groups.h>

#include "sv_common.cuh"


namespace sv {

constexpr int kWalkRows = 16;    // rows reduced per round (one cluster barrier)
constexpr int kWalkSlots = 32;   // requests in flight per cluster (one warp's lanes)
constexpr int kWalkCache = 2048; // cached node records per block (A * N <= this)
constexpr int kWalkRing = 2048;  // pending rows; a power of two >= kWalkCache
constexpr int kWalkJumps = 12;   // pointer-jumping rounds (2^11 > SPEC_MAX_NODES)
static_assert((kWalkRing & (kWalkRing - 1)) == 0 && kWalkRing >= kWalkCache, "ring size");
static_assert(kWalkCache % kThreads == 0, "cache is scanned in whole block strides");
static_assert(kWalkSlots == 32 && kWalkRows <= 32, "slots and rows are warp lanes");

struct WalkShared {
    float2 part[2][kWalkRows];         // this block's (max or NaN, argmax bits) per row
    float redf[kWarps];
    int redi[kWarps];
    int g[kWalkRows];                  // merged argmax of the round's rows
    int cnt[kWalkRows];                // children queued by the row
    unsigned ring[kWalkRing];          // pending rows: node | slot << 16
    int tok[kWalkCache];               // node token, at slot * N + node
    short par[kWalkCache];             // node parent (-1 for the root)
    short dep[kWalkCache];             // node depth
    short anc[kWalkCache];             // pointer-jumping scratch
    // deepest kept node of the slot's request, as one key whose maximum is
    // the deepest node with the lowest index: depth << 42 | (1023 - node) << 32 | argmax
    unsigned long long best[kWalkSlots];
    int req[kWalkSlots];               // request of the slot, -1 when free
    int pend[kWalkSlots];              // rows of the slot queued or in the round
    int err[kWalkSlots];               // status bits of the request
    int fresh[kWalkSlots];             // slots filled by the last admission, in slot order
    int qh, qt, next, active, nfresh;
};

// Warp 0: requests with no pending row are done (rank 0 writes their
// outputs) and their slots are freed; free slots then take the cluster's
// next requests in slot order.  One lane per slot.
__device__ __forceinline__ void walk_book(const Params &p, WalkShared &sh, int A, int ncl, int rank)
{
    const int lane = threadIdx.x & 31;
    const int N = p.N, W = p.max_depth + 1;
    const unsigned lt = (1u << lane) - 1u;
    const bool in = lane < A;
    const int rq = in ? sh.req[lane] : -1;
    const bool done = in && rq >= 0 && sh.pend[lane] == 0;
    const unsigned dmask = __ballot_sync(kFull, done);
    if (rank == 0) {
        for (unsigned m = dmask; m; m &= m - 1u) {
            const int t = __ffs(m) - 1;
            const int b = __shfl_sync(kFull, rq, t);
            const int err = sh.err[t];
            const unsigned long long key = sh.best[t];
            const int D = err ? -1 : static_cast<int>(key >> 42);
            int32_t *out = p.out + static_cast<int64_t>(b) * W;
            int32_t *path = p.path ? p.path + static_cast<int64_t>(b) * W : nullptr;
            for (int j = D + 1 + lane; j < W; j += 32) {  // past the bonus (everything on an error)
                out[j] = -1;
                if (path) path[j] = -1;
            }
            if (lane == 0) {
                if (err) {
                    p.acc[b] = -1;
                    report(p.status, err);
                } else {
                    const int base = t * N;
                    for (int node = 1023 - static_cast<int>((key >> 32) & 1023u); node > 0;
                         node = sh.par[base + node]) {
                        const int d = sh.dep[base + node];
                        out[d - 1] = sh.tok[base + node];
                        if (path) path[d] = node;
                    }
                    if (path) path[0] = 0;
                    out[D] = static_cast<int>(static_cast<unsigned>(key & 0xFFFFFFFFull));
                    p.acc[b] = D;
                }
            }
        }
    }
    const int next = sh.next;
    const bool free_slot = in && (rq < 0 || done);
    const unsigned fmask = __ballot_sync(kFull, free_slot);
    const int nr = next + __popc(fmask & lt) * ncl;
    const bool fresh = free_slot && nr < p.B;
    const unsigned frmask = __ballot_sync(kFull, fresh);
    if (done) sh.req[lane] = -1;
    if (fresh) {
        sh.req[lane] = nr;
        sh.pend[lane] = 0;
        sh.err[lane] = 0;
        sh.best[lane] = 0ull;
        sh.fresh[__popc(frmask & lt)] = lane;
    }
    __syncwarp();
    if (lane == 0) {
        const int nf = __popc(frmask);
        sh.next = next + nf * ncl;
        sh.active += nf - __popc(dmask);
        sh.nfresh = nf;
    }
}

// Whole block, after an admission: cache the node records of the fresh
// requests, find malformed input (its error bits, and no queued row), and
// queue the roots of the others.
__device__ __forceinline__ void walk_load(const Params &p, WalkShared &sh, bool chain)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = p.N, E = sh.nfresh * N;
    for (int x = tid; x < E; x += kThreads) {
        const int f = x / N, i = x - f * N;
        const int s = sh.fresh[f], e = s * N + i;
        const int b = sh.req[s];
        int par = i - 1, tk = 0, bits = 0;
        if (chain) {  // the chain of a linear request: parent i - 1, token = draft i - 1
            if (i > 0) {
                tk = __ldg(p.tokens + static_cast<int64_t>(b) * p.k + (i - 1));
                if (tk < 0 || tk >= p.V) bits |= kStToken;
            }
        } else {
            par = __ldg(p.parents + static_cast<int64_t>(b) * N + i);
            if (i == 0) {
                if (par != -1) bits |= kStTree;
            } else if (par < 0 || par >= i) {
                bits |= kStTree;
            } else {
                tk = __ldg(p.tokens + static_cast<int64_t>(b) * N + i);
                if (tk < 0 || tk >= p.V) bits |= kStToken;
            }
        }
        const bool ok = (i > 0) && !(bits & kStTree);
        sh.tok[e] = tk;
        sh.par[e] = static_cast<short>(ok ? par : -1);
        sh.anc[e] = static_cast<short>(ok ? par : 0);
        sh.dep[e] = static_cast<short>(chain ? i : (i > 0 ? 1 : 0));
        if (bits) atomicOr(&sh.err[s], bits);
    }
    __syncthreads();

    // depths by pointer jumping: dep[e] is the distance from node e to
    // anc[e]; each round doubles the jump, and a jump that reached the root
    // is final
    if (!chain) {
        constexpr int kPer = kWalkCache / kThreads;
        auto entry = [&](int x) {
            const int f = x / N;
            return sh.fresh[f] * N + (x - f * N);
        };
#pragma unroll 1
        for (int round = 0; round < kWalkJumps; ++round) {
            short nd[kPer], na[kPer];
            int more = 0;
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int x = tid + j * kThreads;
                nd[j] = na[j] = 0;
                if (x < E) {
                    const int e = entry(x);
                    const int a = sh.anc[e];
                    nd[j] = sh.dep[e];
                    na[j] = static_cast<short>(a);
                    if (a != 0) {
                        const int base = e - (x % N);
                        nd[j] = static_cast<short>(nd[j] + sh.dep[base + a]);
                        na[j] = sh.anc[base + a];
                        more |= (na[j] != 0);
                    }
                }
            }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int x = tid + j * kThreads;
                if (x < E) {
                    const int e = entry(x);
                    sh.dep[e] = nd[j];
                    sh.anc[e] = na[j];
                }
            }
            if (!__syncthreads_or(more)) break;
        }
        // a node deeper than max_depth is a malformed tree (checked only
        // when the parent array itself is well formed)
        for (int x = tid; x < E; x += kThreads) {
            const int e = entry(x), s = sh.fresh[x / N];
            if (!(sh.err[s] & kStTree) && sh.dep[e] > p.max_depth) atomicOr(&sh.err[s], kStTree);
        }
        __syncthreads();
    }
    if (warp == 0) {
        const int F = sh.nfresh;
        const int s = lane < F ? sh.fresh[lane] : 0;
        const bool ok = lane < F && sh.err[s] == 0;
        const unsigned m = __ballot_sync(kFull, ok);
        const int qt = sh.qt;
        if (ok) {
            sh.ring[(qt + __popc(m & ((1u << lane) - 1u))) & (kWalkRing - 1)] = static_cast<unsigned>(s) << 16;
            sh.pend[s] = 1;
        }
        __syncwarp();
        if (lane == 0) sh.qt = qt + __popc(m);
    }
    __syncthreads();
}

template <class Tag, int CL>
__global__ void __launch_bounds__(kThreads) k_greedy_walk(const Params p, int slice, int A, int chain_i)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    constexpr int U = 4;
    constexpr int kChunk = kThreads * kVec * U;  // entries of a slice read per step
    static_assert(kWalkRows * CL <= kThreads && 32 % CL == 0, "merge layout");

    __shared__ WalkShared sh;
    const bool chain = chain_i != 0;
    const int rank = static_cast<int>(cluster.block_rank());
    const int cid = blockIdx.x / CL, ncl = gridDim.x / CL;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = p.N;
    const int s_begin = min(p.V, rank * slice), s_end = min(p.V, s_begin + slice);
    const int iters = max(1, (s_end - s_begin + kChunk - 1) / kChunk);

    for (int s = tid; s < kWalkSlots; s += kThreads) {
        sh.req[s] = -1;
        sh.pend[s] = 0;
    }
    if (tid == 0) {
        sh.qh = sh.qt = 0;
        sh.next = cid;
        sh.active = 0;
    }
    __syncthreads();

    auto slot_node = [&](int qh, int r, int &s) {
        const unsigned e = sh.ring[(qh + r) & (kWalkRing - 1)];
        s = static_cast<int>(e >> 16);
        return static_cast<int>(e & 0xFFFFu);
    };
    auto row_of = [&](int qh, int r) {
        int s;
        const int node = slot_node(qh, r, s);
        return static_cast<const char *>(p.tl) +
               (static_cast<int64_t>(sh.req[s]) * N + node) * p.stride * kEsz;
    };
    auto load = [&](const char *row, int it, uint4 (&raw)[U]) {
        const int base = s_begin + it * kChunk;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e0 = base + (tid + u * kThreads) * kVec;
            raw[u] = e0 < s_end ? ldg_vec(row + static_cast<int64_t>(e0) * kEsz)
                                : make_uint4(Tag::kNegInfWord, Tag::kNegInfWord, Tag::kNegInfWord,
                                             Tag::kNegInfWord);
        }
    };

    // every iteration admits or completes requests or reduces at least one
    // row, so the loop ends within (requests owned) * (N + 1) + 2
    // iterations; the bound guards the cluster barriers against a logic error
    const int owned = cid < p.B ? (p.B - cid + ncl - 1) / ncl : 0;
    const int64_t limit = static_cast<int64_t>(owned) * (N + 1) + 4;
    int64_t iter = 0;
    int buf = 0;
#pragma unroll 1
    for (;;) {
        if (++iter > limit) {  // identical in every block of the cluster
            if (rank == 0 && tid == 0) report(p.status, kStTimeout);
            break;
        }
        if (warp == 0) walk_book(p, sh, A, ncl, rank);
        __syncthreads();
        if (sh.nfresh) walk_load(p, sh, chain);
        const int qh = sh.qh, qt = sh.qt;
        const bool done = sh.active == 0 && sh.next >= p.B;
        __syncthreads();  // all threads hold the control state before it changes
        if (done) break;
        if (qh == qt) continue;
        const int nb = min(kWalkRows, qt - qh);

        // this block's slice of each row of the round, reads one step ahead
        {
            int r = 0, it = 0;
            const char *row = row_of(qh, 0);
            uint4 cur[U], nxt[U];
            load(row, 0, cur);
            float best = -INFINITY;
            int idx = INT_MAX;
            bool nan = false;
#pragma unroll 1
            for (;;) {
                int nr = r, nit = it + 1;
                const char *nrow = row;
                if (nit == iters) {
                    nit = 0;
                    if (++nr < nb) nrow = row_of(qh, nr);
                }
                if (nr < nb) load(nrow, nit, nxt);
                const int base = s_begin + it * kChunk;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int e0 = base + (tid + u * kThreads) * kVec;
                    uint4 raw = cur[u];
                    if (e0 < s_end && e0 + kVec > s_end) raw = mask_tail<Tag>(raw, s_end - e0);
                    float x[kVec];
                    unpack<Tag>(raw, x);
#pragma unroll
                    for (int e = 0; e < kVec; ++e) {
                        nan |= (x[e] != x[e]);
                        if (x[e] > best) {
                            best = x[e];
                            idx = e0 + e;
                        }
                    }
                }
                if (it == iters - 1) {  // row r of the round: merge the block
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const float ov = __shfl_xor_sync(kFull, best, o);
                        const int oi = __shfl_xor_sync(kFull, idx, o);
                        argmax_take(best, idx, ov, oi);
                    }
                    const int any_nan = __syncthreads_or(nan ? 1 : 0);
                    if (lane == 0) {
                        sh.redf[warp] = best;
                        sh.redi[warp] = idx;
                    }
                    __syncthreads();
                    if (tid == 0) {
                        float bv = sh.redf[0];
                        int bi = sh.redi[0];
                        for (int w = 1; w < kWarps; ++w) argmax_take(bv, bi, sh.redf[w], sh.redi[w]);
                        sh.part[buf][r] =
                            make_float2(any_nan ? __int_as_float(0x7FC00000) : bv, __int_as_float(bi));
                    }
                    best = -INFINITY;
                    idx = INT_MAX;
                    nan = false;
                }
                if (nr >= nb) break;
#pragma unroll
                for (int u = 0; u < U; ++u) cur[u] = nxt[u];
                r = nr;
                it = nit;
                row = nrow;
            }
        }
        cluster.sync();  // every block's partials of the round are visible

        // merge: CL lanes per row (the argmax rule does not depend on the
        // order); the row's lead lane records errors and the deepest node
        if (tid < kWalkRows * CL) {
            const int r = tid / CL, rr = tid % CL;
            float bv = -INFINITY;
            int bi = INT_MAX, nn = 0;
            if (r < nb) {
                const float2 v = cluster.map_shared_rank(&sh.part[buf][0], rr)[r];
                if (v.x != v.x) nn = 1;
                else {
                    bv = v.x;
                    bi = __float_as_int(v.y);
                }
            }
#pragma unroll
            for (int o = CL / 2; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(kFull, bv, o);
                const int oi = __shfl_xor_sync(kFull, bi, o);
                nn |= __shfl_xor_sync(kFull, nn, o);
                argmax_take(bv, bi, ov, oi);
            }
            if (rr == 0 && r < nb) {
                const int g = (bi == INT_MAX) ? 0 : bi;  // an all -inf row has argmax 0
                sh.g[r] = g;
                int s;
                const int node = slot_node(qh, r, s);
                if (nn) atomicOr(&sh.err[s], kStLogit);
                const unsigned long long key =
                    (static_cast<unsigned long long>(sh.dep[s * N + node]) << 42) |
                    (static_cast<unsigned long long>(1023 - node) << 32) | static_cast<unsigned>(g);
                atomicMax(&sh.best[s], key);
            }
        }
        __syncthreads();

        // kept children of each row, queued in (row, index) order: a warp
        // per row counts them, then writes them at its prefix offset
        for (int pass = 0; pass < 2; ++pass) {
            for (int r = warp; r < nb; r += kWarps) {
                int s;
                const int node = slot_node(qh, r, s);
                const int base = s * N, g = sh.g[r];
                const bool live = sh.err[s] == 0;
                int off = qt;
                if (pass == 1) {
                    int sum = lane < r ? sh.cnt[lane] : 0;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
                    off += sum;
                }
                int count = 0;
                for (int c0 = node + 1; c0 < N; c0 += 32) {
                    const int c = c0 + lane;
                    const bool kept = live && c < N && sh.par[base + c] == node && sh.tok[base + c] == g;
                    const unsigned m = __ballot_sync(kFull, kept);
                    if (pass == 1 && kept)
                        sh.ring[(off + count + __popc(m & ((1u << lane) - 1u))) & (kWalkRing - 1)] =
                            static_cast<unsigned>(c) | (static_cast<unsigned>(s) << 16);
                    count += __popc(m);
                }
                if (lane == 0) {
                    if (pass == 0) sh.cnt[r] = count;
                    else atomicAdd(&sh.pend[s], count - 1);  // the row is done, its children pending
                }
            }
            if (pass == 1 && tid == 0) {
                int total = 0;
                for (int r = 0; r < nb; ++r) total += sh.cnt[r];
                sh.qh = qh + nb;
                sh.qt = qt + total;
            }
            __syncthreads();
        }
        buf ^= 1;
    }
    cluster.sync();  // no block leaves while another may still read its partials
}

}  // namespace sv
