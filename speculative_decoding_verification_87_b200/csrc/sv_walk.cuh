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
// every update is computed from the same inputs in the same order, so no
// second barrier is needed to broadcast it.  The children of a processed
// node whose token equals the row's argmax join the queue; a request is
// done when none of its rows is pending, and rank 0 writes its outputs.
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
constexpr int kWalkSlots = 32;   // requests in flight per cluster
constexpr int kWalkCache = 2048; // cached node records per block (A * N <= this)
constexpr int kWalkRing = 2048;  // pending rows; a power of two >= kWalkCache
constexpr int kWalkJumps = 12;   // pointer-jumping rounds (2^11 > SPEC_MAX_NODES)
static_assert((kWalkRing & (kWalkRing - 1)) == 0 && kWalkRing >= kWalkCache, "ring size");
static_assert(kWalkCache % kThreads == 0, "cache is scanned in whole block strides");

struct WalkShared {
    float2 part[2][kWalkRows];         // this block's (max or NaN, argmax bits) per row
    float redf[kWarps];
    int redi[kWarps];
    int g[kWalkRows];                  // merged argmax of the round's rows
    int nan[kWalkRows];                // a NaN was seen in the row
    int cnt[kWalkRows];                // children queued by the row
    unsigned ring[kWalkRing];          // pending rows: node | slot << 16
    int tok[kWalkCache];               // node token, at slot * N + node
    short par[kWalkCache];             // node parent (-1 for the root)
    short dep[kWalkCache];             // node depth
    short anc[kWalkCache];             // pointer-jumping scratch
    int req[kWalkSlots];               // request of the slot, -1 when free
    int pend[kWalkSlots];              // rows of the slot queued or in the round
    int err[kWalkSlots];               // status bits of the request
    int bd[kWalkSlots], bn[kWalkSlots], bg[kWalkSlots];  // deepest kept node: depth, index, argmax
    int fresh[kWalkSlots];             // admitted by the current admission pass
    int qh, qt, next, active, any_fresh;
};

// Fill free slots with the cluster's next requests and cache their node
// records; requests with malformed input get their error bits here (and no
// queued row); the others queue their root.
__device__ __forceinline__ void walk_admit(const Params &p, WalkShared &sh, int A, int ncl,
                                           bool chain)
{
    const int tid = threadIdx.x;
    const int N = p.N;
    if (tid == 0) {
        int any = 0;
        for (int s = 0; s < A; ++s) {
            sh.fresh[s] = 0;
            if (sh.req[s] < 0 && sh.next < p.B) {
                sh.req[s] = sh.next;
                sh.next += ncl;
                sh.fresh[s] = 1;
                sh.err[s] = 0;
                sh.pend[s] = 0;
                sh.bd[s] = -1;
                sh.bn[s] = 0;
                sh.bg[s] = 0;
                ++sh.active;
                any = 1;
            }
        }
        sh.any_fresh = any;
    }
    __syncthreads();
    if (!sh.any_fresh) return;  // block-uniform

    // node records of the fresh slots (a chain's are implicit but cached alike)
    for (int e = tid; e < A * N; e += kThreads) {
        const int s = e / N, i = e - s * N;
        if (!sh.fresh[s]) continue;
        const int b = sh.req[s];
        int par = i - 1, tk = 0, bits = 0;
        if (chain) {
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

    // depths: dep[e] is the distance from node e to anc[e]; each round
    // doubles the jump, and a node whose jump reached the root is final
    if (!chain) {
        constexpr int kPer = kWalkCache / kThreads;
#pragma unroll 1
        for (int round = 0; round < kWalkJumps; ++round) {
            short nd[kPer], na[kPer];
            int more = 0;
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int e = tid + j * kThreads;
                nd[j] = na[j] = 0;
                if (e < A * N) {
                    const int s = e / N;
                    const int a = sh.anc[e];
                    nd[j] = sh.dep[e];
                    na[j] = static_cast<short>(a);
                    if (sh.fresh[s] && a != 0) {
                        const int base = s * N;
                        nd[j] = static_cast<short>(nd[j] + sh.dep[base + a]);
                        na[j] = sh.anc[base + a];
                        more |= (na[j] != 0);
                    }
                }
            }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int e = tid + j * kThreads;
                if (e < A * N) {
                    sh.dep[e] = nd[j];
                    sh.anc[e] = na[j];
                }
            }
            if (!__syncthreads_or(more)) break;
        }
        // a node deeper than max_depth is a malformed tree (checked only
        // when the parent array itself is well formed)
        for (int e = tid; e < A * N; e += kThreads) {
            const int s = e / N;
            if (sh.fresh[s] && !(sh.err[s] & kStTree) && sh.dep[e] > p.max_depth)
                atomicOr(&sh.err[s], kStTree);
        }
        __syncthreads();
    }
    if (tid == 0) {
        for (int s = 0; s < A; ++s) {
            if (sh.fresh[s] && !sh.err[s]) {
                sh.ring[sh.qt & (kWalkRing - 1)] = static_cast<unsigned>(s) << 16;  // the root
                ++sh.qt;
                sh.pend[s] = 1;
            }
        }
    }
    __syncthreads();
}

// Requests with no pending row are done: rank 0 writes their outputs, every
// block frees their slots.
__device__ __forceinline__ void walk_complete(const Params &p, WalkShared &sh, int A, int rank)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = p.N, W = p.max_depth + 1;
    if (rank == 0) {
        for (int s = warp; s < A; s += kWarps) {
            if (sh.req[s] < 0 || sh.pend[s] != 0) continue;
            const int b = sh.req[s];
            const int err = sh.err[s];
            const int D = err ? -1 : sh.bd[s];
            int32_t *out = p.out + static_cast<int64_t>(b) * W;
            int32_t *path = p.path ? p.path + static_cast<int64_t>(b) * W : nullptr;
            // entries past the bonus (all of them on an error)
            for (int j = D + 1 + lane; j < W; j += 32) {
                out[j] = -1;
                if (path) path[j] = -1;
            }
            if (lane == 0) {
                if (err) {
                    p.acc[b] = -1;
                    report(p.status, err);
                } else {
                    const int base = s * N;
                    for (int node = sh.bn[s]; node > 0; node = sh.par[base + node]) {
                        const int d = sh.dep[base + node];
                        out[d - 1] = sh.tok[base + node];
                        if (path) path[d] = node;
                    }
                    if (path) path[0] = 0;
                    out[D] = sh.bg[s];
                    p.acc[b] = D;
                }
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        for (int s = 0; s < A; ++s) {
            if (sh.req[s] >= 0 && sh.pend[s] == 0) {
                sh.req[s] = -1;
                --sh.active;
            }
        }
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

    for (int s = tid; s < kWalkSlots; s += kThreads) sh.req[s] = -1;
    if (tid == 0) {
        sh.qh = sh.qt = 0;
        sh.next = cid;
        sh.active = 0;
    }
    __syncthreads();

    auto row_of = [&](int qh, int r) {
        const unsigned e = sh.ring[(qh + r) & (kWalkRing - 1)];
        const int node = static_cast<int>(e & 0xFFFFu), s = static_cast<int>(e >> 16);
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

    // every iteration admits requests or reduces at least one row, so the
    // loop ends within (requests owned) * (N + 1) + 2 iterations; the bound
    // guards the cluster barriers against a logic error
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
        walk_admit(p, sh, A, ncl, chain);
        walk_complete(p, sh, A, rank);  // requests rejected at admission
        const int qh = sh.qh, qt = sh.qt;
        const bool done = sh.active == 0 && sh.next >= p.B;
        __syncthreads();  // all threads hold the control state before thread 0 changes it
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

        // merge: CL lanes per row, in slice order (the argmax rule does not
        // depend on the order)
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
                sh.g[r] = (bi == INT_MAX) ? 0 : bi;  // an all -inf row has argmax 0
                sh.nan[r] = nn;
            }
        }
        __syncthreads();

        // errors and the deepest kept node, in queue order
        if (tid == 0) {
            for (int r = 0; r < nb; ++r) {
                const unsigned e = sh.ring[(qh + r) & (kWalkRing - 1)];
                const int node = static_cast<int>(e & 0xFFFFu), s = static_cast<int>(e >> 16);
                if (sh.nan[r]) sh.err[s] |= kStLogit;
                const int d = sh.dep[s * N + node];
                if (d > sh.bd[s] || (d == sh.bd[s] && node < sh.bn[s])) {
                    sh.bd[s] = d;
                    sh.bn[s] = node;
                    sh.bg[s] = sh.g[r];
                }
            }
        }
        __syncthreads();

        // kept children of each row, queued in (row, index) order: a warp
        // per row counts them, then writes them at its prefix offset
        for (int pass = 0; pass < 2; ++pass) {
            for (int r = warp; r < nb; r += kWarps) {
                const unsigned e = sh.ring[(qh + r) & (kWalkRing - 1)];
                const int node = static_cast<int>(e & 0xFFFFu), s = static_cast<int>(e >> 16);
                const int base = s * N, g = sh.g[r];
                const bool live = sh.err[s] == 0;
                int off = qt;
                if (pass == 1) {
                    const int c = lane < r ? sh.cnt[lane] : 0;  // r < kWalkRows <= 32
                    int sum = c;
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
                if (pass == 0 && lane == 0) sh.cnt[r] = count;
            }
            __syncthreads();
        }
        if (tid == 0) {
            int total = 0;
            for (int r = 0; r < nb; ++r) {
                const int s = static_cast<int>(sh.ring[(qh + r) & (kWalkRing - 1)] >> 16);
                sh.pend[s] += sh.cnt[r] - 1;
                total += sh.cnt[r];
            }
            sh.qh = qh + nb;
            sh.qt = qt + total;
        }
        __syncthreads();
        walk_complete(p, sh, A, rank);
        buf ^= 1;
    }
    cluster.sync();  // no block leaves while another may still read its partials
}

}  // namespace sv
