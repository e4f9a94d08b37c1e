// sv_exact.cuh -- distribution-exact stochastic tree verification.
//
// "Accelerating Sonar through speculation", section "EAGLE": drafts form a
// tree of top-K candidates and the longest acceptable sequence is kept, plus
// one target token; "Speculative decoding explained", section "Draft and
// verification loop": a rejected draft is replaced by a token from an
// adjusted distribution, which keeps the target's distribution.  Applied to
// one sibling after another (Leviathan et al.'s rule, repeated): walk from
// the root; at node u the children are tested in index order against the
// current distribution p, with q_u the draft row u's children were drawn
// from; an accepted child becomes the node (p = its target row); a rejected
// child replaces p by norm(max(0, p - q_u)); with no child left the token is
// drawn from the current p.
//
// Closed form used here: after r rejections at a node the current
// distribution is max(0, p - c_r q) / D_r with c_1 = 1, c_{r+1} = c_r + D_r
// and D_r = sum_v max(0, p(v) - c_r q(v)) (p, q the node's normalised target
// and draft rows): one scalar pair per rejection instead of a V-entry row.
//
// One thread-block cluster of kExactCluster blocks owns a request at a time.
// Every block keeps an identical copy of the walk (every thread computes the
// same scalars from the same inputs), and each owns one contiguous slice of
// the vocabulary for the fp64 sweeps the walk needs:
//   * after the first rejection at a node: the exact normalisers E = sum e,
//     F = sum f of the node's target and draft rows (e, f: exp((l - max)/T));
//   * after every rejection: D = sum max(0, e/E - c f/F);
//   * at the end: the weights of the draw (e, or the residual) and an
//     inverse CDF refined slice -> thread chunk -> entry.
// A sweep's block totals are exchanged through distributed shared memory
// after one cluster barrier and summed in rank order, so every block holds
// the same fp64 values.  The pass-1 row statistics (k_pass1) give the first
// test at each node, as in the independent-test tree mode.
#pragma once

#include <cooperative_groups.h>

#include "sv_verify.cuh"

namespace sv {

constexpr int kExactCluster = 8;

struct ExactShared {
    double s[2 * kMaxNodes];  // merged row sums: target rows [0, N), draft rows [N, 2N)
    float m[2 * kMaxNodes];   // merged row maxima
    TreeScratch ts;           // depth, flags (bit 1: has a child)
    double wsum[kWarps];      // block reduction scratch
    double2 xchg[2];          // this block's totals of the last two sweeps (read by the cluster)
    double tsum[kThreads];    // per-thread chunk sums of the draw sweep
    double before;            // the draw: running sum before the chosen thread's chunk
    unsigned char finite[2 * kMaxNodes];  // a row has a partial with a finite max
    unsigned char merged[kMaxNodes];      // node's rows merged into s, m
    int bad;                  // a partial holds NaN or +inf
    int err;
    int sel;                  // the draw: the chosen thread
};

// This thread's entries of the slice: [lo, hi), contiguous, whole vectors.
struct ExactChunk {
    int lo, hi;
};

// One sweep over this thread's entries of target row toff (and draft row
// doff when two): f(xt, xd) -> double2 per entry, summed in index order.
template <class Tag, bool kTwo, class F>
__device__ __forceinline__ double2 chunk_sweep(const Params &p, const ExactChunk &ch, int64_t toff,
                                               int64_t doff, F f)
{
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    constexpr int kB = 4;  // vectors loaded together (their latencies overlap)
    const char *trow = static_cast<const char *>(p.tl) + toff * kEsz;
    const char *drow = static_cast<const char *>(p.dl) + doff * kEsz;
    double2 acc = make_double2(0.0, 0.0);
    for (int e0 = ch.lo; e0 < ch.hi; e0 += kB * kVec) {
        uint4 tv[kB], dv[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int e = e0 + u * kVec;
            tv[u] = e < ch.hi ? ldg_vec(trow + static_cast<int64_t>(e) * kEsz) : make_uint4(0, 0, 0, 0);
            dv[u] = (kTwo && e < ch.hi) ? ldg_vec(drow + static_cast<int64_t>(e) * kEsz) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int e = e0 + u * kVec;
            if (e >= ch.hi) break;
            uint4 a = tv[u], d = dv[u];
            if (e + kVec > p.V) {
                a = mask_tail<Tag>(a, p.V - e);
                if (kTwo) d = mask_tail<Tag>(d, p.V - e);
            }
            float xt[kVec], xd[kVec];
            unpack<Tag>(a, xt);
            if (kTwo) unpack<Tag>(d, xd);
#pragma unroll
            for (int i = 0; i < kVec; ++i) {
                const double2 w = f(xt[i], kTwo ? xd[i] : 0.f);
                acc.x += w.x;
                acc.y += w.y;
            }
        }
    }
    return acc;
}

// Block totals (lane 0 of each warp, warps in order), published to the
// cluster; after one cluster barrier every thread sums the blocks' totals
// in rank order.  xb: the exchange buffer of this sweep (alternates).
template <int CL>
__device__ __forceinline__ double2 cluster_total(ExactShared &sh, double2 v, int &xb)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const double a = warp_sum(v.x), b = warp_sum(v.y);
    if (lane == 0) {
        sh.wsum[warp] = a;
        sh.tsum[warp] = b;  // tsum is free outside the draw sweep
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double ta = 0.0, tb = 0.0;
        for (int w = 0; w < kWarps; ++w) {
            ta += sh.wsum[w];
            tb += sh.tsum[w];
        }
        sh.xchg[xb] = make_double2(ta, tb);
    }
    cluster.sync();
    double2 t = make_double2(0.0, 0.0);
    for (int r = 0; r < CL; ++r) {
        const double2 o = *cluster.map_shared_rank(&sh.xchg[xb], r);
        t.x += o.x;
        t.y += o.y;
    }
    xb ^= 1;
    return t;
}

// The first index of W[0, n) with positive weight whose running sum
// (starting at 0, index order) exceeds target; if rounding leaves none, the
// last index with positive weight (-1 if none).  One thread.
__device__ __forceinline__ int icdf_seq(const double *W, int n, double target, double &before)
{
    double run = 0.0, lastb = 0.0;
    int last = -1;
    for (int i = 0; i < n; ++i) {
        const double w = W[i];
        if (w > 0.0) {
            if (run + w > target) {
                before = run;
                return i;
            }
            last = i;
            lastb = run;
        }
        run += w;
    }
    before = lastb;
    return last;
}

template <class Tag, int CL>
__global__ void __launch_bounds__(kThreads) k_tree_exact(const __grid_constant__ Params p, int slice,
                                                          int chunk)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ ExactShared sh;
    __shared__ double tab[kExp2Tab];
    constexpr int kVec = Tag::kVec;
    const int rank = static_cast<int>(cluster.block_rank());
    const int cid = blockIdx.x / CL, ncl = gridDim.x / CL;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = p.N, W = p.max_depth + 1;
    for (int j = tid; j < kExp2Tab; j += kThreads) tab[j] = p.exp2tab[j];
    // pass 1 complete and its partials visible
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    __syncthreads();
    const int s_lo = min(p.V, rank * slice), s_hi = min(p.V, s_lo + slice);
    ExactChunk ch;
    ch.lo = min(s_hi, s_lo + tid * chunk);
    ch.hi = min(s_hi, ch.lo + chunk);
    int xb = 0;
    RowStats rs;
    rs.s = sh.s;
    rs.m = sh.m;
    rs.idx = nullptr;

#pragma unroll 1
    for (int b = cid; b < p.B; b += ncl) {
        const int32_t *pa = p.parents + static_cast<int64_t>(b) * N;
        const int32_t *tk = p.tokens + static_cast<int64_t>(b) * N;
        // children flags
        for (int i = tid; i < N; i += kThreads) sh.ts.flag[i] = 0;
        __syncthreads();
        for (int i = 1 + tid; i < N; i += kThreads) {
            const int par = __ldg(pa + i);
            if (par >= 0 && par < i) sh.ts.flag[par] = 1;
        }
        __syncthreads();
        // every row the mode reads (each target row, the draft rows of nodes
        // with children) must have a finite normaliser: no partial holds a
        // NaN or +inf, and some partial's max is finite (a partial with a
        // finite max has a sum of at least 1).  Checked on the partials, in
        // parallel; rows are merged only when the walk reaches their node.
        if (tid == 0) sh.bad = 0;
        for (int i = tid; i < 2 * N; i += kThreads) sh.finite[i] = 0;
        __syncthreads();
        {
            const float2 *part = p.rowpart + static_cast<int64_t>(b) * p.R * p.S;
            int bad = 0;
            constexpr int kB = 8;  // partials loaded together (their latencies overlap)
            const int total = 2 * N * p.S;
            for (int i0 = tid; i0 < total; i0 += kB * kThreads) {
                float2 v[kB];
                int rr[kB];
#pragma unroll
                for (int u = 0; u < kB; ++u) {
                    const int i = i0 + u * kThreads;
                    rr[u] = -1;
                    if (i < total) {
                        const int r = i / p.S;
                        if (r < N || (sh.ts.flag[r - N] & 1)) {
                            rr[u] = r;
                            v[u] = __ldcg(part + i);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < kB; ++u) {
                    if (rr[u] < 0) continue;
                    if (v[u].x != v[u].x || v[u].y != v[u].y || v[u].x == INFINITY) bad = 1;
                    else if (v[u].x != -INFINITY) sh.finite[rr[u]] = 1;
                }
            }
            if (bad) sh.bad = 1;
            for (int i = tid; i < N; i += kThreads) sh.merged[i] = 0;
        }
        __syncthreads();
        // tree, token and row checks (warp 0), as the independent-test mode
        if (warp == 0) {
            int err = 0;
            for (int i = lane; i < N; i += 32) {
                const int par = __ldg(pa + i);
                if (i == 0) {
                    if (par != -1) err |= kStTree;
                } else if (par < 0 || par >= i) {
                    err |= kStTree;
                } else {
                    const int t = __ldg(tk + i);
                    if (t < 0 || t >= p.V) err |= kStToken;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) err |= __shfl_xor_sync(kFull, err, o);
            if (lane == 0 && !(err & kStTree)) {
                sh.ts.depth[0] = 0;
                for (int i = 1; i < N; ++i) {
                    const int d = sh.ts.depth[__ldg(pa + i)] + 1;
                    sh.ts.depth[i] = static_cast<short>(d);
                    if (d > p.max_depth) err |= kStTree;
                }
            }
            err = __shfl_sync(kFull, err, 0);
            bool bad = sh.bad != 0;
            if (!(err & kStTree))
                for (int r = lane; r < 2 * N; r += 32) {
                    if (r >= N && !(sh.ts.flag[r - N] & 1)) continue;
                    bad |= !sh.finite[r];
                }
            if (__any_sync(kFull, bad)) err |= kStLogit;
            if (lane == 0) sh.err = err;
        }
        __syncthreads();
        const int err = sh.err;
        if (err) {
            if (rank == 0) {
                for (int j = tid; j < W; j += kThreads) {
                    p.out[static_cast<int64_t>(b) * W + j] = -1;
                    if (p.path) p.path[static_cast<int64_t>(b) * W + j] = -1;
                }
                if (tid == 0) {
                    p.acc[b] = -1;
                    report(p.status, err);
                }
            }
            __syncthreads();
            continue;
        }

        // the walk (every thread computes the same values)
        int u = 0;          // current node
        int last = 0;       // children of u are scanned past this index
        int rej = 0;        // rejections at u that changed p
        double c = 0.0, D = 1.0;  // current p = max(0, p_u - c q_u) / D  (c = 0: p_u)
        bool exact = false;       // E, F known for u
        double E = 0.0, F = 0.0;
        // the merged statistics of node u's target and draft rows, once
        auto need = [&](int node) {
            if (!sh.merged[node]) {
                if (warp == 0) merge_row<kTreeStochastic>(p, b, node, rs);
                else if (warp == 1 && (sh.ts.flag[node] & 1)) merge_row<kTreeStochastic>(p, b, N + node, rs);
                __syncthreads();
                if (tid == 0) sh.merged[node] = 1;
                __syncthreads();
            }
        };
#pragma unroll 1
        for (;;) {
            need(u);
            // next child of u in index order (warp-wide ballots, every warp alike)
            int chn = -1;
            for (int base = last + 1; base < N && chn < 0; base += 32) {
                const int i = base + lane;
                const unsigned hit = __ballot_sync(kFull, i < N && __ldg(pa + i) == u);
                if (hit) chn = base + __ffs(hit) - 1;
            }
            if (chn < 0) break;
            last = chn;
            const int t = __ldg(tk + chn);
            const int64_t off_u = (static_cast<int64_t>(b) * N + u) * p.stride;
            const double lt = logit_f64_at<Tag>(p.tl, off_u + t);
            const double ld = logit_f64_at<Tag>(p.dl, off_u + t);
            double lp, lq;
            if (rej == 0) {
                lp = (lt - static_cast<double>(sh.m[u])) * p.inv_t - log(sh.s[u]);
                lq = (ld - static_cast<double>(sh.m[N + u])) * p.inv_t - log(sh.s[N + u]);
            } else {
                const double pt = exp((lt - static_cast<double>(sh.m[u])) * p.inv_t) / E;
                const double qt = exp((ld - static_cast<double>(sh.m[N + u])) * p.inv_t) / F;
                const double pr = pt - c * qt;
                lp = pr > 0.0 ? log(pr / D) : -INFINITY;
                lq = log(qt);
            }
            const double ua = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(chn - 1),
                                             kPurposeAccept, p.offset);
            if (accept_test(lp, lq, ua)) {
                u = chn;
                last = chn;
                rej = 0;
                c = 0.0;
                D = 1.0;
                exact = false;
                continue;
            }
            // rejected: the residual of the current p against q_u
            const double nmt = neg_mc(p, sh.m[u]), nmd = neg_mc(p, sh.m[N + u]);
            const int64_t toff = off_u, doff = off_u;
            if (!exact) {
                const double2 ef = chunk_sweep<Tag, true>(p, ch, toff, doff, [&](float xt, float xd) {
                    return make_double2(exp2_fp64(entry_z(p, xt, nmt), tab), exp2_fp64(entry_z(p, xd, nmd), tab));
                });
                const double2 tot = cluster_total<CL>(sh, ef, xb);
                E = tot.x;
                F = tot.y;
                exact = true;
            }
            const double cn = (rej == 0) ? 1.0 : c + D;
            const double isp = 1.0 / E, isq = cn / F;
            const double2 dr = chunk_sweep<Tag, true>(p, ch, toff, doff, [&](float xt, float xd) {
                const double pp = exp2_fp64(entry_z(p, xt, nmt), tab) * isp;
                const double qq = exp2_fp64(entry_z(p, xd, nmd), tab) * isq;
                return make_double2(pp > qq ? pp - qq : 0.0, 0.0);
            });
            const double Dn = cluster_total<CL>(sh, dr, xb).x;
            if (Dn > 0.0) {  // a zero mass (rounding only) leaves p unchanged
                c = cn;
                D = Dn;
                ++rej;
            }
        }

        // the draw at u: weights e (no rejection) or max(0, e/E - c f/F)
        need(u);
        const int64_t off_u = (static_cast<int64_t>(b) * N + u) * p.stride;
        const double nmt = neg_mc(p, sh.m[u]), nmd = neg_mc(p, sh.m[N + u]);
        const double isp = rej ? 1.0 / E : 1.0, isq = rej ? c / F : 0.0;
        auto weight = [&](float xt, float xd) {
            const double et = exp2_fp64(entry_z(p, xt, nmt), tab);
            if (!rej) return et;
            const double pp = et * isp, qq = exp2_fp64(entry_z(p, xd, nmd), tab) * isq;
            return pp > qq ? pp - qq : 0.0;
        };
        double mine;
        if (rej) mine = chunk_sweep<Tag, true>(p, ch, off_u, off_u, [&](float xt, float xd) { return make_double2(weight(xt, xd), 0.0); }).x;
        else mine = chunk_sweep<Tag, false>(p, ch, off_u, off_u, [&](float xt, float xd) { return make_double2(weight(xt, xd), 0.0); }).x;
        const double Z = cluster_total<CL>(sh, make_double2(mine, 0.0), xb).x;
        // the block totals are still in every block's exchange slot: pick the
        // block (the same in every block), then, inside it, the thread chunk
        // and the entry, each the first with positive weight whose running
        // sum passes the target (if rounding leaves none, the last positive)
        const int xr = xb ^ 1;
        const double us = philox_uniform(p.seed, static_cast<uint32_t>(b), static_cast<uint32_t>(u),
                                         kPurposeSample, p.offset);
        const double target = us * Z;
        double run = 0.0, before_block = 0.0, blast_before = 0.0;
        int bstar = -1, blast = -1;
        for (int r = 0; r < CL; ++r) {
            const double w = cluster.map_shared_rank(&sh.xchg[xr], r)->x;
            if (w > 0.0) {
                if (run + w > target) {
                    bstar = r;
                    before_block = run;
                    break;
                }
                blast = r;
                blast_before = run;
            }
            run += w;
        }
        if (bstar < 0) {
            bstar = blast < 0 ? 0 : blast;
            before_block = blast_before;
        }
        const int D0 = sh.ts.depth[u];
        if (rank == bstar) {
            sh.tsum[tid] = mine;
            __syncthreads();
            if (warp == 0) {
                // lane l owns threads [8 l, 8 l + 8): block sums, one scan,
                // then the lane that holds the target walks its eight
                constexpr int kPer = kThreads / 32;
                const double tl = target - before_block;
                double bs = 0.0;
                int blast = -1;
                for (int i = 0; i < kPer; ++i) {
                    const double v = sh.tsum[lane * kPer + i];
                    bs += v;
                    if (v > 0.0) blast = lane * kPer + i;
                }
                const double incl = warp_incl_scan(bs);
                double excl = __shfl_up_sync(kFull, incl, 1);
                if (lane == 0) excl = 0.0;
                const unsigned hit = __ballot_sync(kFull, bs > 0.0 && incl > tl);
                int L = hit ? __ffs(hit) - 1 : -1;
                if (L < 0) {  // rounding: the last lane with positive weight
                    const unsigned pos = __ballot_sync(kFull, blast >= 0);
                    L = pos ? 31 - __clz(pos) : 0;
                }
                if (lane == L) {
                    double bt = 0.0;
                    const int t = icdf_seq(sh.tsum + L * kPer, kPer, tl - excl, bt);
                    sh.sel = t < 0 ? (blast >= 0 ? blast : 0) : L * kPer + t;
                    sh.before = excl + (t < 0 ? 0.0 : bt);
                    if (t < 0 && blast >= 0) {  // the prefix before the lane's last positive thread
                        double pre = excl;
                        for (int i = L * kPer; i < blast; ++i) pre += sh.tsum[i];
                        sh.before = pre;
                    }
                }
            }
            __syncthreads();
            if (tid == sh.sel) {
                const double tt = target - before_block - sh.before;
                constexpr int kEsz = sizeof(typename Tag::elem);
                double runl = 0.0;
                int tok = -1, lastp = ch.lo;
                for (int e0 = ch.lo; e0 < ch.hi && tok < 0; e0 += kVec) {
                    uint4 tv = ldg_vec(static_cast<const char *>(p.tl) + (off_u + e0) * kEsz);
                    uint4 dv = rej ? ldg_vec(static_cast<const char *>(p.dl) + (off_u + e0) * kEsz)
                                   : make_uint4(0, 0, 0, 0);
                    if (e0 + kVec > p.V) {
                        tv = mask_tail<Tag>(tv, p.V - e0);
                        dv = mask_tail<Tag>(dv, p.V - e0);
                    }
                    float xt[kVec], xd[kVec];
                    unpack<Tag>(tv, xt);
                    unpack<Tag>(dv, xd);
                    for (int e = 0; e < kVec && tok < 0; ++e) {
                        const double w = weight(xt[e], xd[e]);
                        if (w > 0.0) {
                            if (runl + w > tt) tok = e0 + e;
                            else lastp = e0 + e;
                        }
                        runl += w;
                    }
                }
                p.out[static_cast<int64_t>(b) * W + D0] = tok < 0 ? lastp : tok;
            }
        }
        if (rank == 0) {
            if (tid == 0) {
                int32_t *out = p.out + static_cast<int64_t>(b) * W;
                int32_t *path = p.path ? p.path + static_cast<int64_t>(b) * W : nullptr;
                for (int j = D0 + 1; j < W; ++j) out[j] = -1;
                if (path)
                    for (int j = 0; j < W; ++j) path[j] = -1;
                for (int node = u; node != 0; node = __ldg(pa + node)) {
                    out[sh.ts.depth[node] - 1] = __ldg(tk + node);
                    if (path) path[sh.ts.depth[node]] = node;
                }
                if (path) path[0] = 0;
                p.acc[b] = D0;
            }
        }
        __syncthreads();
    }
    cluster.sync();  // no block leaves while another may still read its exchange slots
}

}  // namespace sv
