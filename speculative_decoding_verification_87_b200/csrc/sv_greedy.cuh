// sv_greedy.cuh -- greedy (argmax-match) verification without workspace.
//
// "Accelerating Sonar through speculation", section "Target-Draft": the
// draft emits its top token at each step, so a draft is kept exactly when it
// equals the target's top token; at the first mismatch (or after all k) the
// target's top token is emitted.
//
// One thread-block cluster owns a request at a time: each of its CL blocks
// reduces one contiguous slice of each of the k+1 target rows to (max,
// lowest argmax, NaN seen) in its shared memory; after a cluster barrier the
// rank-0 block merges the CL partials through distributed shared memory,
// scans for the first mismatch and writes the outputs.  Partials are double
// buffered, so one barrier per request suffices.  Clusters stride over the
// batch.
#pragma once

#include <cooperative_groups.h>

#include "sv_common.cuh"


namespace sv {

constexpr int kMaxRowsGreedy = 33;  // k + 1 with k <= 32

template <class Tag, int CL>
__global__ void __launch_bounds__(kThreads) k_greedy_cluster(const Params p, int slice)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    constexpr int U = 4;

    __shared__ float2 part[2][kMaxRowsGreedy];
    __shared__ float redf[kWarps];
    __shared__ int redi[kWarps];
    __shared__ int g_sh[kMaxRowsGreedy];
    __shared__ int nan_sh;

    const int rank = static_cast<int>(cluster.block_rank());
    const int cid = blockIdx.x / CL, ncl = gridDim.x / CL;
    const int k = p.k, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int s_begin = min(p.V, rank * slice), s_end = min(p.V, s_begin + slice);

    int it = 0;
    for (int b = cid; b < p.B; b += ncl, ++it) {
        const int buf = it & 1;
        for (int j = 0; j <= k; ++j) {
            const char *row = static_cast<const char *>(p.tl) +
                              (static_cast<int64_t>(b) * (k + 1) + j) * p.stride * kEsz;
            float best = -INFINITY;
            int idx = INT_MAX;
            bool nan = false;
            for (int base = s_begin; base < s_end; base += kThreads * kVec * U) {
                uint4 raw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int e0 = base + (tid + u * kThreads) * kVec;
                    raw[u] = e0 < s_end ? ldg_vec(row + static_cast<int64_t>(e0) * kEsz)
                                        : make_uint4(Tag::kNegInfWord, Tag::kNegInfWord,
                                                     Tag::kNegInfWord, Tag::kNegInfWord);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int e0 = base + (tid + u * kThreads) * kVec;
                    if (e0 < s_end && e0 + kVec > s_end) raw[u] = mask_tail<Tag>(raw[u], s_end - e0);
                    float x[kVec];
                    unpack<Tag>(raw[u], x);
#pragma unroll
                    for (int e = 0; e < kVec; ++e) {
                        nan |= (x[e] != x[e]);
                        if (x[e] > best) {
                            best = x[e];
                            idx = e0 + e;
                        }
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(kFull, best, o);
                const int oi = __shfl_xor_sync(kFull, idx, o);
                argmax_take(best, idx, ov, oi);
            }
            const int any_nan = __syncthreads_or(nan ? 1 : 0);
            if (lane == 0) {
                redf[warp] = best;
                redi[warp] = idx;
            }
            __syncthreads();
            if (tid == 0) {
                float bv = redf[0];
                int bi = redi[0];
                for (int w = 1; w < kWarps; ++w) argmax_take(bv, bi, redf[w], redi[w]);
                part[buf][j] = make_float2(any_nan ? __int_as_float(0x7FC00000) : bv,
                                           __int_as_float(bi));
            }
            __syncthreads();
        }
        cluster.sync();
        if (rank == 0) {
            if (tid == 0) nan_sh = 0;
            __syncthreads();
            for (int j = tid; j <= k; j += kThreads) {
                float bv = -INFINITY;
                int bi = INT_MAX;
                bool nan = false;
                for (int r = 0; r < CL; ++r) {  // slices in index order
                    const float2 *rp = cluster.map_shared_rank(&part[buf][0], r);
                    const float2 v = rp[j];
                    if (v.x != v.x) nan = true;
                    else argmax_take(bv, bi, v.x, __float_as_int(v.y));
                }
                if (nan) atomicOr(&nan_sh, 1);
                g_sh[j] = (bi == INT_MAX) ? 0 : bi;
            }
            __syncthreads();
            if (warp == 0) {
                int x = -1;
                bool tok_ok = true;
                if (lane < k) {
                    x = __ldg(p.tokens + static_cast<int64_t>(b) * k + lane);
                    tok_ok = (x >= 0 && x < p.V);
                }
                const int bits = (__any_sync(kFull, !tok_ok) ? kStToken : 0) |
                                 (nan_sh ? kStLogit : 0);
                const unsigned mism = __ballot_sync(kFull, lane < k && x != g_sh[lane < k ? lane : 0]);
                const int n = mism ? __ffs(mism) - 1 : k;
                int32_t *out = p.out + static_cast<int64_t>(b) * (k + 1);
                for (int j = lane; j <= k; j += 32) {
                    int v = -1;
                    if (!bits) v = (j < n) ? x : (j == n ? g_sh[n] : -1);  // j < n implies j == lane
                    out[j] = v;
                }
                if (lane == 0) {
                    p.acc[b] = bits ? -1 : n;
                    report(p.status, bits);
                }
            }
        }
    }
    cluster.sync();  // no block leaves while rank 0 may still read its partials
}

}  // namespace sv
