// sv_greedy.cuh -- greedy (argmax-match) verification.
//
// "Accelerating Sonar through speculation", section "Target-Draft": the
// draft emits its top token at each step, so a draft is kept exactly when it
// equals the target's top token; at the first mismatch (or after all k) the
// target's top token is emitted.
//
// Two forms with identical outputs:
//
//  * With a workspace: pass 1 streams every target row as the greedy tree
//    mode does (k_pass1: (max, lowest argmax, NaN seen) per 2048-entry item,
//    stored as partials), then k_greedy_decide merges each row's partials
//    and scans for the first mismatch, a block per request.
//
//  * Without a workspace (k_greedy_cluster): one thread-block cluster owns a
//    request at a time; each of its CL blocks reduces one contiguous slice of
//    each of the k+1 rows in its shared memory, a block's reads running one
//    step ahead of its reductions.  The cluster merge is pipelined by one
//    request: at the end of request r a block publishes its partials (double
//    buffered by request parity) and arrives on the split cluster barrier; at
//    the end of request r+1 it waits for that phase, and the rank-0 block
//    merges request r's partials of all CL blocks through distributed shared
//    memory and writes the outputs.  No block waits for the request it has
//    just finished.
#pragma once

#include <cooperative_groups.h>

#include "sv_common.cuh"


namespace sv {

constexpr int kMaxRowsGreedy = 33;  // k + 1 with k <= 32

// Split cluster barrier (all threads of every block of the cluster, in
// step): arrive with release semantics, wait with acquire semantics; a
// thread waits for a phase before it arrives for the next one.
__device__ __forceinline__ void cluster_arrive()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait()
{
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

template <class Tag, int CL>
__global__ void __launch_bounds__(kThreads) k_greedy_cluster(const Params p, int slice)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    constexpr int kVec = Tag::kVec;
    constexpr int kEsz = sizeof(typename Tag::elem);
    constexpr int U = 4;
    constexpr int kChunk = kThreads * kVec * U;  // entries of a slice read per step

    __shared__ float2 part[2][kMaxRowsGreedy];
    __shared__ float2 wpart[2][kMaxRowsGreedy][kWarps];
    __shared__ int g_sh[kMaxRowsGreedy];
    __shared__ int nan_sh;

    const int rank = static_cast<int>(cluster.block_rank());
    const int cid = blockIdx.x / CL, ncl = gridDim.x / CL;
    const int k = p.k, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int s_begin = min(p.V, rank * slice), s_end = min(p.V, s_begin + slice);
    // steps per row (an empty slice still takes one, so every row is reduced)
    const int iters = max(1, (s_end - s_begin + kChunk - 1) / kChunk);

    // The block's steps form one sequence over (request, row, step); the
    // loads of the next step are issued before the current one is reduced,
    // so they overlap the reduction and the block and cluster barriers.
    auto load = [&](int b, int j, int it, uint4 (&raw)[U]) {
        const char *row = static_cast<const char *>(p.tl) +
                          (static_cast<int64_t>(b) * (k + 1) + j) * p.stride * kEsz;
        const int base = s_begin + it * kChunk;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e0 = base + (tid + u * kThreads) * kVec;
            raw[u] = e0 < s_end ? ldg_vec(row + static_cast<int64_t>(e0) * kEsz)
                                : make_uint4(Tag::kNegInfWord, Tag::kNegInfWord, Tag::kNegInfWord,
                                             Tag::kNegInfWord);
        }
    };
    int b = cid, j = 0, it = 0;
    uint4 cur[U], nxt[U];
    if (b < p.B) load(b, j, it, cur);
    float best = -INFINITY;
    int idx = INT_MAX;
    bool nan = false;
    int rq = 0, prev_b = -1;  // requests done by this cluster; the last one
    // rank 0: merge request bb's partials (buffer buf) of all blocks and
    // write its outputs (every thread of the block calls it)
    auto merge_write = [&](int bb, int buf) {
        if (tid == 0) nan_sh = 0;
        __syncthreads();
        for (int jj = tid; jj <= k; jj += kThreads) {
            float bv = -INFINITY;
            int bi = INT_MAX;
            bool nn = false;
            for (int r = 0; r < CL; ++r) {  // slices in index order
                const float2 *rp = cluster.map_shared_rank(&part[buf][0], r);
                const float2 v = rp[jj];
                if (v.x != v.x) nn = true;
                else argmax_take(bv, bi, v.x, __float_as_int(v.y));
            }
            if (nn) atomicOr(&nan_sh, 1);
            g_sh[jj] = (bi == INT_MAX) ? 0 : bi;
        }
        __syncthreads();
        if (warp == 0) {
            int x = -1;
            bool tok_ok = true;
            if (lane < k) {
                x = __ldg(p.tokens + static_cast<int64_t>(bb) * k + lane);
                tok_ok = (x >= 0 && x < p.V);
            }
            const int bits = (__any_sync(kFull, !tok_ok) ? kStToken : 0) | (nan_sh ? kStLogit : 0);
            const unsigned mism = __ballot_sync(kFull, lane < k && x != g_sh[lane < k ? lane : 0]);
            const int n = mism ? __ffs(mism) - 1 : k;
            int32_t *out = p.out + static_cast<int64_t>(bb) * (k + 1);
            for (int jj = lane; jj <= k; jj += 32) {
                int v = -1;
                if (!bits) v = (jj < n) ? x : (jj == n ? g_sh[n] : -1);  // jj < n implies jj == lane
                out[jj] = v;
            }
            if (lane == 0) {
                p.acc[bb] = bits ? -1 : n;
                report(p.status, bits);
            }
        }
    };
#pragma unroll 1
    while (b < p.B) {
        // the step after this one
        int nb = b, nj = j, nit = it + 1;
        if (nit == iters) {
            nit = 0;
            if (++nj > k) {
                nj = 0;
                nb += ncl;
            }
        }
        if (nb < p.B) load(nb, nj, nit, nxt);
        const int base = s_begin + it * kChunk;
        // a thread visits its entries in increasing index order, so a later
        // entry equal to the running max never replaces it (ties go to the
        // lowest index); a vector's packed max decides whether any entry of
        // it can matter, and only then are its entries searched
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e0 = base + (tid + u * kThreads) * kVec;
            uint4 raw = cur[u];
            if (e0 < s_end && e0 + kVec > s_end) raw = mask_tail<Tag>(raw, s_end - e0);
            const float vm = vec_max<Tag>(raw);  // NaN if any entry is NaN
            if (!(vm <= best)) {
                if (vm != vm) {
                    nan = true;
                } else {
                    float x[kVec];
                    unpack<Tag>(raw, x);
                    int first = kVec - 1;
#pragma unroll
                    for (int e = kVec - 1; e >= 0; --e)
                        if (x[e] == vm) first = e;
                    best = vm;
                    idx = e0 + first;
                }
            }
        }
        if (it == iters - 1) {  // row j of request b is reduced in this block
            const int buf = rq & 1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(kFull, best, o);
                const int oi = __shfl_xor_sync(kFull, idx, o);
                argmax_take(best, idx, ov, oi);
            }
            nan = __any_sync(kFull, nan);
            if (lane == 0) wpart[buf][j][warp] = make_float2(nan ? __int_as_float(0x7FC00000) : best, __int_as_float(idx));
            best = -INFINITY;
            idx = INT_MAX;
            nan = false;
            if (j == k) {  // the request is reduced in every warp of the block
                __syncthreads();
                // phase rq-1 (the previous request) is complete in every
                // block: rank 0 merges it now
                if (rq > 0) {
                    cluster_wait();
                    if (rank == 0) merge_write(prev_b, buf ^ 1);
                }
                for (int jj = tid; jj <= k; jj += kThreads) {
                    float bv = -INFINITY;
                    int bi = INT_MAX;
                    bool nn = false;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) {
                        const float2 v = wpart[buf][jj][w];
                        if (v.x != v.x) nn = true;
                        else argmax_take(bv, bi, v.x, __float_as_int(v.y));
                    }
                    part[buf][jj] = make_float2(nn ? __int_as_float(0x7FC00000) : bv, __int_as_float(bi));
                }
                cluster_arrive();  // phase rq: this block's partials of request b are in place
                prev_b = b;
                ++rq;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) cur[u] = nxt[u];
        b = nb;
        j = nj;
        it = nit;
    }
    // the last request: wait for its phase and merge it; then one full
    // barrier so that no block leaves while rank 0 may still read its
    // partials
    if (rq > 0) {
        cluster_wait();
        if (rank == 0) merge_write(prev_b, (rq - 1) & 1);
    }
    cluster.sync();
}

// The decide step of the workspace form: a block per request (blocks stride
// over the batch), a warp per row (rows w, w + kWarps, ...).  A row's S
// pass-1 partials are merged lane-strided and then across the warp;
// argmax_take breaks ties by the lower index, so the result is the lowest
// argmax whatever the merge order.  Warp 0 then scans for the first
// mismatch.  The draft tokens are inputs and are read before pass 1 ends.
template <class Tag>
__global__ void __launch_bounds__(kThreads) k_greedy_decide(const __grid_constant__ Params p)
{
    __shared__ int g_sh[kMaxRowsGreedy];
    __shared__ int bits_sh;
    const int k = p.k, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int b = blockIdx.x;
    auto token = [&](int bb) {
        return (bb < p.B && lane < k) ? __ldg(p.tokens + static_cast<int64_t>(bb) * k + lane) : -1;
    };
    int x = warp == 0 ? token(b) : -1;
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    for (; b < p.B; b += gridDim.x) {
        if (tid == 0) bits_sh = 0;
        __syncthreads();
        for (int r = warp; r <= k; r += kWarps) {
            const float2 *pp = p.rowpart + (static_cast<int64_t>(b) * (k + 1) + r) * p.S;
            float bv = -INFINITY;
            int bi = INT_MAX;
            bool nan = false;
            for (int s = lane; s < p.S; s += 32) {
                const float2 v = __ldcg(pp + s);
                if (v.x != v.x) nan = true;
                else argmax_take(bv, bi, v.x, __float_as_int(v.y));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(kFull, bv, o);
                const int oi = __shfl_xor_sync(kFull, bi, o);
                argmax_take(bv, bi, ov, oi);
            }
            if (__any_sync(kFull, nan) && lane == 0) atomicOr(&bits_sh, kStLogit);
            if (lane == 0) g_sh[r] = (bi == INT_MAX) ? 0 : bi;
        }
        __syncthreads();
        if (warp == 0) {
            const bool tok_ok = lane >= k || (x >= 0 && x < p.V);
            const int bits = (__any_sync(kFull, !tok_ok) ? kStToken : 0) | bits_sh;
            const unsigned mism = __ballot_sync(kFull, lane < k && x != g_sh[lane < k ? lane : 0]);
            const int n = mism ? __ffs(mism) - 1 : k;
            int32_t *out = p.out + static_cast<int64_t>(b) * (k + 1);
            for (int jj = lane; jj <= k; jj += 32) {
                int v = -1;
                if (!bits) v = (jj < n) ? x : (jj == n ? g_sh[n] : -1);  // jj < n implies jj == lane
                out[jj] = v;
            }
            if (lane == 0) {
                p.acc[b] = bits ? -1 : n;
                report(p.status, bits);
            }
            x = token(b + gridDim.x);
        }
    }
}

}  // namespace sv
