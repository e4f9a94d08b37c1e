// walk.cu -- C ABI of the walking greedy calls (sv_walk.cuh):
// spec_verify_greedy_walk and spec_verify_tree_greedy_walk, one launch of
// the cluster kernel k_greedy_walk each; no workspace.  Everything is
// enqueued on the caller's stream; no host synchronisation.  The argument
// rules are those of spec_verify_greedy and spec_verify_tree.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/specverify.h"
#include "sv_common.cuh"
#include "sv_walk.cuh"

namespace sv {
namespace {

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The logit layout rules shared with the other calls: a known dtype,
// 1 <= V <= row_stride, 16-byte row pitch.
int check_shape(spec_dtype_t dtype, int64_t stride, int V)
{
    if (dtype != SPEC_F32 && dtype != SPEC_BF16) return SPEC_EINVAL;
    if (V < 1 || stride < V) return SPEC_EINVAL;
    if ((stride * (dtype == SPEC_BF16 ? 2 : 4)) % 16 != 0) return SPEC_EALIGN;
    return SPEC_OK;
}

std::mutex g_walk_mu;

// Largest number of co-resident walking clusters, per device and dtype.
constexpr int kWalkCluster = 8;
int g_walk_clusters[64][2];

template <class Tag>
int walk_max_clusters(int dtype_index)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    std::lock_guard<std::mutex> lock(g_walk_mu);
    int &slot = g_walk_clusters[dev][dtype_index];
    if (slot > 0) return slot;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kWalkCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(kWalkCluster);
    cfg.blockDim = dim3(kThreads);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_greedy_walk<Tag, kWalkCluster>, &cfg) != cudaSuccess ||
        n < 1)
        return -1;
    slot = n;
    return n;
}

// One cluster per request up to the co-resident maximum; a cluster keeps up
// to A requests in flight, as many as its node cache holds.
template <class Tag>
int launch_walk(Params &p, bool chain, cudaStream_t st, int dtype_index)
{
    const int maxc = walk_max_clusters<Tag>(dtype_index);
    if (maxc < 1) return SPEC_ECUDA;
    const int ncl = std::min(maxc, p.B);
    const int A = std::min(kWalkSlots, kWalkCache / p.N);
    const int slice = static_cast<int>(ceil_div(ceil_div(p.V, kWalkCluster), Tag::kVec) * Tag::kVec);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kWalkCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(ncl) * kWalkCluster);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_greedy_walk<Tag, kWalkCluster>, p, slice, A, chain ? 1 : 0) !=
        cudaSuccess)
        return SPEC_ECUDA;
    return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}

void walk_params(Params &p, const void *tl, int64_t stride, int B, int V)
{
    std::memset(&p, 0, sizeof p);
    p.tl = tl;
    p.stride = stride;
    p.B = B;
    p.V = V;
}

}  // namespace
}  // namespace sv

using namespace sv;

extern "C" int spec_verify_greedy_walk(const void *target_logits, spec_dtype_t dtype,
                                       int64_t row_stride, const int32_t *draft_tokens, int batch,
                                       int k, int vocab, int32_t *out_tokens,
                                       int32_t *accepted_len, int32_t *status, cudaStream_t stream)
{
    if (batch < 0 || k < 1) return SPEC_EINVAL;
    if (k > SPEC_MAX_K) return SPEC_EUNSUPPORTED;
    int rc = check_shape(dtype, row_stride, vocab);
    if (rc != SPEC_OK) return rc;
    if (batch == 0) return SPEC_OK;
    if (!target_logits) return SPEC_EINVAL;
    if (!aligned16(target_logits)) return SPEC_EALIGN;
    if (!draft_tokens || !out_tokens || !accepted_len) return SPEC_EINVAL;
    Params p;
    walk_params(p, target_logits, row_stride, batch, vocab);
    p.tokens = draft_tokens;
    p.k = k;
    p.N = k + 1;  // the chain root, k drafts
    p.max_depth = k;
    p.out = out_tokens;
    p.acc = accepted_len;
    p.status = status;
    return dtype == SPEC_BF16 ? launch_walk<Bf16>(p, true, stream, 1)
                              : launch_walk<F32>(p, true, stream, 0);
}

extern "C" int spec_verify_tree_greedy_walk(const void *target_logits, spec_dtype_t dtype,
                                            int64_t row_stride, const int32_t *node_tokens,
                                            const int32_t *parents, int batch, int num_nodes,
                                            int max_depth, int vocab, int32_t *out_tokens,
                                            int32_t *accepted_len, int32_t *out_path_nodes,
                                            int32_t *status, cudaStream_t stream)
{
    if (batch < 0 || num_nodes < 1 || max_depth < 1) return SPEC_EINVAL;
    if (num_nodes > SPEC_MAX_NODES) return SPEC_EUNSUPPORTED;
    int rc = check_shape(dtype, row_stride, vocab);
    if (rc != SPEC_OK) return rc;
    if (batch == 0) return SPEC_OK;
    if (!target_logits) return SPEC_EINVAL;
    if (!aligned16(target_logits)) return SPEC_EALIGN;
    if (!node_tokens || !parents || !out_tokens || !accepted_len) return SPEC_EINVAL;
    if (static_cast<int64_t>(batch) * (max_depth + 1) > INT_MAX) return SPEC_EUNSUPPORTED;
    Params p;
    walk_params(p, target_logits, row_stride, batch, vocab);
    p.tokens = node_tokens;
    p.parents = parents;
    p.N = num_nodes;
    p.max_depth = max_depth;
    p.out = out_tokens;
    p.acc = accepted_len;
    p.path = out_path_nodes;
    p.status = status;
    return dtype == SPEC_BF16 ? launch_walk<Bf16>(p, false, stream, 1)
                              : launch_walk<F32>(p, false, stream, 0);
}
