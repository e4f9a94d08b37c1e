// specverify.cu -- kernels and C ABI of libspecverify.so (sm_100a).
//
// Call flow of spec_verify_linear (all on the caller's stream, no host sync):
//   memset(counters) -> k_pass1 (one streaming read of the 2k+1 rows of every
//   request; the last block of each request decides n) -> k_pass2a (fp64
//   normalisers of the residual row pair) -> k_pass2b (fp64 segment weights;
//   the last block of each request draws the token).
// spec_verify_tree: memset -> k_pass1 (tree decide) [-> k_pass2b if stochastic].
// spec_verify_greedy: k_greedy_cluster alone (no workspace).
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/specverify.h"
#include "sv_common.cuh"
#include "sv_decide.cuh"
#include "sv_greedy.cuh"
#include "sv_philox.cuh"
#include "sv_sample.cuh"
#include "sv_stats.cuh"

namespace sv {

template <class Tag, int MODE, int U>
__global__ void __launch_bounds__(kThreads) k_pass1(const Params p)
{
    __shared__ float redf[kWarps];
    __shared__ int redi[kWarps];
    const int64_t item = blockIdx.x;
    const int s = static_cast<int>(item % p.S);
    const int64_t br = item / p.S;
    const int r = static_cast<int>(br % p.R);
    const int b = static_cast<int>(br / p.R);
    constexpr int kEsz = sizeof(typename Tag::elem);

    const void *base;
    int64_t row_index;
    bool active = true;
    if (MODE == kLinear) {
        if (r <= p.k) {
            base = p.tl;
            row_index = static_cast<int64_t>(b) * (p.k + 1) + r;
        } else {
            base = p.dl;
            row_index = static_cast<int64_t>(b) * p.k + (r - p.k - 1);
        }
    } else if (r < p.N) {
        base = p.tl;
        row_index = static_cast<int64_t>(b) * p.N + r;
    } else {
        base = p.dl;
        row_index = static_cast<int64_t>(b) * p.N + (r - p.N);
        active = node_has_child(p, b, r - p.N);
    }
    if (active) {
        const char *row = static_cast<const char *>(base) + row_index * p.stride * kEsz;
        const int seg_begin = s * p.seg;
        const int seg_end = min(p.V, seg_begin + p.seg);
        uint4 raw[U];
        load_segment<Tag, U>(row, seg_begin, seg_end, raw);
        float2 part;
        if (MODE == kTreeGreedy) part = segment_argmax_partial<Tag, U>(raw, seg_begin, redf, redi);
        else part = segment_softmax_partial<Tag, U>(raw, p.c, redf);
        if (threadIdx.x == 0) p.rowpart[br * p.S + s] = part;
    }
    if (arrive_last(&p.cnt1[b], static_cast<unsigned>(p.R * p.S))) {
        if (MODE == kLinear) decide_linear<Tag>(p, b);
        else decide_tree<Tag, MODE>(p, b);
    }
}

__global__ void k_debug_uniforms(uint64_t seed, uint32_t offset, uint32_t purpose, int batch,
                                 int count, int first, double *out)
{
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<int64_t>(batch) * count) return;
    const int b = static_cast<int>(i / count), j = static_cast<int>(i % count);
    out[i] = philox_uniform(seed, static_cast<uint32_t>(b), static_cast<uint32_t>(first + j), purpose,
                            offset);
}

// ------------------------------------------------------------ host helpers
namespace {

constexpr size_t kAlign = 256;
constexpr int kMinSeg = kThreads * F32::kVec;  // smallest pass-1 segment (fp32, U = 1)

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Workspace layout; counters first.  Region sizes use the smallest pass-1
// segment, so any per-call segment choice fits.
struct Layout {
    size_t cnt, rowpart, rowstat, req, p2a, p2b, total;
    bool ok;
};

Layout layout(int B, int R, int V)
{
    Layout L{};
    L.ok = false;
    if (B < 0 || R < 1 || V < 1) return L;
    const int64_t smax = ceil_div(V, kMinSeg);
    const int64_t s2 = ceil_div(V, kSeg2);
    size_t off = 0;
    L.cnt = off;
    off = align_up(off + sizeof(unsigned) * 3 * static_cast<size_t>(B));
    L.rowpart = off;
    off = align_up(off + sizeof(float2) * static_cast<size_t>(B) * R * smax);
    L.rowstat = off;
    off = align_up(off + sizeof(RowStat) * static_cast<size_t>(B) * R);
    L.req = off;
    off = align_up(off + sizeof(ReqInfo) * static_cast<size_t>(B));
    L.p2a = off;
    off = align_up(off + sizeof(double2) * static_cast<size_t>(B) * s2);
    L.p2b = off;
    off = align_up(off + sizeof(double) * static_cast<size_t>(B) * s2);
    L.total = off < kAlign ? kAlign : off;
    L.ok = true;
    return L;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(spec_dtype_t d) { return d == SPEC_BF16 ? 2 : 4; }
int vec_of(spec_dtype_t d) { return d == SPEC_BF16 ? Bf16::kVec : F32::kVec; }

// Shape checks that hold for every batch size (an empty batch included).
int check_shape(spec_dtype_t dtype, int64_t stride, int V)
{
    if (dtype != SPEC_F32 && dtype != SPEC_BF16) return SPEC_EINVAL;
    if (V < 1 || stride < V) return SPEC_EINVAL;
    if ((stride * elem_size(dtype)) % 16 != 0) return SPEC_EALIGN;
    return SPEC_OK;
}

// Pointer checks, for a non-empty batch.
int check_rows(const void *tl, const void *dl, bool need_dl)
{
    if (!tl || (need_dl && !dl)) return SPEC_EINVAL;
    if (!aligned16(tl) || (need_dl && !aligned16(dl))) return SPEC_EALIGN;
    return SPEC_OK;
}

// Pass-1 vectors per thread: enough blocks to fill the GPU several times.
int choose_u(int B, int R, int V, int vec)
{
    for (int u : {4, 2}) {
        const int64_t S = ceil_div(V, static_cast<int64_t>(kThreads) * vec * u);
        if (static_cast<int64_t>(B) * R * S >= 2048) return u;
    }
    return 1;
}

void fill_workspace(Params &p, void *ws, const Layout &L)
{
    char *w = static_cast<char *>(ws);
    auto *cnt = reinterpret_cast<unsigned *>(w + L.cnt);
    p.cnt1 = cnt;
    p.cnt2a = cnt + p.B;
    p.cnt2b = cnt + 2 * static_cast<int64_t>(p.B);
    p.rowpart = reinterpret_cast<float2 *>(w + L.rowpart);
    p.rowstat = reinterpret_cast<RowStat *>(w + L.rowstat);
    p.req = reinterpret_cast<ReqInfo *>(w + L.req);
    p.p2a = reinterpret_cast<double2 *>(w + L.p2a);
    p.p2b = reinterpret_cast<double *>(w + L.p2b);
}

template <class Tag, int MODE>
cudaError_t launch_pass1(const Params &p, int U, cudaStream_t st)
{
    const unsigned grid = static_cast<unsigned>(static_cast<int64_t>(p.B) * p.R * p.S);
    switch (U) {
    case 4: k_pass1<Tag, MODE, 4><<<grid, kThreads, 0, st>>>(p); break;
    case 2: k_pass1<Tag, MODE, 2><<<grid, kThreads, 0, st>>>(p); break;
    default: k_pass1<Tag, MODE, 1><<<grid, kThreads, 0, st>>>(p); break;
    }
    return cudaGetLastError();
}

template <class Tag>
cudaError_t launch_pass2(const Params &p, bool with_2a, cudaStream_t st)
{
    const unsigned grid = static_cast<unsigned>(static_cast<int64_t>(p.B) * p.S2);
    if (with_2a) {
        k_pass2a<Tag><<<grid, kThreads, 0, st>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    k_pass2b<Tag><<<grid, kThreads, 0, st>>>(p);
    return cudaGetLastError();
}

// Largest number of co-resident greedy clusters, per device and dtype.
constexpr int kGreedyCluster = 8;
std::mutex g_mu;
int g_max_clusters[64][2];

template <class Tag>
int greedy_max_clusters(int dtype_index)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    std::lock_guard<std::mutex> lock(g_mu);
    int &slot = g_max_clusters[dev][dtype_index];
    if (slot > 0) return slot;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kGreedyCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(kGreedyCluster);
    cfg.blockDim = dim3(kThreads);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_greedy_cluster<Tag, kGreedyCluster>, &cfg) !=
            cudaSuccess ||
        n < 1)
        return -1;
    slot = n;
    return n;
}

template <class Tag>
int launch_greedy(Params &p, cudaStream_t st, int dtype_index)
{
    const int maxc = greedy_max_clusters<Tag>(dtype_index);
    if (maxc < 1) return SPEC_ECUDA;
    const int64_t rounds = ceil_div(p.B, maxc);
    const int ncl = static_cast<int>(ceil_div(p.B, rounds));
    const int slice = static_cast<int>(ceil_div(ceil_div(p.V, kGreedyCluster), Tag::kVec) * Tag::kVec);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kGreedyCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(ncl) * kGreedyCluster);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_greedy_cluster<Tag, kGreedyCluster>, p, slice) != cudaSuccess)
        return SPEC_ECUDA;
    return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}

void base_params(Params &p, const void *tl, const void *dl, int64_t stride, int B, int V,
                 float T, uint64_t seed, uint32_t offset)
{
    std::memset(&p, 0, sizeof p);
    p.tl = tl;
    p.dl = dl;
    p.stride = stride;
    p.B = B;
    p.V = V;
    const double t = static_cast<double>(T);
    p.inv_t = 1.0 / t;
    p.c = static_cast<float>(1.4426950408889634 / t);  // log2(e) / T
    p.seed = seed;
    p.offset = offset;
    p.S2 = static_cast<int>(ceil_div(V, kSeg2));
}

}  // namespace
}  // namespace sv

using namespace sv;

extern "C" size_t spec_verify_workspace_size(int batch, int rows_per_req, int vocab)
{
    const Layout L = layout(batch, rows_per_req, vocab);
    return L.ok ? L.total : 0;
}

extern "C" const char *spec_verify_strerror(int code)
{
    switch (code) {
    case SPEC_OK: return "ok";
    case SPEC_EINVAL: return "invalid argument (size, count, temperature or NULL pointer)";
    case SPEC_EALIGN: return "logit base pointer or row pitch not 16-byte aligned";
    case SPEC_EUNSUPPORTED: return "size beyond the supported limits";
    case SPEC_ECUDA: return "CUDA launch or query failed";
    case SPEC_EWORKSPACE: return "workspace NULL, not 256-byte aligned, or too small";
    default: return "unknown error code";
    }
}

extern "C" int spec_verify_linear(const void *target_logits, const void *draft_logits,
                                  spec_dtype_t dtype, int64_t row_stride,
                                  const int32_t *draft_tokens, int batch, int k, int vocab,
                                  float temperature, uint64_t seed, uint32_t offset,
                                  int32_t *out_tokens, int32_t *accepted_len, float *dbg_logp,
                                  float *dbg_logq, int32_t *status, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream)
{
    if (batch < 0 || k < 1) return SPEC_EINVAL;
    if (k > SPEC_MAX_K) return SPEC_EUNSUPPORTED;
    if (!(temperature > 0.f) || !(temperature < INFINITY)) return SPEC_EINVAL;
    int rc = check_shape(dtype, row_stride, vocab);
    if (rc != SPEC_OK) return rc;
    if (batch == 0) return SPEC_OK;
    rc = check_rows(target_logits, draft_logits, true);
    if (rc != SPEC_OK) return rc;
    if (!draft_tokens || !out_tokens || !accepted_len) return SPEC_EINVAL;
    const int R = 2 * k + 1;
    const Layout L = layout(batch, R, vocab);
    if (!L.ok) return SPEC_EINVAL;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
        workspace_bytes < L.total)
        return SPEC_EWORKSPACE;
    const int vec = vec_of(dtype);
    const int U = choose_u(batch, R, vocab, vec);
    const int seg = kThreads * vec * U;
    const int64_t S = ceil_div(vocab, seg);
    if (static_cast<int64_t>(batch) * R * S > INT_MAX ||
        static_cast<int64_t>(batch) * ceil_div(vocab, kSeg2) > INT_MAX)
        return SPEC_EUNSUPPORTED;

    Params p;
    base_params(p, target_logits, draft_logits, row_stride, batch, vocab, temperature, seed, offset);
    p.tokens = draft_tokens;
    p.k = k;
    p.R = R;
    p.S = static_cast<int>(S);
    p.seg = seg;
    p.out = out_tokens;
    p.acc = accepted_len;
    p.dbg_lp = dbg_logp;
    p.dbg_lq = dbg_logq;
    p.status = status;
    fill_workspace(p, workspace, L);

    if (cudaMemsetAsync(p.cnt1, 0, sizeof(unsigned) * 3 * static_cast<size_t>(batch), stream) !=
        cudaSuccess)
        return SPEC_ECUDA;
    cudaError_t e;
    if (dtype == SPEC_BF16) {
        e = launch_pass1<Bf16, kLinear>(p, U, stream);
        if (e == cudaSuccess) e = launch_pass2<Bf16>(p, true, stream);
    } else {
        e = launch_pass1<F32, kLinear>(p, U, stream);
        if (e == cudaSuccess) e = launch_pass2<F32>(p, true, stream);
    }
    return e == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}

extern "C" int spec_verify_greedy(const void *target_logits, spec_dtype_t dtype,
                                  int64_t row_stride, const int32_t *draft_tokens, int batch,
                                  int k, int vocab, int32_t *out_tokens, int32_t *accepted_len,
                                  int32_t *status, cudaStream_t stream)
{
    if (batch < 0 || k < 1) return SPEC_EINVAL;
    if (k > SPEC_MAX_K) return SPEC_EUNSUPPORTED;
    int rc = check_shape(dtype, row_stride, vocab);
    if (rc != SPEC_OK) return rc;
    if (batch == 0) return SPEC_OK;
    rc = check_rows(target_logits, nullptr, false);
    if (rc != SPEC_OK) return rc;
    if (!draft_tokens || !out_tokens || !accepted_len) return SPEC_EINVAL;
    Params p;
    base_params(p, target_logits, nullptr, row_stride, batch, vocab, 1.0f, 0, 0);
    p.tokens = draft_tokens;
    p.k = k;
    p.out = out_tokens;
    p.acc = accepted_len;
    p.status = status;
    return dtype == SPEC_BF16 ? launch_greedy<Bf16>(p, stream, 1) : launch_greedy<F32>(p, stream, 0);
}

extern "C" int spec_verify_tree(const void *target_logits, const void *draft_logits,
                                spec_dtype_t dtype, int64_t row_stride,
                                const int32_t *node_tokens, const int32_t *parents, int batch,
                                int num_nodes, int max_depth, int vocab, int stochastic,
                                float temperature, uint64_t seed, uint32_t offset,
                                int32_t *out_tokens, int32_t *accepted_len,
                                int32_t *out_path_nodes, int32_t *status, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream)
{
    if (batch < 0 || num_nodes < 1 || max_depth < 1) return SPEC_EINVAL;
    if (num_nodes > SPEC_MAX_NODES) return SPEC_EUNSUPPORTED;
    if (stochastic && (!(temperature > 0.f) || !(temperature < INFINITY))) return SPEC_EINVAL;
    int rc = check_shape(dtype, row_stride, vocab);
    if (rc != SPEC_OK) return rc;
    if (batch == 0) return SPEC_OK;
    rc = check_rows(target_logits, draft_logits, stochastic != 0);
    if (rc != SPEC_OK) return rc;
    if (!node_tokens || !parents || !out_tokens || !accepted_len) return SPEC_EINVAL;
    const int R = stochastic ? 2 * num_nodes : num_nodes;
    const Layout L = layout(batch, R, vocab);
    if (!L.ok) return SPEC_EINVAL;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
        workspace_bytes < L.total)
        return SPEC_EWORKSPACE;
    const int vec = vec_of(dtype);
    const int U = choose_u(batch, R, vocab, vec);
    const int seg = kThreads * vec * U;
    const int64_t S = ceil_div(vocab, seg);
    if (static_cast<int64_t>(batch) * R * S > INT_MAX ||
        static_cast<int64_t>(batch) * ceil_div(vocab, kSeg2) > INT_MAX ||
        static_cast<int64_t>(batch) * (max_depth + 1) > INT_MAX)
        return SPEC_EUNSUPPORTED;

    Params p;
    base_params(p, target_logits, draft_logits, row_stride, batch, vocab,
                stochastic ? temperature : 1.0f, seed, offset);
    p.tokens = node_tokens;
    p.parents = parents;
    p.N = num_nodes;
    p.max_depth = max_depth;
    p.R = R;
    p.S = static_cast<int>(S);
    p.seg = seg;
    p.out = out_tokens;
    p.acc = accepted_len;
    p.path = out_path_nodes;
    p.status = status;
    fill_workspace(p, workspace, L);

    if (cudaMemsetAsync(p.cnt1, 0, sizeof(unsigned) * 3 * static_cast<size_t>(batch), stream) !=
        cudaSuccess)
        return SPEC_ECUDA;
    cudaError_t e;
    if (dtype == SPEC_BF16) {
        e = stochastic ? launch_pass1<Bf16, kTreeStochastic>(p, U, stream)
                       : launch_pass1<Bf16, kTreeGreedy>(p, U, stream);
        if (e == cudaSuccess && stochastic) e = launch_pass2<Bf16>(p, false, stream);
    } else {
        e = stochastic ? launch_pass1<F32, kTreeStochastic>(p, U, stream)
                       : launch_pass1<F32, kTreeGreedy>(p, U, stream);
        if (e == cudaSuccess && stochastic) e = launch_pass2<F32>(p, false, stream);
    }
    return e == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}

extern "C" int spec_verify_debug_uniforms(uint64_t seed, uint32_t offset, uint32_t purpose,
                                          int batch, int count, int first_position, double *out,
                                          cudaStream_t stream)
{
    if (batch < 0 || count < 0 || !out) return SPEC_EINVAL;
    const int64_t n = static_cast<int64_t>(batch) * count;
    if (n == 0) return SPEC_OK;
    const int64_t blocks = ceil_div(n, 256);
    if (blocks > INT_MAX) return SPEC_EUNSUPPORTED;
    k_debug_uniforms<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(seed, offset, purpose, batch,
                                                                         count, first_position, out);
    return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}
