// specverify.cu -- C ABI of libspecverify.so (sm_100a) and its launches.
//
// spec_verify_linear: one memset of the call's counters and pass-1
// partials, then a cooperative launch of the persistent kernel k_fused
// (sv_fused.cuh); batches of one or two requests take the four-kernel path
// of the tree calls instead (pass 1, decide, pass 2, finalize).
// spec_verify_tree: the pass-1 kernel, the decide kernel and, where a token
// is drawn, the pass-2 and finalize kernels (sv_verify.cuh), each a
// programmatic dependent of the one before.
// spec_verify_greedy: with a workspace, k_pass1 (greedy tree mode over the
// target rows) and k_greedy_decide; without one, one launch of the cluster
// kernel k_greedy_cluster (sv_greedy.cuh).
// Everything is enqueued on the caller's stream; no host synchronisation.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/specverify.h"
#include "sv_common.cuh"
#include "sv_verify.cuh"
#include "sv_fused.cuh"
#include "sv_exp64.cuh"
#include "sv_greedy.cuh"
#include "sv_exact.cuh"
#include "sv_philox.cuh"

namespace sv {

__global__ void k_debug_uniforms(uint64_t seed, uint32_t offset, uint32_t purpose, int batch,
                                 int count, int first, double *out)
{
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<int64_t>(batch) * count) return;
    const int b = static_cast<int>(i / count), j = static_cast<int>(i % count);
    out[i] = philox_uniform(seed, static_cast<uint32_t>(b), static_cast<uint32_t>(first + j), purpose,
                            offset);
}

__global__ void k_debug_exp2(const double *z, double *out, int n, int kind, Params p)
{
    __shared__ double tab[kExp2Tab];
    for (int j = threadIdx.x; j < kExp2Tab; j += blockDim.x) tab[j] = p.exp2tab[j];
    __syncthreads();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const double zi = z[i];
    if (kind == 1) out[i] = f32_to_f64(ex2_fma(static_cast<float>(zi)));
    else if (kind == 2) out[i] = f32_to_f64(ex2_approx(static_cast<float>(zi)));
    else out[i] = exp2_fp64(zi, tab);
}

// ------------------------------------------------------------ host helpers
namespace {

constexpr size_t kAlign = 256;
constexpr int kItemMin = Pass1Shape<F32>::kItem;  // the shorter pass-1 item (fp32)

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Workspace layout.  Every region a call reads is written earlier in the
// same call; the one-kernel path first clears its counters and sets the
// pass-1 partials to all ones.  Region sizes use the shorter pass-1 item,
// so both dtypes fit.
struct Layout {
    size_t counters, rowpart, req, p2part, p2amb, ambbits, p2w, p2lane, total;
    bool ok;
};

Layout layout(int B, int R, int V)
{
    Layout L{};
    L.ok = false;
    if (B < 0 || R < 1 || V < 1) return L;
    const int64_t smax = ceil_div(V, kItemMin);
    const int64_t s2 = ceil_div(V, kSeg2);
    const int64_t w32 = s2 * (kSeg2 / 32);  // whole segments (16-byte aligned rows of the bitmap)
    size_t off = 0;
    L.counters = off;  // p2cnt[B], decided[B], p2claim, a_claim; rowpart follows directly
    off = align_up(off + sizeof(unsigned) * (2 * static_cast<size_t>(B) + 2));
    L.rowpart = off;
    off = align_up(off + sizeof(float2) * static_cast<size_t>(B) * R * smax);
    L.req = off;
    off = align_up(off + sizeof(ReqInfo) * static_cast<size_t>(B));
    L.p2part = off;
    off = align_up(off + sizeof(double4) * static_cast<size_t>(B) * s2);
    L.p2amb = off;
    off = align_up(off + sizeof(int) * static_cast<size_t>(B) * s2);
    L.ambbits = off;
    off = align_up(off + sizeof(unsigned) * static_cast<size_t>(B) * w32);
    L.p2w = off;
    off = align_up(off + 2 * sizeof(double) * static_cast<size_t>(B) * s2);
    L.p2lane = off;
    off = align_up(off + sizeof(double2) * 32 * static_cast<size_t>(B) * s2);
    L.total = off < kAlign ? kAlign : off;
    L.ok = true;
    return L;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(spec_dtype_t d) { return d == SPEC_BF16 ? 2 : 4; }

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

void fill_workspace(Params &p, void *ws, const Layout &L)
{
    char *w = static_cast<char *>(ws);
    auto *cnt = reinterpret_cast<unsigned *>(w + L.counters);
    p.p2cnt = cnt;
    p.decided = cnt + p.B;
    p.p2claim = p.decided + p.B;
    p.a_claim = p.p2claim + 1;
    p.rowpart = reinterpret_cast<float2 *>(w + L.rowpart);
    p.req = reinterpret_cast<ReqInfo *>(w + L.req);
    p.p2part = reinterpret_cast<double4 *>(w + L.p2part);
    p.p2amb = reinterpret_cast<int *>(w + L.p2amb);
    p.ambbits = reinterpret_cast<unsigned *>(w + L.ambbits);
    p.p2w = reinterpret_cast<double *>(w + L.p2w);
    p.p2lane = reinterpret_cast<double2 *>(w + L.p2lane);
}

// 2^(j/256), j = 0..255, from the host math library.
void fill_exp2_table(Params &p)
{
    for (int j = 0; j < kExp2Tab; ++j) p.exp2tab[j] = std::exp2(static_cast<double>(j) / kExp2Tab);
}


// Occupancy per device, dtype and mode, of the pass kernels.
std::mutex g_mu;
int g_pass1_blocks[64][2][3];
int g_pass2_blocks[64][2][3];
bool g_final_attr[64][2][3];
bool g_decide_attr[64][2][3];
int g_sm_count[64];

// Decide dynamic shared memory: the merged statistics of a request's rows.
size_t decide_smem(int R, int S)
{
    size_t n = (sizeof(double) + sizeof(float) + sizeof(int)) * static_cast<size_t>(R);
    n = (n + 15) / 16 * 16;
    if (static_cast<int64_t>(R) * S <= kDecideStageMax) n += sizeof(float2) * static_cast<size_t>(R) * S;
    return n;
}

// Finalize dynamic shared memory: the segment weights of each warp, for
// vocabularies up to kMaxS2Shared segments (else the workspace holds them).
size_t finalize_smem(int S2)
{
    return S2 <= kMaxS2Shared ? 2 * sizeof(double) * kWarps * static_cast<size_t>(S2) : 0;
}

template <class Tag, int MODE>
constexpr int pass1_min_blocks()
{
    return 2;
}

template <class Kernel>
int blocks_per_sm(int &slot, Kernel kernel, size_t dyn_smem)
{
    if (slot > 0) return slot;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(dyn_smem)) != cudaSuccess)
        return -1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, dyn_smem) != cudaSuccess || n < 1)
        return -1;
    slot = n;
    return n;
}

int sm_count(int dev)
{
    int &slot = g_sm_count[dev];
    if (slot > 0) return slot;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        return -1;
    slot = n;
    return n;
}

// A launch that may begin while the previous kernel on the stream drains
// (the kernel itself waits for it with griddepcontrol.wait).
template <class Kernel>
int launch_dependent(Kernel kernel, int64_t blocks, size_t dyn, cudaStream_t st, const Params &p,
                     int threads = kThreads, int cluster = 1)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cluster > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, kernel, p) == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}

// Blocks per request of the tree decide step (a cluster): enough that the
// batch's clusters cover about two waves of SMs, at most kDecideClusterMax.
constexpr int kDecideClusterMax = 4;
int decide_cluster(int B, int R, int sms)
{
    int g = std::max(1, std::min(kDecideClusterMax, (2 * sms) / std::max(1, B)));
    return std::min(g, R);
}

// Pass 1's static share (whole rounds of the grid's warps for about 88% of
// the items; the rest is claimed in chunks) and its claim counter, set to
// all ones on the stream before the launch.
int prep_pass1(Params &p, int64_t blocks, cudaStream_t st)
{
    const uint64_t W = static_cast<uint64_t>(blocks) * kWarps;
    p.nAs = static_cast<unsigned>((static_cast<uint64_t>(p.nA) * 88 / 100) / W * W);
    return cudaMemsetAsync(p.a_claim, 0xFF, sizeof(unsigned), st) == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}

// Launch pass 1, then the decide step and, where a token is drawn, pass 2
// and the finalize step, each a programmatic dependent of the one before.
// Pass grids are at most one resident wave.
template <class Tag, int MODE>
int launch_verify(Params &p, const Layout &L, void *ws, int dtype_index, cudaStream_t st)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SPEC_ECUDA;
    constexpr int kMin1 = pass1_min_blocks<Tag, MODE>();
    int per_sm1, per_sm2 = 1, sms;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        per_sm1 = blocks_per_sm(g_pass1_blocks[dev][dtype_index][MODE], k_pass1<Tag, MODE, kMin1>, kRingBytes);
        bool &dattr = g_decide_attr[dev][dtype_index][MODE];
        if (!dattr) {
            // the largest decide footprint: 2 * kMaxNodes rows' statistics plus staged partials
            if (cudaFuncSetAttribute(k_decide<Tag, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(decide_smem(2 * kMaxNodes, 0) +
                                                      sizeof(float2) * kDecideStageMax)) != cudaSuccess)
                return SPEC_ECUDA;
            dattr = true;
        }
        if (p.nP > 0) {
            per_sm2 = blocks_per_sm(g_pass2_blocks[dev][dtype_index][MODE], k_pass2<Tag, MODE>,
                                    StageShape<Tag>::kBytes);
            bool &attr = g_final_attr[dev][dtype_index][MODE];
            if (!attr) {
                if (cudaFuncSetAttribute(k_finalize<Tag, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(finalize_smem(kMaxS2Shared))) != cudaSuccess)
                    return SPEC_ECUDA;
                attr = true;
            }
        }
        sms = sm_count(dev);
    }
    if (per_sm1 < 1 || per_sm2 < 1 || sms < 1) return SPEC_ECUDA;
    const int64_t blocks1 =
        std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(per_sm1) * sms, ceil_div(p.nA, kWarps)));
    if (prep_pass1(p, blocks1, st) != SPEC_OK) return SPEC_ECUDA;
    k_pass1<Tag, MODE, kMin1><<<static_cast<unsigned>(blocks1), kThreads, kRingBytes, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SPEC_ECUDA;
    const int G = MODE == kLinear ? 1 : decide_cluster(p.B, p.R, sms);
    const int64_t blocksd =
        G > 1 ? static_cast<int64_t>(p.B) * G
              : std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(2) * sms, p.B));
    if (launch_dependent(k_decide<Tag, MODE>, blocksd, decide_smem(p.R, p.S), st, p, kDecideThreads, G) !=
        SPEC_OK)
        return SPEC_ECUDA;
    if (p.nP == 0) return SPEC_OK;

    const int64_t blocks2 =
        std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(per_sm2) * sms, ceil_div(p.nP, kWarps)));
    if (launch_dependent(k_pass2<Tag, MODE>, blocks2, StageShape<Tag>::kBytes, st, p) != SPEC_OK)
        return SPEC_ECUDA;
    // finalize: a latency chain per request, so one warp per block (one per
    // SM while the batch fits the SMs), up to 8 warps per block beyond
    const int fw = static_cast<int>(std::min<int64_t>(kWarps, std::max<int64_t>(1, ceil_div(p.B, sms))));
    const int64_t blocks3 = std::max<int64_t>(1, ceil_div(p.B, fw));
    return launch_dependent(k_finalize<Tag, MODE>, std::min<int64_t>(blocks3, static_cast<int64_t>(sms) * 8),
                            static_cast<size_t>(fw) * 2 * sizeof(double) * (p.S2 <= kMaxS2Shared ? p.S2 : 0), st, p,
                            32 * fw);
}

// The one-kernel linear path: clear the counters and partials, then one
// cooperative launch, exactly one resident wave (a grid that cannot be
// resident at once fails to launch: SPEC_ECUDA).
int g_fused_blocks[64][2];
template <class Tag>
int launch_fused(Params &p, const Layout &L, void *ws, int dtype_index, cudaStream_t st)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SPEC_ECUDA;
    int per_sm, sms;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        per_sm = blocks_per_sm(g_fused_blocks[dev][dtype_index], k_fused<Tag>, kFusedSmem);
        sms = sm_count(dev);
    }
    if (per_sm < 1 || sms < 1) return SPEC_ECUDA;
    // whole static rounds for about the first 88% of the pass-1 items
    const unsigned W = static_cast<unsigned>(per_sm * sms * kStreamers);
    p.nAs = static_cast<unsigned>((static_cast<uint64_t>(p.nA) * 88 / 100) / W * W);
    // counters and pass-1 partials to all ones (kPartEmpty), one contiguous range
    const size_t clear = L.rowpart - L.counters + sizeof(float2) * static_cast<size_t>(p.nA);
    if (cudaMemsetAsync(static_cast<char *>(ws) + L.counters, 0xFF, clear, st) != cudaSuccess)
        return SPEC_ECUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(per_sm * sms));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kFusedSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_fused<Tag>, p) != cudaSuccess) {
        (void)cudaGetLastError();  // the error is returned, not left for the next call
        return SPEC_ECUDA;
    }
    return SPEC_OK;
}

// The distribution-exact tree mode: pass 1 as the independent-test mode,
// then the cluster kernel k_tree_exact (one cluster per request, up to the
// co-resident maximum), a programmatic dependent of pass 1.
int g_exact_clusters[64][2];
template <class Tag>
int launch_exact(Params &p, int dtype_index, cudaStream_t st)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SPEC_ECUDA;
    int per_sm1, sms, maxc;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        per_sm1 = blocks_per_sm(g_pass1_blocks[dev][dtype_index][kTreeStochastic],
                                k_pass1<Tag, kTreeStochastic, 2>, kRingBytes);
        sms = sm_count(dev);
        int &slot = g_exact_clusters[dev][dtype_index];
        if (slot < 1) {
            cudaLaunchConfig_t q = {};
            cudaLaunchAttribute qa[1];
            qa[0].id = cudaLaunchAttributeClusterDimension;
            qa[0].val.clusterDim.x = kExactCluster;
            qa[0].val.clusterDim.y = 1;
            qa[0].val.clusterDim.z = 1;
            q.gridDim = dim3(kExactCluster);
            q.blockDim = dim3(kThreads);
            q.attrs = qa;
            q.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, k_tree_exact<Tag, kExactCluster>, &q) != cudaSuccess || n < 1)
                return SPEC_ECUDA;
            slot = n;
        }
        maxc = slot;
    }
    if (per_sm1 < 1 || sms < 1 || maxc < 1) return SPEC_ECUDA;
    const int64_t blocks1 =
        std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(per_sm1) * sms, ceil_div(p.nA, kWarps)));
    if (prep_pass1(p, blocks1, st) != SPEC_OK) return SPEC_ECUDA;
    k_pass1<Tag, kTreeStochastic, 2><<<static_cast<unsigned>(blocks1), kThreads, kRingBytes, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SPEC_ECUDA;
    const int ncl = std::min(maxc, p.B);
    const int slice = static_cast<int>(ceil_div(ceil_div(p.V, kExactCluster), Tag::kVec) * Tag::kVec);
    const int chunk = static_cast<int>(ceil_div(ceil_div(slice, kThreads), Tag::kVec) * Tag::kVec);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kExactCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(ncl) * kExactCluster);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, k_tree_exact<Tag, kExactCluster>, p, slice, chunk) != cudaSuccess) {
        (void)cudaGetLastError();
        return SPEC_ECUDA;
    }
    return SPEC_OK;
}

// Largest number of co-resident greedy clusters, per device and dtype.
constexpr int kGreedyCluster = 8;
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

// The workspace form of greedy verification: k_pass1 in the greedy tree
// mode over the k + 1 target rows of each request, then k_greedy_decide as
// its programmatic dependent.
template <class Tag>
int launch_greedy_streamed(Params &p, int dtype_index, cudaStream_t st)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SPEC_ECUDA;
    constexpr int kMin1 = pass1_min_blocks<Tag, kTreeGreedy>();
    int per_sm1, sms;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        per_sm1 = blocks_per_sm(g_pass1_blocks[dev][dtype_index][kTreeGreedy], k_pass1<Tag, kTreeGreedy, kMin1>,
                                kRingBytes);
        sms = sm_count(dev);
    }
    if (per_sm1 < 1 || sms < 1) return SPEC_ECUDA;
    const int64_t blocks1 =
        std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(per_sm1) * sms, ceil_div(p.nA, kWarps)));
    if (prep_pass1(p, blocks1, st) != SPEC_OK) return SPEC_ECUDA;
    k_pass1<Tag, kTreeGreedy, kMin1><<<static_cast<unsigned>(blocks1), kThreads, kRingBytes, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SPEC_ECUDA;
    const int64_t blocksd = std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(4) * sms, p.B));
    return launch_dependent(k_greedy_decide<Tag>, blocksd, 0, st, p);
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
    p.c64 = 1.4426950408889634074 / t;  // log2(e) / T
    p.c = static_cast<float>(p.c64);
    p.seed = seed;
    p.offset = offset;
    p.S2 = static_cast<int>(ceil_div(V, kSeg2));
    p.W32 = p.S2 * (kSeg2 / 32);
    p.poll_limit = kWaitPolls;
    fill_exp2_table(p);
}

// Item counts shared by the linear and tree calls.
int setup_items(Params &p, int R, spec_dtype_t dtype, bool pass2)
{
    p.R = R;
    p.S = static_cast<int>(ceil_div(p.V, dtype == SPEC_BF16 ? Pass1Shape<Bf16>::kItem : Pass1Shape<F32>::kItem));
    const int64_t nA = static_cast<int64_t>(p.B) * R * p.S;
    const int64_t nP = pass2 ? static_cast<int64_t>(p.B) * p.S2 : 0;
    if (nA >= (int64_t(1) << 31) || nP >= (int64_t(1) << 31)) return SPEC_EUNSUPPORTED;
    p.nA = static_cast<unsigned>(nA);
    p.nP = static_cast<unsigned>(nP);
    p.div_req = make_fastdiv(static_cast<uint32_t>(R) * static_cast<uint32_t>(p.S));
    p.div_s = make_fastdiv(static_cast<uint32_t>(p.S));
    p.div_s2 = make_fastdiv(static_cast<uint32_t>(p.S2));
    return SPEC_OK;
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

namespace {

// Batches up to this size take the four-kernel linear path.
constexpr int kFourKernelMaxBatch = 2;

// spec_verify_linear, with the diagnostic switches of
// spec_verify_debug_wait_expiry (poll_limit 0: the normal limit).
int linear_call(const void *target_logits, const void *draft_logits, spec_dtype_t dtype,
                int64_t row_stride, const int32_t *draft_tokens, int batch, int k, int vocab,
                float temperature, uint64_t seed, uint32_t offset, int32_t *out_tokens,
                int32_t *accepted_len, float *dbg_logp, float *dbg_logq, int32_t *status,
                void *workspace, size_t workspace_bytes, cudaStream_t stream, bool diag,
                unsigned poll_limit)
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
    if (static_cast<int64_t>(batch) * (k + 1) > INT_MAX) return SPEC_EUNSUPPORTED;

    Params p;
    base_params(p, target_logits, draft_logits, row_stride, batch, vocab, temperature, seed, offset);
    p.tokens = draft_tokens;
    p.k = k;
    p.out = out_tokens;
    p.acc = accepted_len;
    p.dbg_lp = dbg_logp;
    p.dbg_lq = dbg_logq;
    p.status = status;
    if (diag) {
        p.diag_no_partials = 1;
        p.poll_limit = poll_limit;
    }
    rc = setup_items(p, R, dtype, true);
    if (rc != SPEC_OK) return rc;
    fill_workspace(p, workspace, L);
    // one or two requests leave the one-kernel path nothing to overlap (no
    // later request streams while an earlier one draws): the four
    // programmatic-dependent kernels, each over the whole GPU, finish first
    if (batch <= kFourKernelMaxBatch && !diag)
        return dtype == SPEC_BF16 ? launch_verify<Bf16, kLinear>(p, L, workspace, 1, stream)
                                  : launch_verify<F32, kLinear>(p, L, workspace, 0, stream);
    return dtype == SPEC_BF16 ? launch_fused<Bf16>(p, L, workspace, 1, stream)
                              : launch_fused<F32>(p, L, workspace, 0, stream);
}

}  // namespace

extern "C" int spec_verify_linear(const void *target_logits, const void *draft_logits,
                                  spec_dtype_t dtype, int64_t row_stride,
                                  const int32_t *draft_tokens, int batch, int k, int vocab,
                                  float temperature, uint64_t seed, uint32_t offset,
                                  int32_t *out_tokens, int32_t *accepted_len, float *dbg_logp,
                                  float *dbg_logq, int32_t *status, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream)
{
    return linear_call(target_logits, draft_logits, dtype, row_stride, draft_tokens, batch, k,
                       vocab, temperature, seed, offset, out_tokens, accepted_len, dbg_logp,
                       dbg_logq, status, workspace, workspace_bytes, stream, false, 0);
}

extern "C" int spec_verify_debug_wait_expiry(const void *target_logits, const void *draft_logits,
                                             spec_dtype_t dtype, int64_t row_stride,
                                             const int32_t *draft_tokens, int batch, int k,
                                             int vocab, float temperature, uint32_t poll_limit,
                                             int32_t *out_tokens, int32_t *accepted_len,
                                             int32_t *status, void *workspace,
                                             size_t workspace_bytes, cudaStream_t stream)
{
    if (poll_limit < 1 || poll_limit > SPEC_DEBUG_MAX_POLLS) return SPEC_EINVAL;
    if (!status) return SPEC_EINVAL;
    return linear_call(target_logits, draft_logits, dtype, row_stride, draft_tokens, batch, k,
                       vocab, temperature, 0, 0, out_tokens, accepted_len, nullptr, nullptr,
                       status, workspace, workspace_bytes, stream, true, poll_limit);
}

extern "C" int spec_verify_greedy(const void *target_logits, spec_dtype_t dtype,
                                  int64_t row_stride, const int32_t *draft_tokens, int batch,
                                  int k, int vocab, int32_t *out_tokens, int32_t *accepted_len,
                                  int32_t *status, void *workspace, size_t workspace_bytes,
                                  cudaStream_t stream)
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
    if (!workspace)
        return dtype == SPEC_BF16 ? launch_greedy<Bf16>(p, stream, 1) : launch_greedy<F32>(p, stream, 0);
    // the workspace form: pass 1 as a greedy tree whose N = k + 1 nodes are
    // the target rows, then the linear decide step
    const Layout L = layout(batch, k + 1, vocab);
    if (!L.ok) return SPEC_EINVAL;
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || workspace_bytes < L.total)
        return SPEC_EWORKSPACE;
    p.N = k + 1;
    rc = setup_items(p, k + 1, dtype, false);
    if (rc != SPEC_OK) return rc;
    fill_workspace(p, workspace, L);
    return dtype == SPEC_BF16 ? launch_greedy_streamed<Bf16>(p, 1, stream)
                              : launch_greedy_streamed<F32>(p, 0, stream);
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
    if (stochastic < 0 || stochastic > 2) return SPEC_EINVAL;
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
    if (static_cast<int64_t>(batch) * (max_depth + 1) > INT_MAX) return SPEC_EUNSUPPORTED;

    Params p;
    base_params(p, target_logits, draft_logits, row_stride, batch, vocab,
                stochastic ? temperature : 1.0f, seed, offset);
    p.tokens = node_tokens;
    p.parents = parents;
    p.N = num_nodes;
    p.max_depth = max_depth;
    p.out = out_tokens;
    p.acc = accepted_len;
    p.path = out_path_nodes;
    p.status = status;
    rc = setup_items(p, R, dtype, stochastic == 1);
    if (rc != SPEC_OK) return rc;
    fill_workspace(p, workspace, L);
    if (stochastic == 2)
        return dtype == SPEC_BF16 ? launch_exact<Bf16>(p, 1, stream) : launch_exact<F32>(p, 0, stream);
    if (dtype == SPEC_BF16)
        return stochastic ? launch_verify<Bf16, kTreeStochastic>(p, L, workspace, 1, stream)
                          : launch_verify<Bf16, kTreeGreedy>(p, L, workspace, 1, stream);
    return stochastic ? launch_verify<F32, kTreeStochastic>(p, L, workspace, 0, stream)
                      : launch_verify<F32, kTreeGreedy>(p, L, workspace, 0, stream);
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

extern "C" int spec_verify_debug_exp2(const double *z, double *out, int n, int kind,
                                      cudaStream_t stream)
{
    if (n < 0 || (n > 0 && (!z || !out)) || kind < 0 || kind > 2) return SPEC_EINVAL;
    if (n == 0) return SPEC_OK;
    Params p;
    std::memset(&p, 0, sizeof p);
    fill_exp2_table(p);
    const int blocks = static_cast<int>(ceil_div(n, 256));
    k_debug_exp2<<<blocks, 256, 0, stream>>>(z, out, n, kind, p);
    return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}
