// noalloc.cu -- spec_verify_linear_noalloc: linear verification whose
// scratch memory is a fixed array compiled into the library.
//
// Some callers cannot allocate device memory: a plugin whose host
// framework owns the whole device pool and offers no workspace, or a
// serving loop that bans cudaMalloc once it is running (the call can block
// on the device and can fail under memory pressure).  This entry point
// takes the same inputs and outputs as spec_verify_linear but no workspace:
// it uses kScratchBytes of device memory that every GPU loading the library
// reserves until the process exits.
//
// Set-up: the first call on a device (with that device current) looks up
// the array's device address with cudaGetSymbolAddress; later calls reuse
// it for the life of the process.  Make that first call before any stream
// capture begins.  The cached address does not survive cudaDeviceReset (the
// module is loaded again into the new context): a device must not be reset
// while this library may still be called on it.
// Sharing: all calls on a device use the same array.  Each call clears the
// counters it needs before use, so stale contents from an earlier call do
// no harm, but calls that overlap on the GPU (other streams, other host
// threads) race on the array and must be serialised by the caller.
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/specverify.h"

namespace {

constexpr size_t kScratchBytes = SPEC_NOALLOC_SCRATCH_BYTES;  // per device
constexpr int kMaxDevices = 64;

// In host code this name is only a stand-in for the device symbol: the
// kernels receive the address cudaGetSymbolAddress returns, never this.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once).
int scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SPEC_ECUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return SPEC_ECUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SPEC_OK;
}

}  // namespace

extern "C" int spec_verify_linear_noalloc(const void *target_logits, const void *draft_logits,
                                          spec_dtype_t dtype, int64_t row_stride,
                                          const int32_t *draft_tokens, int batch, int k,
                                          int vocab, float temperature, uint64_t seed,
                                          uint32_t offset, int32_t *out_tokens,
                                          int32_t *accepted_len, float *dbg_logp,
                                          float *dbg_logq, int32_t *status, cudaStream_t stream)
{
    void *scratch = nullptr;
    if (batch > 0 && k >= 1) {
        const size_t need = spec_verify_workspace_size(batch, 2 * k + 1, vocab);
        if (need > kScratchBytes) {
            // beyond the static scratch; but an invalid argument keeps the
            // code spec_verify_linear gives it: without a workspace it runs
            // every other check, enqueues nothing and, if they pass, reports
            // the workspace
            const int rc = spec_verify_linear(target_logits, draft_logits, dtype, row_stride,
                                              draft_tokens, batch, k, vocab, temperature, seed,
                                              offset, out_tokens, accepted_len, dbg_logp, dbg_logq,
                                              status, nullptr, 0, stream);
            return rc == SPEC_EWORKSPACE ? SPEC_EUNSUPPORTED : rc;
        }
        if (need > 0) {
            const int rc = scratch_address(&scratch);
            if (rc != SPEC_OK) return rc;
        }
    }
    return spec_verify_linear(target_logits, draft_logits, dtype, row_stride, draft_tokens, batch,
                              k, vocab, temperature, seed, offset, out_tokens, accepted_len,
                              dbg_logp, dbg_logq, status, scratch, kScratchBytes, stream);
}
