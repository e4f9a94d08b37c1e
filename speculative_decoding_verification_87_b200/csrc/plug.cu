// plug.cu -- spec_plug_tokens: the next step's input tokens, written on the
// device from a verification's outputs.
//
// "Accelerating Sonar through speculation", section "MTP schedule for one
// token": after verification a kernel plugs the next target tokens into
// their positions, so the accepted count need not travel to the CPU before
// the next step is launched (section "Inference with speculative
// decoding": that count is otherwise a GPU-to-CPU synchronisation point);
// section "MTP": the draft reads the target's input tokens shifted one
// position left of the hidden states.  One warp per request, one lane per
// position; a few hundred bytes per request, so the launch, not the
// memory system, bounds it.
#include <climits>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/specverify.h"

namespace {

constexpr int kPlugThreads = 256;

__global__ void __launch_bounds__(kPlugThreads) k_plug(const int32_t *in, const int32_t *out,
                                                       const int32_t *acc, int B, int k,
                                                       int32_t *next, int32_t *seq, int32_t *len,
                                                       int cap, int32_t *status)
{
    const int lane = threadIdx.x & 31;
    const int64_t b = (static_cast<int64_t>(blockIdx.x) * kPlugThreads + threadIdx.x) >> 5;
    if (b >= B) return;
    const int W = k + 1;
    const int n = __ldg(acc + b);
    int bits = 0;
    if (n < 0 || n > k) {
        if (n != -1) bits |= SPEC_STATUS_TOKEN;
        if (next)
            for (int i = lane; i < W; i += 32) next[b * W + i] = -1;
    } else {
        const int en = __ldg(out + b * W + n);
        if (next)
            for (int i = lane; i < W; i += 32)
                next[b * W + i] = (i == n || i == k) ? en : __ldg(in + b * W + i + 1);
        if (seq) {
            int L = 0;
            if (lane == 0) L = len[b];
            L = __shfl_sync(0xFFFFFFFFu, L, 0);
            if (L < 0 || static_cast<int64_t>(L) + n + 1 > cap) {
                bits |= SPEC_STATUS_CAPACITY;
            } else {
                for (int j = lane; j <= n; j += 32)
                    seq[b * static_cast<int64_t>(cap) + L + j] = __ldg(out + b * W + j);
                if (lane == 0) len[b] = L + n + 1;
            }
        }
    }
    if (lane == 0 && status && bits) atomicOr(status, bits);
}

}  // namespace

extern "C" int spec_plug_tokens(const int32_t *in_tokens, const int32_t *out_tokens,
                                const int32_t *accepted_len, int batch, int k,
                                int32_t *next_tokens, int32_t *seq_tokens, int32_t *seq_len,
                                int capacity, int32_t *status, cudaStream_t stream)
{
    if (batch < 0 || k < 1 || capacity < 0) return SPEC_EINVAL;
    if (k > SPEC_MAX_K) return SPEC_EUNSUPPORTED;
    if ((seq_tokens == nullptr) != (seq_len == nullptr)) return SPEC_EINVAL;
    if (batch == 0) return SPEC_OK;
    if (!out_tokens || !accepted_len || (next_tokens && !in_tokens)) return SPEC_EINVAL;
    if (!next_tokens && !seq_tokens) return SPEC_OK;  // nothing asked for
    const int64_t blocks = (static_cast<int64_t>(batch) * 32 + kPlugThreads - 1) / kPlugThreads;
    if (blocks > INT_MAX) return SPEC_EUNSUPPORTED;
    k_plug<<<static_cast<unsigned>(blocks), kPlugThreads, 0, stream>>>(
        in_tokens, out_tokens, accepted_len, batch, k, next_tokens, seq_tokens, seq_len, capacity,
        status);
    return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}
