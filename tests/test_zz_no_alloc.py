"""spec_verify_linear_noalloc: the linear verification entry point that
allocates nothing.

It exists for callers that cannot allocate device memory, such as a plugin
whose host framework owns the whole device pool and offers no workspace,
or a serving loop that forbids cudaMalloc while it runs.  Such a caller
passes only inputs and outputs; the library uses a static scratch array
compiled into it.  These tests call it through the C ABI and check that two
calls in a row (with different batch sizes, so the second runs over the
first one's leftover scratch contents) give exactly the tokens and
accepted lengths of spec_verify_linear, and that a request needing more
scratch than the array holds is refused before anything runs.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from speculative_decoding_verification_87_b200 import workloads as wl
from parity import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from speculative_decoding_verification_87_b200 import binding, build
    build.build()
    binding.load_library()
    return binding


def _both(sv, w, seed, offset):
    tl, dl = to_device(w.target), to_device(w.draft)
    x = to_device(w.tokens.astype(np.int32))
    B, k = w.batch, w.k
    ref_out, ref_acc = sv.spec_verify_linear(tl, dl, x, w.vocab, w.temperature, seed, offset)
    out = torch.full((B, k + 1), -7, dtype=torch.int32, device="cuda")
    acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    lp = torch.empty((B, k), dtype=torch.float32, device="cuda")
    ref_lp = torch.empty((B, k), dtype=torch.float32, device="cuda")
    sv.spec_verify_linear(tl, dl, x, w.vocab, w.temperature, seed, offset, dbg_logp=ref_lp)
    sv.spec_verify_linear_noalloc(tl, dl, x, w.vocab, w.temperature, seed, offset, out, acc,
                                  dbg_logp=lp)
    torch.cuda.synchronize()
    return (ref_out.cpu().numpy(), ref_acc.cpu().numpy(), ref_lp.cpu().numpy(),
            out.cpu().numpy(), acc.cpu().numpy(), lp.cpu().numpy())


def test_noalloc_matches_workspace_entry_point_twice(sv):
    first = wl.peaked_linear(seed=31, batch=24, k=8, vocab=128256, temperature=0.7,
                             sigma=(0.5, 2.0))
    second = wl.peaked_linear(seed=32, batch=9, k=5, vocab=50021, temperature=1.0,
                              sigma=(0.5, 2.0), pad=3)
    for w, offset in ((first, 0), (second, 1)):
        assert sv.workspace_size(w.batch, 2 * w.k + 1, w.vocab) <= sv.NOALLOC_SCRATCH_BYTES
        ref_out, ref_acc, ref_lp, out, acc, lp = _both(sv, w, seed=99, offset=offset)
        # same kernels, same inputs: tokens and lengths exactly equal, log p
        # within the parity tolerance (1e-5)
        assert np.array_equal(out, ref_out)
        assert np.array_equal(acc, ref_acc)
        assert np.all(np.abs(lp - ref_lp) <= 1e-5)
        assert np.all((acc >= 0) & (acc <= w.k))


def test_noalloc_refuses_requests_beyond_its_scratch(sv):
    lib = sv.load_library()
    B, k, V = 4096, 8, 128256
    assert sv.workspace_size(B, 2 * k + 1, V) > sv.NOALLOC_SCRATCH_BYTES
    P = ctypes.c_void_p
    # refused on the host before any pointer is touched
    rc = lib.spec_verify_linear_noalloc(P(0x1000), P(0x2000), 1, V, P(0x3000), B, k, V, 1.0, 0,
                                        0, P(0x4000), P(0x5000), None, None, None, None)
    assert rc == -3  # SPEC_EUNSUPPORTED
