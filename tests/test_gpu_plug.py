"""GPU parity of spec_plug_tokens with the oracle's token plug (bit-exact),
on random verification outputs with error and capacity cases, and chained
directly after spec_verify_linear on the device."""
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


def _random_case(rng, B, k, cap):
    inp = rng.integers(0, 1000, (B, k + 1)).astype(np.int32)
    acc = rng.integers(-1, k + 1, B).astype(np.int32)
    acc[rng.random(B) < 0.03] = k + 3             # malformed accepted lengths
    out = np.full((B, k + 1), -1, np.int32)
    for b in range(B):
        n = acc[b]
        if 0 <= n <= k:
            out[b, :n] = inp[b, 1:n + 1]
            out[b, n] = rng.integers(0, 1000)
    seq = rng.integers(0, 1000, (B, cap)).astype(np.int32)
    ln = rng.integers(0, cap - k + 2, B).astype(np.int32)  # some rows without room
    ln[rng.random(B) < 0.02] = -3
    return inp, out, acc, seq, ln


@pytest.mark.parametrize("B,k", [(1, 1), (37, 4), (1000, 8), (300, 32)])
def test_plug_matches_oracle(sv, orc, B, k):
    rng = np.random.default_rng(B * 100 + k)
    cap = 3 * (k + 1)
    inp, out, acc, seq, ln = _random_case(rng, B, k, cap)
    o = orc.plug_tokens(inp, out, acc, seq, ln)
    seq_d, ln_d = to_device(seq), to_device(ln)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nxt = sv.spec_plug_tokens(to_device(inp), to_device(out), to_device(acc), seq_tokens=seq_d,
                              seq_len=ln_d, status=status)
    torch.cuda.synchronize()
    assert np.array_equal(nxt.cpu().numpy(), o["next"])
    assert np.array_equal(seq_d.cpu().numpy(), o["seq"])
    assert np.array_equal(ln_d.cpu().numpy(), o["len"])
    assert int(status.item()) == o["err"]


def test_plug_after_linear_verification_on_device(sv, orc):
    """Verification outputs feed the plug without leaving the device; the
    result equals the oracle's plug of the oracle's verification."""
    w = wl.peaked_linear(seed=77, batch=48, k=6, vocab=5000, temperature=0.8, sigma=(0.5, 2.0))
    B, k = w.batch, w.k
    last = np.arange(B, dtype=np.int32)[:, None] + 17       # the last committed tokens
    inp = np.concatenate([last, w.tokens.astype(np.int32)], axis=1)
    seq = np.zeros((B, 64), np.int32)
    ln = np.full(B, 5, np.int32)
    out_d, acc_d = sv.spec_verify_linear(to_device(w.target), to_device(w.draft),
                                         to_device(w.tokens.astype(np.int32)), w.vocab,
                                         w.temperature, 3, 1)
    seq_d, ln_d = to_device(seq), to_device(ln)
    nxt = sv.spec_plug_tokens(to_device(inp), out_d, acc_d, seq_tokens=seq_d, seq_len=ln_d)
    torch.cuda.synchronize()
    ov = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 3, 1)
    flagged = (ov["smp_margin"] < 1e-5) | (ov["acc_margin"] < 1e-5).any(axis=1)
    assert not flagged.any()  # this seed has no trial within the margins
    assert np.array_equal(out_d.cpu().numpy(), ov["out"])
    o = orc.plug_tokens(inp, ov["out"], ov["acc"], seq, ln)
    assert np.array_equal(nxt.cpu().numpy(), o["next"])
    assert np.array_equal(seq_d.cpu().numpy(), o["seq"]) and np.array_equal(ln_d.cpu().numpy(), o["len"])
