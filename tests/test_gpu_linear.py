"""GPU parity of spec_verify_linear against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_87_b200 import workloads as wl
from parity import (FlagTally, LinearOnDevice, compare_linear, oracle_linear_many, run_linear_gpu,
                    to_device)
from stats_util import brute_force_linear, chisquare_pvalue, softmax64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from speculative_decoding_verification_87_b200 import binding, build
    build.build()
    binding.load_library()
    return binding


def test_device_philox_matches_oracle(sv, orc):
    for purpose, first in ((0, 0), (1, 5)):
        g = sv.spec_verify_debug_uniforms(0xDEADBEEF12345678, 77, purpose, 1000, 1000, first)
        o = orc.uniforms(0xDEADBEEF12345678, 77, purpose, 1000, 1000, first)
        assert np.array_equal(g.cpu().numpy(), o)


def test_tiny_config_matches_oracle(sv, orc):
    w = wl.config_tiny(seed=0)
    tally = FlagTally()
    for off in range(50):
        g = run_linear_gpu(sv, w, seed=0, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 0, off)
        assert g["status"] == 0
        tally.add(compare_linear(g, o, w.k))
    tally.check()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("vocab,pad", [(5000, 0), (4097, 3), (12345, 9), (1, 0), (8193, 0)])
def test_ragged_vocab_and_stride(sv, orc, dtype, vocab, pad):
    w = wl.peaked_linear(seed=vocab, batch=6, k=3, vocab=vocab, temperature=0.8,
                         sigma=(0.5, 2.0), dtype=dtype, pad=pad)
    # garbage past the vocabulary must never be read as a logit
    t, d = w.target.copy(), w.draft.copy()
    if t.shape[-1] > vocab:
        nan = np.uint16(0x7FC0) if dtype == "bf16" else np.float32(np.nan)
        t[..., vocab:] = nan
        d[..., vocab:] = nan
    w.target, w.draft = t, d
    tally = FlagTally()
    for off in range(8):
        g = run_linear_gpu(sv, w, seed=3, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 3, off)
        assert g["status"] == 0 and np.all(o["err"] == 0)
        tally.add(compare_linear(g, o, w.k))
    tally.check()


@pytest.mark.parametrize("k", [1, 2, 7, 32])
def test_draft_counts(sv, orc, k):
    w = wl.peaked_linear(seed=100 + k, batch=8, k=k, vocab=3000, temperature=1.0,
                         sigma=(0.2, 0.6))
    tally = FlagTally()
    for off in range(4):
        g = run_linear_gpu(sv, w, seed=9, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 9, off)
        tally.add(compare_linear(g, o, w.k))
    tally.check()


def test_special_cases(sv, orc):
    w = wl.tiny_linear(seed=3, batch=16, k=4, vocab=64)
    # q == p: every draft accepted, bonus from row k
    eq = wl.LinearWorkload("eq", w.target, np.ascontiguousarray(w.target[:, :4]), w.tokens, 64,
                           1.0, "f32")
    tally = FlagTally()
    for off in range(10):
        g = run_linear_gpu(sv, eq, seed=1, offset=off)
        assert np.all(g["acc"] == 4)
        o = orc.verify_linear(eq.target, eq.draft, eq.tokens, 64, 1.0, 1, off)
        tally.add(compare_linear(g, o, 4))
    # p_0(x_0) == 0: first draft always rejected, residual never returns x_0
    t = w.target.copy()
    for b in range(16):
        t[b, 0, w.tokens[b, 0]] = -np.inf
    z = wl.LinearWorkload("zero", t, w.draft, w.tokens, 64, 1.0, "f32")
    for off in range(10):
        g = run_linear_gpu(sv, z, seed=1, offset=off)
        assert np.all(g["acc"] == 0)
        assert np.all(g["out"][:, 0] != w.tokens[:, 0])
        # log p_0(x_0) = -inf on both sides (checked by compare_linear)
        assert np.all(np.isneginf(g["logp"][:, 0]))
        o = orc.verify_linear(z.target, z.draft, z.tokens, 64, 1.0, 1, off)
        tally.add(compare_linear(g, o, 4))
    tally.check()


def test_input_errors_are_reported(sv, orc):
    w = wl.tiny_linear(seed=9, batch=6, k=2, vocab=16)
    t, d, x = w.target.copy(), w.draft.copy(), w.tokens.copy()
    x[0, 1] = 16
    x[1, 0] = -1
    t[2, 2, 3] = np.nan
    d[3, 0, :] = -np.inf
    t[4, 1, 0] = np.inf
    bad = wl.LinearWorkload("bad", t, d, x, 16, 1.0, "f32")
    g = run_linear_gpu(sv, bad, seed=0, offset=0, dbg=False)
    o = orc.verify_linear(t, d, x, 16, 1.0, 0, 0)
    assert g["status"] == (1 | 4)
    assert np.array_equal(g["acc"], o["acc"]) and np.array_equal(g["out"], o["out"])
    assert np.all(g["acc"][:5] == -1) and g["acc"][5] >= 0


def test_empty_batch(sv):
    t = torch.zeros((0, 3, 16), dtype=torch.float32, device="cuda")
    d = torch.zeros((0, 2, 16), dtype=torch.float32, device="cuda")
    x = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    out, acc = sv.spec_verify_linear(t, d, x, 16, 1.0)
    assert out.shape == (0, 3) and acc.shape == (0,)


def test_host_side_argument_errors(sv):
    t = torch.zeros((2, 3, 16), dtype=torch.float32, device="cuda")
    d = torch.zeros((2, 2, 16), dtype=torch.float32, device="cuda")
    x = torch.zeros((2, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(sv.SpecVerifyError, match="-1"):
        sv.spec_verify_linear(t, d, x, 16, 0.0)  # temperature must be > 0
    with pytest.raises(sv.SpecVerifyError, match="-1"):
        sv.spec_verify_linear(t, d, x, 17, 1.0)  # vocab > stride
    t2 = torch.zeros((2, 3, 18), dtype=torch.float32, device="cuda")
    d2 = torch.zeros((2, 2, 18), dtype=torch.float32, device="cuda")
    with pytest.raises(sv.SpecVerifyError, match="-2"):
        sv.spec_verify_linear(t2, d2, x, 16, 1.0)  # 72-byte rows are not 16-byte multiples


def _full_size(sv, orc, w, seed, offsets):
    """GPU calls at every offset (inputs resident, outputs read once) against
    the oracle's, spread over the host's cores; returns the tally and the
    GPU's accepted lengths."""
    dev = LinearOnDevice(sv, w)
    gpu = dev.run_many(seed, offsets)
    orcs = oracle_linear_many(orc, w, seed, offsets)
    tally = FlagTally()
    lens = []
    for g, o in zip(gpu, orcs):
        assert g["status"] == 0
        tally.add(compare_linear(g, o, w.k))
        lens.extend(g["acc"].tolist())
    return tally, np.array(lens)


def test_batched_config_100_offsets(sv, orc):
    """B=64, k=8, V=128256 bf16, T=0.7 at 100 offsets: 6400 requests,
    more than 2e4 decisions plus draws, so the 1e-4 flag budget is tested
    against the expected rate of about 2e-5 per trial."""
    w = wl.config_batched(seed=0)
    tally, lens = _full_size(sv, orc, w, 123, range(100))
    t = tally.check(min_trials=20_000)
    print("batched", t, "mean accepted", lens.mean())
    assert lens.min() == 0 and lens.max() == w.k  # residual and bonus draws both exercised


def test_single_config_3000_steps(sv, orc):
    """B=1, k=4, V=128256 bf16, T=1: 3000 seeded steps (offsets), more than
    1e4 decisions plus draws."""
    w = wl.config_single(seed=0)
    tally, lens = _full_size(sv, orc, w, 123, range(3000))
    t = tally.check(min_trials=10_000)
    print("single", t, "mean accepted", lens.mean())


def test_tiny_config_1e6_trials(sv, orc):
    """GPU outputs equal the oracle's on 1e6 trials per request of the tiny
    configuration, and follow the target distribution (chi-square)."""
    base = wl.config_tiny(seed=0)
    p = softmax64(wl.as_f32(base.target, base.vocab), base.temperature)
    per_chunk, chunks = 250_000, 4
    outs = [[] for _ in range(base.batch)]
    accs = [[] for _ in range(base.batch)]
    tally = FlagTally()
    for c in range(chunks):
        rep = wl.replicate_requests(base, per_chunk, draft_rng_seed=5000 + c)
        g = run_linear_gpu(sv, rep, seed=31, offset=c, dbg=False)
        (o,) = oracle_linear_many(orc, rep, 31, [c])
        tally.add(compare_linear(g, o, rep.k, check_logp=False))
        for b in range(base.batch):
            outs[b].append(g["out"][b * per_chunk:(b + 1) * per_chunk])
            accs[b].append(g["acc"][b * per_chunk:(b + 1) * per_chunk])
    print("tiny 1e6", tally.check())
    for b in range(base.batch):
        out, acc = np.concatenate(outs[b]), np.concatenate(accs[b])
        for j in range(base.k + 1):
            sel = acc >= j
            counts = np.bincount(out[sel, j], minlength=base.vocab)
            pv, bad = chisquare_pvalue(counts, p[b, j])
            assert bad == 0 and pv > 1e-3, (b, j, pv)


def test_brute_force_v8_k2_on_gpu(sv, orc):
    """4e5 GPU trials at V=8, k=2 (fresh drafts each): the frequencies of
    (accepted length, emitted tokens) match the exact joint enumerated over
    every draft sequence, and every output equals the oracle's."""
    V, k, T = 8, 2, 1.0
    base = wl.tiny_linear(seed=21, batch=1, k=k, vocab=V)
    p = softmax64(wl.as_f32(base.target, V), T)[0]
    q = softmax64(wl.as_f32(base.draft, V), T)[0]
    dist = brute_force_linear(p, q, k)
    keys = sorted(dist)
    index = {key: i for i, key in enumerate(keys)}
    counts = np.zeros(len(keys))
    tally = FlagTally()
    unknown = 0
    for c in range(4):
        rep = wl.replicate_requests(base, 100_000, draft_rng_seed=7000 + c)
        g = run_linear_gpu(sv, rep, seed=17, offset=c, dbg=False)
        (o,) = oracle_linear_many(orc, rep, 17, [c])
        tally.add(compare_linear(g, o, k, check_logp=False))
        for row, n in zip(g["out"], g["acc"]):
            key = (int(n),) + tuple(int(v) for v in row[:n + 1])
            if key in index:
                counts[index[key]] += 1
            else:
                unknown += 1
    print("brute force v8 k2", tally.check(min_trials=400_000))
    assert unknown == 0
    pv, bad = chisquare_pvalue(counts, [dist[key] for key in keys])
    assert bad == 0 and pv > 1e-3, pv


def test_near_identical_rows_mark_many_entries(sv, orc):
    """Draft rows within ~1% of the target rows: residual draws whose p - q
    sign is undecided from fp32 for many entries (resolved exactly)."""
    w = wl.peaked_linear(seed=31, batch=32, k=32, vocab=20000, temperature=1.0,
                         sigma=(0.02, 0.02), dtype="f32")
    tally, lens = _full_size(sv, orc, w, 5, range(3))
    tally.check()
    assert int(np.sum(lens < w.k)) > 0


def test_masked_vocabulary_is_never_drawn(sv, orc):
    """-inf logits (a masked tail and scattered holes) in both rows."""
    w = wl.peaked_linear(seed=41, batch=24, k=4, vocab=20000, temperature=0.9,
                         sigma=(0.5, 2.0), dtype="bf16")
    V = w.vocab
    rng = np.random.default_rng(7)
    holes = rng.choice(15000, size=500, replace=False)
    t, d = w.target.copy(), w.draft.copy()
    for a in (t, d):
        a[..., 15000:V] = np.uint16(0xFF80)
        a[..., holes] = np.uint16(0xFF80)
    w.target, w.draft = t, d
    w.tokens = wl.gumbel_max(rng, wl.as_f32(d, V), w.temperature).astype(np.int32)
    masked = np.zeros(V, bool)
    masked[15000:] = True
    masked[holes] = True
    tally = FlagTally()
    for off in range(4):
        g = run_linear_gpu(sv, w, seed=9, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 9, off)
        assert g["status"] == 0
        tally.add(compare_linear(g, o, w.k))
        out = g["out"]
        assert not np.any(masked[out[out >= 0]])
    tally.check()


def test_more_requests_than_task_warps(sv, orc):
    """B = 700: the decide tasks outnumber the warps that take tasks first."""
    w = wl.peaked_linear(seed=51, batch=700, k=3, vocab=2000, temperature=1.0,
                         sigma=(0.5, 2.0), dtype="bf16")
    tally, _ = _full_size(sv, orc, w, 11, range(1))
    tally.check()


def test_expired_waits_end_the_kernel_with_a_status(sv, orc):
    """The diagnostic call stores no pass-1 partial, so every bounded wait
    of the one-kernel path runs out: the kernel must return (no hang) with
    SPEC_STATUS_TIMEOUT set and every output left at -1, and the next
    normal call on the same workspace and context must be correct."""
    w = wl.peaked_linear(seed=61, batch=8, k=4, vocab=20000, temperature=0.9,
                         sigma=(0.5, 2.0), dtype="bf16")
    tl, dl = to_device(w.target), to_device(w.draft)
    x = to_device(w.tokens.astype(np.int32))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, acc = sv.spec_verify_debug_wait_expiry(tl, dl, x, w.vocab, w.temperature, 32, status)
    torch.cuda.synchronize()
    assert int(status.item()) & sv.STATUS_TIMEOUT
    assert np.all(out.cpu().numpy() == -1) and np.all(acc.cpu().numpy() == -1)
    tally = FlagTally()
    g = run_linear_gpu(sv, w, seed=2, offset=0)
    o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 2, 0)
    assert g["status"] == 0
    tally.add(compare_linear(g, o, w.k))
    tally.check()


def test_both_linear_paths_agree_across_the_batch_boundary(sv, orc):
    """Batches of one or two requests take the four-kernel path, larger ones
    the one-kernel path.  The uniforms are keyed by request index, so the
    first requests of a batch of 3 (one kernel), 2 and 1 (four kernels) must
    give the same outputs (the two paths merge the normalisers in different
    orders, so only trials inside the oracle's margins may differ), and
    match the oracle under the parity rules."""
    import dataclasses
    w3 = wl.peaked_linear(seed=71, batch=3, k=6, vocab=30011, temperature=0.8, sigma=(0.5, 2.0))
    tally = FlagTally()
    outs = {}
    for B in (3, 2, 1):
        w = dataclasses.replace(w3, target=w3.target[:B].copy(), draft=w3.draft[:B].copy(),
                                tokens=w3.tokens[:B].copy())
        for off in range(40):
            g = run_linear_gpu(sv, w, seed=5, offset=off)
            o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 5, off)
            assert g["status"] == 0
            tally.add(compare_linear(g, o, w.k))
            flagged = (o["smp_margin"] < 1e-5) | (o["acc_margin"] < 1e-5).any(axis=1)
            outs[(B, off)] = (g["out"], g["acc"], flagged)
    tally.check()
    for off in range(40):
        o3, a3, f3 = outs[(3, off)]
        for B in (2, 1):
            oB, aB, fB = outs[(B, off)]
            same = np.all(oB == o3[:B], axis=1) & (aB == a3[:B])
            assert np.all(same | fB | f3[:B]), (B, off)
