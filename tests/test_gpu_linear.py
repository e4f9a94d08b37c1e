"""GPU parity of spec_verify_linear against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_87_b200 import workloads as wl
from parity import compare_linear, run_linear_gpu, to_device
from stats_util import chisquare_pvalue, softmax64

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
    for off in range(50):
        g = run_linear_gpu(sv, w, seed=0, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 0, off)
        assert g["status"] == 0
        compare_linear(g, o, w.k)


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
    for off in range(8):
        g = run_linear_gpu(sv, w, seed=3, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 3, off)
        assert g["status"] == 0 and np.all(o["err"] == 0)
        compare_linear(g, o, w.k)


@pytest.mark.parametrize("k", [1, 2, 7, 32])
def test_draft_counts(sv, orc, k):
    w = wl.peaked_linear(seed=100 + k, batch=8, k=k, vocab=3000, temperature=1.0,
                         sigma=(0.2, 0.6))
    for off in range(4):
        g = run_linear_gpu(sv, w, seed=9, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 9, off)
        compare_linear(g, o, w.k)


def test_special_cases(sv, orc):
    w = wl.tiny_linear(seed=3, batch=16, k=4, vocab=64)
    # q == p: every draft accepted, bonus from row k
    eq = wl.LinearWorkload("eq", w.target, np.ascontiguousarray(w.target[:, :4]), w.tokens, 64,
                           1.0, "f32")
    for off in range(10):
        g = run_linear_gpu(sv, eq, seed=1, offset=off)
        assert np.all(g["acc"] == 4)
        o = orc.verify_linear(eq.target, eq.draft, eq.tokens, 64, 1.0, 1, off)
        compare_linear(g, o, 4)
    # p_0(x_0) == 0: first draft always rejected, residual never returns x_0
    t = w.target.copy()
    for b in range(16):
        t[b, 0, w.tokens[b, 0]] = -np.inf
    z = wl.LinearWorkload("zero", t, w.draft, w.tokens, 64, 1.0, "f32")
    for off in range(10):
        g = run_linear_gpu(sv, z, seed=1, offset=off)
        assert np.all(g["acc"] == 0)
        assert np.all(g["out"][:, 0] != w.tokens[:, 0])
        o = orc.verify_linear(z.target, z.draft, z.tokens, 64, 1.0, 1, off)
        compare_linear(g, o, 4)


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


@pytest.mark.parametrize("cfg", ["single", "batched"])
def test_full_size_configs(sv, orc, cfg):
    w = wl.config_single(seed=0) if cfg == "single" else wl.config_batched(seed=0)
    offsets = range(24) if cfg == "single" else range(3)
    tot = dict(trials=0, flagged_trials=0, flagged_mismatch=0)
    lens = []
    for off in offsets:
        g = run_linear_gpu(sv, w, seed=123, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 123, off)
        assert g["status"] == 0
        r = compare_linear(g, o, w.k)
        for key in tot:
            tot[key] += r[key]
        lens.extend(g["acc"].tolist())
    print(cfg, tot, "mean accepted", np.mean(lens))
    if cfg == "batched":
        assert min(lens) == 0 or max(lens) == w.k or len(set(lens)) > 3


def test_tiny_config_1e6_trials(sv, orc):
    """GPU outputs equal the oracle's on 1e6 trials per request of the tiny
    configuration, and follow the target distribution (chi-square)."""
    base = wl.config_tiny(seed=0)
    p = softmax64(wl.as_f32(base.target, base.vocab), base.temperature)
    per_chunk, chunks = 250_000, 4
    outs = [[] for _ in range(base.batch)]
    accs = [[] for _ in range(base.batch)]
    tot = dict(trials=0, flagged_trials=0, flagged_mismatch=0)
    for c in range(chunks):
        rep = wl.replicate_requests(base, per_chunk, draft_rng_seed=5000 + c)
        g = run_linear_gpu(sv, rep, seed=31, offset=c, dbg=False)
        o = orc.verify_linear(rep.target, rep.draft, rep.tokens, rep.vocab, rep.temperature, 31, c)
        r = compare_linear(g, o, rep.k, check_logp=False)
        for key in tot:
            tot[key] += r[key]
        for b in range(base.batch):
            outs[b].append(g["out"][b * per_chunk:(b + 1) * per_chunk])
            accs[b].append(g["acc"][b * per_chunk:(b + 1) * per_chunk])
    assert tot["flagged_trials"] <= 1e-4 * tot["trials"], tot
    for b in range(base.batch):
        out, acc = np.concatenate(outs[b]), np.concatenate(accs[b])
        for j in range(base.k + 1):
            sel = acc >= j
            counts = np.bincount(out[sel, j], minlength=base.vocab)
            pv, bad = chisquare_pvalue(counts, p[b, j])
            assert bad == 0 and pv > 1e-3, (b, j, pv)


def test_near_identical_rows_mark_many_entries(sv, orc):
    """Draft rows within ~1% of the target rows: residual draws whose p - q
    sign is undecided from fp32 for many entries (resolved exactly)."""
    w = wl.peaked_linear(seed=31, batch=32, k=32, vocab=20000, temperature=1.0,
                         sigma=(0.02, 0.02), dtype="f32")
    residual = 0
    for off in range(3):
        g = run_linear_gpu(sv, w, seed=5, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 5, off)
        assert g["status"] == 0
        compare_linear(g, o, w.k)
        residual += int(np.sum(g["acc"] < w.k))
    assert residual > 0


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
    for off in range(4):
        g = run_linear_gpu(sv, w, seed=9, offset=off)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 9, off)
        assert g["status"] == 0
        compare_linear(g, o, w.k)
        out = g["out"]
        assert not np.any(masked[out[out >= 0]])


def test_more_requests_than_task_warps(sv, orc):
    """B = 700: the decide tasks outnumber the warps that take tasks first."""
    w = wl.peaked_linear(seed=51, batch=700, k=3, vocab=2000, temperature=1.0,
                         sigma=(0.5, 2.0), dtype="bf16")
    g = run_linear_gpu(sv, w, seed=11, offset=0)
    o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 11, 0)
    assert g["status"] == 0
    compare_linear(g, o, w.k)
