"""Pins of the oracle's linear (stochastic) and greedy verification.

Every pin here comes from outside the oracle: hand arithmetic on tiny rows,
special cases whose outcome is forced, the target-distribution guarantee
("Speculative decoding explained", "Draft and verification loop"), the
accept-length closed form P(n >= j) = prod_{i<j} alpha_i with
alpha_i = sum_v min(p_i(v), q_i(v)) (Leviathan et al.), and brute-force
enumeration at V=8, k=2.
"""
import itertools

import numpy as np
import pytest

from speculative_decoding_verification_87_b200 import workloads as wl
from stats_util import brute_force_linear, chisquare_pvalue, softmax64

LN = np.log


def _f32(rows):
    return np.ascontiguousarray(np.array(rows, dtype=np.float32))


# ---------------------------------------------------------------- hand cases
def _hand_case_1():
    # V=3, k=1, T=1.  p_0 = (.5,.3,.2), q_0 = (.2,.5,.3), x_0 = 1 => p/q = .6
    # bonus row p_1 = (.25,.25,.5)
    tl = _f32([[[LN(.5), LN(.3), LN(.2)], [LN(.25), LN(.25), LN(.5)]]])
    dl = _f32([[[LN(.2), LN(.5), LN(.3)]]])
    x = np.array([[1]], dtype=np.int32)
    return tl, dl, x


def test_hand_accept_then_bonus(orc):
    tl, dl, x = _hand_case_1()
    # u_0 = .5: .5 * .5 = .25 < .3 -> accept.  Bonus CDF (.25,.5,1), u = .6 -> token 2.
    r = orc.verify_linear_u(tl, dl, x, 1.0, [[0.5]], [[0.0, 0.6]])
    assert r["err"][0] == 0
    assert r["acc"][0] == 1
    assert list(r["out"][0]) == [1, 2]
    assert abs(r["logp"][0, 0] - LN(.3)) < 1e-6
    assert abs(r["logq"][0, 0] - LN(.5)) < 1e-6
    assert abs(r["acc_margin"][0, 0] - abs(0.5 - 0.6)) < 1e-6
    # bucket of token 2 is [.5, 1): .6 sits .1 above its lower edge, width .5
    assert abs(r["smp_margin"][0] - 0.1 / 0.5) < 1e-6


def test_hand_reject_then_residual(orc):
    tl, dl, x = _hand_case_1()
    # u_0 = .7: .35 > .3 -> reject.  max(0, p - q) = (.3, 0, 0) -> token 0 for any u.
    for us in (0.0, 0.3, 0.999):
        r = orc.verify_linear_u(tl, dl, x, 1.0, [[0.7]], [[us, 0.5]])
        assert r["acc"][0] == 0
        assert list(r["out"][0]) == [0, -1]


def test_hand_bonus_cdf_edges(orc):
    tl, dl, x = _hand_case_1()
    # C = (.25, .5, 1): u*Z just below .25 -> 0, in [.25, .5) -> 1, >= .5 -> 2
    for us, tok in ((0.0, 0), (0.2, 0), (0.3, 1), (0.49, 1), (0.51, 2), (1 - 2 ** -24, 2)):
        r = orc.verify_linear_u(tl, dl, x, 1.0, [[0.0]], [[0.0, us]])
        assert r["out"][0, 1] == tok, (us, tok)


def test_hand_greedy(orc):
    # V=4, k=2: argmax rows (1,3,3,0)->1 (tie to lowest), (0,0,5,5)->2, (7,7,7,7)->0
    tl = _f32([[[1, 3, 3, 0], [0, 0, 5, 5], [7, 7, 7, 7]]])
    cases = {(1, 2): ([1, 2, 0], 2), (2, 2): ([1, -1, -1], 0), (1, 3): ([1, 2, -1], 1)}
    for drafts, (out, n) in cases.items():
        r = orc.verify_greedy(tl, np.array([drafts], np.int32), 4)
        assert r["err"][0] == 0
        assert list(r["out"][0]) == out and r["acc"][0] == n


# ------------------------------------------------------------ special cases
def test_q_equals_p_accepts_everything(orc):
    w = wl.tiny_linear(seed=3, batch=8, k=4, vocab=32)
    draft = np.ascontiguousarray(w.target[:, :w.k, :])
    for off in range(20):
        r = orc.verify_linear(w.target, draft, w.tokens, w.vocab, 1.0, seed=11, offset=off)
        assert np.all(r["acc"] == w.k)
        assert np.all(r["out"][:, :w.k] == w.tokens)
        assert np.all(np.isinf(r["acc_margin"]))


def test_zero_target_probability_rejects_first(orc):
    # "Best and worst case": the first draft is rejected and replaced.
    w = wl.tiny_linear(seed=4, batch=8, k=4, vocab=32)
    t = w.target.copy()
    for b in range(w.batch):
        t[b, 0, w.tokens[b, 0]] = -np.inf  # p_0(x_0) = 0
    for off in range(50):
        r = orc.verify_linear(t, w.draft, w.tokens, w.vocab, 1.0, seed=5, offset=off)
        assert np.all(r["acc"] == 0)
        assert np.all(r["out"][:, 0] != w.tokens[:, 0])  # residual excludes x_0
        assert np.all(r["out"][:, 1:] == -1)


def test_temperature_scales_logits(orc):
    # softmax(l / T) at T=2 equals softmax((l/2) / 1); halving is exact in fp32
    w = wl.tiny_linear(seed=6, batch=16, k=4, vocab=32)
    r2 = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, 2.0, seed=1, offset=0)
    r1 = orc.verify_linear(w.target * np.float32(0.5), w.draft * np.float32(0.5), w.tokens,
                           w.vocab, 1.0, seed=1, offset=0)
    assert np.array_equal(r1["out"], r2["out"]) and np.array_equal(r1["acc"], r2["acc"])
    assert np.allclose(r1["logp"], r2["logp"], atol=1e-12)


def test_bf16_storage_equals_fp32_of_same_values(orc):
    w = wl.peaked_linear(seed=2, batch=4, k=3, vocab=1000, temperature=0.8)
    t32 = wl.as_f32(w.target, w.vocab).copy()
    d32 = wl.as_f32(w.draft, w.vocab).copy()
    rb = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, 0.8, seed=9, offset=2)
    rf = orc.verify_linear(t32, d32, w.tokens, w.vocab, 0.8, seed=9, offset=2)
    for key in ("out", "acc", "logp", "logq"):
        assert np.array_equal(rb[key], rf[key])


def test_stride_padding_is_ignored(orc):
    w = wl.tiny_linear(seed=8, batch=4, k=3, vocab=29, pad=7)
    assert w.stride > w.vocab
    t = w.target.copy()
    d = w.draft.copy()
    t[..., w.vocab:] = np.nan
    d[..., w.vocab:] = np.nan
    r = orc.verify_linear(t, d, w.tokens, w.vocab, 1.0, seed=2, offset=0)
    assert np.all(r["err"] == 0)
    r2 = orc.verify_linear(np.ascontiguousarray(w.target[..., :w.vocab]),
                           np.ascontiguousarray(w.draft[..., :w.vocab]), w.tokens, w.vocab,
                           1.0, seed=2, offset=0)
    assert np.array_equal(r["out"], r2["out"])


def test_vocab_one(orc):
    t = np.zeros((2, 3, 4), np.float32)
    d = np.zeros((2, 2, 4), np.float32)
    x = np.zeros((2, 2), np.int32)
    r = orc.verify_linear(t, d, x, 1, 1.0, seed=0, offset=0)
    assert np.all(r["acc"] == 2) and np.all(r["out"] == 0)


def test_input_errors(orc):
    w = wl.tiny_linear(seed=9, batch=5, k=2, vocab=16)
    t, d, x = w.target.copy(), w.draft.copy(), w.tokens.copy()
    x[0, 1] = 16          # token out of range
    x[1, 0] = -1
    t[2, 2, 3] = np.nan   # NaN in the bonus row
    d[3, 0, :] = -np.inf  # draft row with no finite maximum
    t[4, 1, 0] = np.inf
    r = orc.verify_linear(t, d, x, w.vocab, 1.0, seed=0, offset=0)
    assert r["err"][0] & orc.ERR_TOKEN and r["err"][1] & orc.ERR_TOKEN
    assert r["err"][2] & orc.ERR_LOGIT and r["err"][3] & orc.ERR_LOGIT
    assert r["err"][4] & orc.ERR_LOGIT
    assert np.all(r["out"] == -1) and np.all(r["acc"] == -1)
    # a partly masked row (some -inf) is valid
    t2 = w.target.copy()
    t2[:, :, :5] = -np.inf
    r2 = orc.verify_linear(t2, w.draft, w.tokens, w.vocab, 1.0, seed=0, offset=0)
    assert np.all(r2["err"] == 0)
    g = orc.verify_greedy(t, x, w.vocab)
    assert g["err"][0] & orc.ERR_TOKEN and g["err"][2] & orc.ERR_LOGIT
    assert g["err"][3] == 0  # greedy never reads draft rows


def test_invariants_on_peaked_batch(orc):
    w = wl.peaked_linear(seed=1, batch=32, k=6, vocab=3000, temperature=0.7, sigma=(0.5, 2.0))
    r = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, 0.7, seed=3, offset=4)
    assert np.all(r["err"] == 0)
    for b in range(w.batch):
        n = r["acc"][b]
        assert 0 <= n <= w.k
        assert np.all(r["out"][b, :n] == w.tokens[b, :n])
        assert 0 <= r["out"][b, n] < w.vocab
        assert np.all(r["out"][b, n + 1:] == -1)
    # log p / log q agree with an fp64 log-softmax of the same row
    for b in range(4):
        for j in range(w.k):
            lp = orc.log_softmax_row(w.target[b, j, :w.vocab], 0.7)
            assert abs(lp[w.tokens[b, j]] - r["logp"][b, j]) < 1e-12


# ---------------------------------------------------- distribution pins
def _trials(orc, base, trials_per_req, chunks, seed=17):
    """Run ``trials_per_req`` independent trials of every request of ``base``
    (fresh drafts each time); returns per-request stacked outputs."""
    outs = [[] for _ in range(base.batch)]
    accs = [[] for _ in range(base.batch)]
    per = trials_per_req // chunks
    for c in range(chunks):
        rep = wl.replicate_requests(base, per, draft_rng_seed=1000 + c)
        r = orc.verify_linear(rep.target, rep.draft, rep.tokens, rep.vocab, rep.temperature,
                              seed=seed, offset=c)
        assert np.all(r["err"] == 0)
        for b in range(base.batch):
            outs[b].append(r["out"][b * per:(b + 1) * per])
            accs[b].append(r["acc"][b * per:(b + 1) * per])
    return [np.concatenate(o) for o in outs], [np.concatenate(a) for a in accs]


@pytest.mark.slow
def test_chi_square_tiny_config_1e6_trials(orc):
    """Emitted tokens follow the target: slot j given n >= j follows p_j
    (the synthetic rows do not depend on the prefix)."""
    base = wl.config_tiny(seed=0)
    T = base.temperature
    p = softmax64(wl.as_f32(base.target, base.vocab), T)
    q = softmax64(wl.as_f32(base.draft, base.vocab), T)
    outs, accs = _trials(orc, base, 1_000_000, 10)
    for b in range(base.batch):
        out, acc = outs[b], accs[b]
        assert np.all((acc >= 0) & (acc <= base.k))
        alpha = np.minimum(p[b, :base.k], q[b]).sum(axis=1)
        for j in range(base.k + 1):
            sel = acc >= j
            counts = np.bincount(out[sel, j], minlength=base.vocab)
            pv, bad = chisquare_pvalue(counts, p[b, j])
            assert bad == 0
            assert pv > 1e-3, (b, j, pv)
        # accept-length closed form: P(n >= j) = prod_{i<j} alpha_i
        hist = np.bincount(acc, minlength=base.k + 1) / len(acc)
        tail = np.concatenate([[1.0], np.cumprod(alpha)])
        expect = tail[:-1] - tail[1:]
        expect = np.append(expect, tail[-1])
        pv, bad = chisquare_pvalue(hist * len(acc), expect)
        assert bad == 0 and pv > 1e-3, (b, pv)


def test_brute_force_rule_keeps_target_joint():
    """The accept/residual rule itself (not the oracle) reproduces the
    target's autoregressive joint: an exact check of the guarantee."""
    rng = np.random.default_rng(0)
    V, k = 8, 2
    p = softmax64(rng.normal(0, 1.5, (k + 1, V)), 1.0)
    q = softmax64(np.log(p[:k]) + rng.normal(0, 0.7, (k, V)), 1.0)
    dist = brute_force_linear(p, q, k)
    assert abs(sum(dist.values()) - 1) < 1e-12
    for j in range(k + 1):
        for z in itertools.product(range(V), repeat=j):
            reach = sum(v for key, v in dist.items() if key[0] >= j and key[1:1 + j] == z)
            for y in range(V):
                got = sum(v for key, v in dist.items()
                          if key[0] >= j and key[1:1 + j] == z and key[1 + j] == y)
                assert abs(got - reach * p[j, y]) < 1e-12


@pytest.mark.slow
def test_brute_force_v8_k2_matches_oracle(orc):
    V, k, T = 8, 2, 1.0
    base = wl.tiny_linear(seed=21, batch=1, k=k, vocab=V)
    p = softmax64(wl.as_f32(base.target, V), T)[0]
    q = softmax64(wl.as_f32(base.draft, V), T)[0]
    dist = brute_force_linear(p, q, k)
    keys = sorted(dist)
    index = {key: i for i, key in enumerate(keys)}
    outs, accs = _trials(orc, base, 400_000, 4)
    out, acc = outs[0], accs[0]
    counts = np.zeros(len(keys))
    unknown = 0
    for o, n in zip(out, acc):
        key = (int(n),) + tuple(int(v) for v in o[:n + 1])
        if key in index:
            counts[index[key]] += 1
        else:
            unknown += 1
    assert unknown == 0
    pv, bad = chisquare_pvalue(counts, [dist[key] for key in keys])
    assert pv > 1e-3, pv
