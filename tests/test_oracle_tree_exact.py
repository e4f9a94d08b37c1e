"""Pins of the oracle's distribution-exact tree mode (recursive rejection
over siblings): hand-worked cases, equality with the linear mode on chain
trees, the root-only draw, input errors, and a chi-square over 1e6 trials
showing that the emitted tokens follow the target distribution when every
node's children are independent draws from its draft distribution (with a
negative control: the independent-test tree mode fails the same test), and
the closed form of a chain of rejections: after r rejections the residual
is norm(max(0, p - c_r q)), one threshold per node."""
import numpy as np
from scipy import stats

from speculative_decoding_verification_87_b200 import workloads as wl
from stats_util import softmax64


def _rows(p):
    return np.log(np.asarray(p, np.float64)).astype(np.float32)


def _hand(orc, tokens, ua, us):
    # root p = (.5, .3, .2), q = (.2, .5, .3); both children's target rows
    # are (.25, .25, .5)
    tl = _rows([[.5, .3, .2], [.25, .25, .5], [.25, .25, .5]])[None]
    dl = _rows([[.2, .5, .3], [.2, .5, .3], [.2, .5, .3]])[None]
    par = np.array([[-1, 0, 0]], np.int32)
    tok = np.array([[-1] + list(tokens)], np.int32)
    return orc.verify_tree_exact_u(tl, dl, tok, par, 1, 3, 1.0, np.array([[0.0] + list(ua)]),
                                   np.array([us]))


def test_hand_cases(orc):
    # child 1 (token 1): p/q = .6 < u = .7, rejected; residual (.3, 0, 0)/.3;
    # child 2 (token 1): p'(1) = 0, rejected; residual (.8, 0, 0)/.8: token 0
    r = _hand(orc, (1, 1), (0.7, 0.1), [0.9, 0.9, 0.9])
    assert r["out"].tolist() == [[0, -1]] and r["acc"].tolist() == [0]
    assert abs(r["acc_margin"][0, 1] - 0.1) < 1e-6 and np.isinf(r["acc_margin"][0, 2])
    # child 2 (token 0) against the residual (1, 0, 0): p'/q = 5, accepted
    # whatever u; node 2 has no children: draw from (.25, .25, .5) at u = .6
    r = _hand(orc, (1, 0), (0.7, 0.99), [0.0, 0.0, 0.6])
    assert r["out"].tolist() == [[0, 2]] and r["acc"].tolist() == [1]
    assert r["path"].tolist() == [[0, 2]]
    # child 1 accepted (u = .5 < .6): child 2 is never tested; draw at node 1
    r = _hand(orc, (1, 1), (0.5, 0.0), [0.0, 0.3, 0.0])
    assert r["out"].tolist() == [[1, 1]] and r["acc"].tolist() == [1]
    assert np.isinf(r["acc_margin"][0, 2])


def test_chain_tree_equals_linear_mode(orc):
    # one child per node: every step is the linear rule, same numbers
    for seed, dtype in ((0, "bf16"), (1, "f32"), (2, "bf16")):
        w = wl.peaked_linear(seed=seed, batch=24, k=5, vocab=700, temperature=0.8,
                             sigma=(0.5, 2.0), dtype=dtype)
        c = wl.chain_tree_from_linear(w)
        lin = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 9, seed)
        ex = orc.verify_tree_exact(c.target, c.draft, c.node_tokens, c.parents, c.max_depth,
                                   c.vocab, c.temperature, 9, seed)
        assert np.array_equal(lin["out"], ex["out"]) and np.array_equal(lin["acc"], ex["acc"])
        assert np.array_equal(lin["smp_margin"], ex["smp_margin"])
        assert len(set(lin["acc"].tolist())) >= 3


def test_root_only_draws_from_the_target_row(orc):
    rng = np.random.default_rng(4)
    V = 50
    row = rng.normal(0, 2, size=(1, 1, V)).astype(np.float32)
    p = softmax64(row[0, 0], 0.9)
    cdf = np.cumsum(p)
    for u in (0.0, 0.123, 0.5, 0.987):
        r = orc.verify_tree_exact_u(row, row, np.array([[-1]], np.int32),
                                    np.array([[-1]], np.int32), 1, V, 0.9, np.zeros((1, 1)),
                                    np.array([[u]]))
        assert r["acc"][0] == 0 and r["out"][0, 0] == int(np.searchsorted(cdf, u, side="right"))


def test_errors_match_the_tree_mode(orc):
    base = wl.draft_tree(seed=2, batch=4, vocab=40, level_widths=(1, 2, 1))
    parents = base.parents.copy()
    tokens = base.node_tokens.copy()
    parents[1, 2] = 2      # not before itself
    tokens[3, 1] = 40      # token out of range
    t = base.target.copy()
    r = orc.verify_tree_exact(t, base.draft, tokens, parents, base.max_depth, 40, 1.0, 0, 0)
    o = orc.verify_tree(t, base.draft, tokens, parents, base.max_depth, 40, True, 1.0, 0, 0)
    assert np.array_equal(r["err"], o["err"]) and r["err"][1] & 2 and r["err"][3] & 1
    assert (r["out"][r["err"] != 0] == -1).all() and (r["acc"][r["err"] != 0] == -1).all()


# -------------------------------------------------------- distribution test
V, K1, K2 = 6, 3, 2   # vocabulary, children of the root, children of each child


def _tables(rng):
    """Target and draft logits as functions of the prefix (so that siblings
    with equal tokens see equal rows): root, after x, after (x, y)."""
    P0 = rng.normal(0, 1.5, V)
    Q0 = P0 + rng.normal(0, 1.0, V)
    P1 = rng.normal(0, 1.5, (V, V))
    Q1 = P1 + rng.normal(0, 1.0, (V, V))
    P2 = rng.normal(0, 1.5, (V, V, V))
    return P0, Q0, P1, Q1, P2


def _trials(rng, tabs, M):
    """M trees: the root's K1 children drawn i.i.d. from q_root, each
    child's K2 children i.i.d. from q_child; node rows from the tables."""
    P0, Q0, P1, Q1, P2 = tabs
    q0, q1 = softmax64(Q0, 1.0), softmax64(Q1, 1.0)
    N = 1 + K1 + K1 * K2
    tok = np.full((M, N), -1, np.int32)
    par = np.full((M, N), -1, np.int32)
    tok[:, 1:1 + K1] = rng.choice(V, size=(M, K1), p=q0)
    par[:, 1:1 + K1] = 0
    cdf1 = np.cumsum(q1, axis=1)
    for c in range(K1):
        x = tok[:, 1 + c]
        for g in range(K2):
            i = 1 + K1 + c * K2 + g
            u = rng.random(M)
            tok[:, i] = np.minimum((u[:, None] > cdf1[x]).sum(axis=1), V - 1)
            par[:, i] = 1 + c
    tl = np.zeros((M, N, V), np.float32)
    dl = np.zeros((M, N, V), np.float32)
    tl[:, 0], dl[:, 0] = P0, Q0
    for c in range(K1):
        x = tok[:, 1 + c]
        tl[:, 1 + c], dl[:, 1 + c] = P1[x], Q1[x]
        for g in range(K2):
            i = 1 + K1 + c * K2 + g
            tl[:, i] = P2[x, tok[:, i]]
    return tl, dl, tok, par


def _emitted_chi2(out, acc, tabs):
    """Pooled chi-square of slot 0 against p_root, slot 1 (given a kept
    first draft) against p(. | x), slot 2 against p(. | x, y)."""
    P0, _, P1, _, P2 = tabs
    groups = [(np.ones(len(acc), bool), softmax64(P0, 1.0), 0)]
    for x in range(V):
        groups.append(((acc >= 1) & (out[:, 0] == x), softmax64(P1[x], 1.0), 1))
        for y in range(V):
            groups.append(((acc >= 2) & (out[:, 0] == x) & (out[:, 1] == y),
                           softmax64(P2[x, y], 1.0), 2))
    stat, dof = 0.0, 0
    for mask, p, slot in groups:
        n = int(mask.sum())
        if n < 50:
            continue
        obs = np.bincount(out[mask, slot], minlength=V).astype(np.float64)
        exp = p * n
        big = exp >= 5
        o = list(obs[big]) + ([obs[~big].sum()] if (~big).any() else [])
        e = list(exp[big]) + ([exp[~big].sum()] if (~big).any() else [])
        if len(o) < 2:
            continue
        stat += float(((np.array(o) - np.array(e)) ** 2 / np.array(e)).sum())
        dof += len(o) - 1
    return float(stats.chi2.sf(stat, dof)), dof


def test_emitted_tokens_follow_the_target_distribution(orc):
    rng = np.random.default_rng(12345)
    tabs = _tables(rng)
    outs, accs, outs_ind, accs_ind = [], [], [], []
    for _ in range(5):  # 5 x 200k = 1e6 trials
        tl, dl, tok, par = _trials(rng, tabs, 200_000)
        M, N = tok.shape
        ua, us = rng.random((M, N)), rng.random((M, N))
        r = orc.verify_tree_exact_u(tl, dl, tok, par, 2, V, 1.0, ua, us)
        outs.append(r["out"])
        accs.append(r["acc"])
        o = orc.verify_tree_u(tl, dl, tok, par, 2, V, True, 1.0, ua, us)
        outs_ind.append(o["out"])
        accs_ind.append(o["acc"])
    out, acc = np.concatenate(outs), np.concatenate(accs)
    assert (acc >= 0).all()
    assert 0.2 < (acc >= 1).mean() < 0.95 and (acc == 2).mean() > 0.05  # every level is exercised
    pval, dof = _emitted_chi2(out, acc, tabs)
    assert dof > 50 and pval > 1e-3, (pval, dof)
    # control: testing every node independently and keeping the deepest
    # accepted one is biased, and the same test sees it
    pval_ind, _ = _emitted_chi2(np.concatenate(outs_ind), np.concatenate(accs_ind), tabs)
    assert pval_ind < 1e-6, pval_ind


# ------------------------------------------------- residual chain closed form
def _nested(p, q, r):
    """r literal residual steps: p <- norm(max(0, p - q))."""
    for _ in range(r):
        w = np.maximum(p - q, 0.0)
        p = w / w.sum()
    return p


def _collapsed(p, q, r):
    """The same as one threshold: norm(max(0, p - c q)) with c_1 = 1 and
    c_{i+1} = c_i + D_i, D_i = sum(max(0, p - c_i q))."""
    c = 1.0
    for _ in range(r - 1):
        c += np.maximum(p - c * q, 0.0).sum()
    w = np.maximum(p - c * q, 0.0)
    return w / w.sum(), c


def test_residual_chain_is_one_threshold():
    rng = np.random.default_rng(21)
    for _ in range(50):
        V = int(rng.integers(5, 80))
        p = softmax64(rng.normal(0, 2, V), 1.0)
        q = softmax64(rng.normal(0, 2, V), 1.0)
        for r in (1, 2, 3, 4):
            a = _nested(p, q, r)
            if not np.isfinite(a).all():  # the mass ran out (p <= c q everywhere)
                break
            b, _ = _collapsed(p, q, r)
            assert np.allclose(a, b, rtol=1e-10, atol=1e-14)


def test_oracle_draw_after_rejections_matches_the_closed_form(orc):
    # a root whose children all carry a token of zero residual mass are all
    # rejected whatever u; the final draw then comes from norm(max(0, p - c q))
    rng = np.random.default_rng(33)
    V, K = 40, 3
    P = rng.normal(0, 2, V)
    Q = P + rng.normal(0, 1.5, V)
    p, q = softmax64(P.astype(np.float32), 1.0), softmax64(Q.astype(np.float32), 1.0)
    dead = int(np.argmin(p - q))  # p < q here, so p - c q < 0 for every c >= 1
    assert p[dead] - q[dead] < 0
    M = 400
    tl = np.tile(P.astype(np.float32), (M, K + 1, 1))
    dl = np.tile(Q.astype(np.float32), (M, K + 1, 1))
    tok = np.full((M, K + 1), dead, np.int32)
    par = np.zeros((M, K + 1), np.int32)
    par[:, 0] = -1
    us = rng.random((M, K + 1))
    r = orc.verify_tree_exact_u(tl, dl, tok, par, 1, V, 1.0, np.full((M, K + 1), 0.5), us)
    assert (r["acc"] == 0).all()
    w, _ = _collapsed(p, q, K)  # K rejections: K residual steps
    want = np.searchsorted(np.cumsum(w), us[:, 0], side="right")
    assert np.array_equal(r["out"][:, 0], want)
