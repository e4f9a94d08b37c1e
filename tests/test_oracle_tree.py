"""Pins of the oracle's tree verification ("Accelerating Sonar through
speculation", section "EAGLE": longest acceptable root-to-node sequence plus
one target token).

Pins: a chain tree equals the linear modes (greedy bit-exact; stochastic
same accepted length with aligned keys), hand-built trees with known
argmaxes, brute-force enumeration of all test outcomes on a 7-node tree,
and structural error cases.
"""
import itertools

import numpy as np
import pytest

from speculative_decoding_verification_87_b200 import workloads as wl
from stats_util import chisquare_pvalue, softmax64


def test_chain_tree_greedy_equals_linear_greedy(orc):
    w = wl.greedy_linear(seed=1, batch=64, k=5, vocab=500)
    g = orc.verify_greedy(w.target, w.tokens, w.vocab)
    c = wl.chain_tree_from_linear(w)
    t = orc.verify_tree(c.target, None, c.node_tokens, c.parents, c.max_depth, c.vocab,
                        False, 1.0, 0, 0)
    assert np.array_equal(g["out"], t["out"])
    assert np.array_equal(g["acc"], t["acc"])
    for b in range(w.batch):
        n = t["acc"][b]
        assert list(t["path"][b, :n + 1]) == list(range(n + 1))
    assert len(set(g["acc"].tolist())) > 2  # several accept lengths exercised


def test_chain_tree_stochastic_matches_linear_accept_length(orc):
    w = wl.peaked_linear(seed=3, batch=64, k=6, vocab=700, temperature=0.9, sigma=(0.5, 2.0))
    c = wl.chain_tree_from_linear(w)
    for off in range(5):
        lin = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, 0.9, seed=4, offset=off)
        tr = orc.verify_tree(c.target, c.draft, c.node_tokens, c.parents, c.max_depth,
                             c.vocab, True, 0.9, 4, off)
        assert np.array_equal(lin["acc"], tr["acc"])
        full = lin["acc"] == w.k
        # all drafts accepted: the bonus is drawn from row k with the same number
        assert np.array_equal(lin["out"][full], tr["out"][full])
        part = ~full
        for b in np.nonzero(part)[0]:
            n = lin["acc"][b]
            assert np.array_equal(lin["out"][b, :n], tr["out"][b, :n])


def _tree_rows(V, rows):
    return np.ascontiguousarray(np.array(rows, dtype=np.float32))[None]


def test_hand_tree_greedy_deepest_lowest_index(orc):
    # V=5.  Tree (node: parent, token):
    #   0 root; 1:(0,2) 2:(0,3) 3:(1,4) 4:(2,1) 5:(2,0) 6:(4,3)
    # argmax of target rows: row0 -> 2 (tie of 2 and 3 -> lowest), row1 -> 4,
    # row2 -> 1, row3 -> 0, row4 -> 3, row5 -> 4, row6 -> 2
    rows = [[0, 1, 5, 5, 0],   # node 0: argmax 2
            [0, 0, 0, 0, 9],   # node 1: argmax 4
            [3, 4, 0, 0, 0],   # node 2: argmax 1
            [1, 0, 0, 0, 0],   # node 3: argmax 0
            [0, 0, 0, 8, 0],   # node 4: argmax 3
            [0, 0, 0, 0, 1],   # node 5: argmax 4
            [0, 0, 6, 0, 0]]   # node 6: argmax 2
    parents = np.array([[-1, 0, 0, 1, 2, 2, 4]], np.int32)
    tokens = np.array([[-1, 2, 3, 4, 1, 0, 3]], np.int32)
    # node1 ok (2 == argmax row0); node2 fails (3 != 2); node3 ok (4 == argmax row1);
    # nodes 4,5,6 sit under rejected node 2.  Deepest accepted: node 3 (depth 2).
    t = orc.verify_tree(_tree_rows(5, rows), None, tokens, parents, 3, 5, False, 1.0, 0, 0)
    assert t["err"][0] == 0
    assert t["acc"][0] == 2
    assert list(t["out"][0]) == [2, 4, 0, -1]   # path tokens 2,4 then argmax row3 = 0
    assert list(t["path"][0]) == [0, 1, 3, -1]
    # make node 2 accepted too: node 4 (token 1 == argmax row2) and node 6
    # (token 3 == argmax row4) are accepted: depth 3 beats depth 2
    tokens2 = tokens.copy()
    tokens2[0, 2] = 2
    t2 = orc.verify_tree(_tree_rows(5, rows), None, tokens2, parents, 3, 5, False, 1.0, 0, 0)
    assert t2["acc"][0] == 3
    assert list(t2["path"][0]) == [0, 2, 4, 6]
    assert list(t2["out"][0]) == [2, 1, 3, 2]
    # tie on depth: drop node 6 (token mismatch) -> nodes 3 (depth 2) and 4 (depth 2)
    # both accepted; the lower index, node 3, wins
    tokens3 = tokens2.copy()
    tokens3[0, 6] = 0
    t3 = orc.verify_tree(_tree_rows(5, rows), None, tokens3, parents, 3, 5, False, 1.0, 0, 0)
    assert t3["acc"][0] == 2
    assert list(t3["path"][0]) == [0, 1, 3, -1]


def test_tree_structure_errors(orc):
    V, N = 6, 4
    t = np.zeros((4, N, V), np.float32)
    parents = np.array([[-1, 0, 1, 2],    # chain of depth 3 > max_depth 2
                        [-1, 0, 2, 0],    # parent not before child
                        [0, 0, 0, 0],     # root parent not -1
                        [-1, 0, 0, 1]], np.int32)
    tokens = np.array([[-1, 0, 0, 0], [-1, 0, 0, 0], [-1, 0, 0, 0], [-1, 0, 9, 0]], np.int32)
    r = orc.verify_tree(t, None, tokens, parents, 2, V, False, 1.0, 0, 0)
    assert r["err"][0] & orc.ERR_TREE
    assert r["err"][1] & orc.ERR_TREE
    assert r["err"][2] & orc.ERR_TREE
    assert r["err"][3] & orc.ERR_TOKEN
    assert np.all(r["out"] == -1) and np.all(r["acc"] == -1) and np.all(r["path"] == -1)


def _brute_force_tree(p, q, tokens, parents):
    """Exact distribution of (d, bonus) by enumerating every outcome of the
    independent per-node tests (Bernoulli(min(1, p_par(t)/q_par(t))))."""
    N, V = p.shape
    depth = [0] * N
    for i in range(1, N):
        depth[i] = depth[parents[i]] + 1
    r = [1.0] * N
    for i in range(1, N):
        par, t = parents[i], tokens[i]
        r[i] = 1.0 if q[par, t] == 0 else min(1.0, p[par, t] / q[par, t])
    dist = {}
    for bits in itertools.product((0, 1), repeat=N - 1):
        test = (1,) + bits
        w = np.prod([r[i] if test[i] else 1 - r[i] for i in range(1, N)])
        if w == 0:
            continue
        acc = [True] + [False] * (N - 1)
        for i in range(1, N):
            acc[i] = acc[parents[i]] and bool(test[i])
        d = max((i for i in range(N) if acc[i]), key=lambda i: (depth[i], -i))
        for y in range(V):
            dist[(d, y)] = dist.get((d, y), 0.0) + w * p[d, y]
    return dist


@pytest.mark.slow
def test_brute_force_tree_stochastic(orc):
    V, T = 6, 1.0
    rng = np.random.default_rng(5)
    parents = np.array([-1, 0, 0, 1, 1, 2, 3], np.int32)
    N = len(parents)
    tl = rng.normal(0, 1.5, (N, V)).astype(np.float32)
    dl = (tl + rng.normal(0, 1.0, (N, V))).astype(np.float32)
    tokens = np.array([-1, 1, 2, 0, 3, 5, 4], np.int32)
    p = softmax64(tl, T)
    q = softmax64(dl, T)
    dist = _brute_force_tree(p, q, tokens, parents)
    keys = sorted(dist)
    index = {key: i for i, key in enumerate(keys)}
    counts = np.zeros(len(keys))
    trials = 100_000
    chunk = 25_000
    for c in range(trials // chunk):
        B = chunk
        r = orc.verify_tree(np.ascontiguousarray(np.broadcast_to(tl, (B, N, V))),
                            np.ascontiguousarray(np.broadcast_to(dl, (B, N, V))),
                            np.tile(tokens, (B, 1)), np.tile(parents, (B, 1)), 3, V, True, T,
                            seed=13, offset=c)
        assert np.all(r["err"] == 0)
        for b in range(B):
            D = r["acc"][b]
            key = (int(r["path"][b, D]), int(r["out"][b, D]))
            counts[index[key]] += 1
    pv, bad = chisquare_pvalue(counts, [dist[key] for key in keys])
    assert pv > 1e-3, pv


def test_generated_eagle_tree_shape():
    w = wl.draft_tree(seed=0, batch=2, vocab=2000)
    assert w.num_nodes == 60 and w.max_depth == 6
    for b in range(w.batch):
        pa = w.parents[b]
        assert pa[0] == -1 and all(0 <= pa[i] < i for i in range(1, 60))
        depth = [0] * 60
        for i in range(1, 60):
            depth[i] = depth[pa[i]] + 1
        assert [depth.count(L) for L in range(7)] == list(wl.EAGLE_LEVEL_WIDTHS)
        assert np.all((w.node_tokens[b, 1:] >= 0) & (w.node_tokens[b, 1:] < w.vocab))


def test_tree_invariants_on_generated_tree(orc):
    w = wl.draft_tree(seed=1, batch=4, vocab=3000)
    for stochastic in (False, True):
        r = orc.verify_tree(w.target, w.draft, w.node_tokens, w.parents, w.max_depth,
                            w.vocab, stochastic, 1.0, seed=2, offset=0)
        assert np.all(r["err"] == 0)
        for b in range(w.batch):
            D = r["acc"][b]
            path = r["path"][b]
            assert path[0] == 0
            for j in range(1, D + 1):
                assert w.parents[b, path[j]] == path[j - 1]
                assert r["out"][b, j - 1] == w.node_tokens[b, path[j]]
            assert np.all(path[D + 1:] == -1) and np.all(r["out"][b, D + 1:] == -1)
