"""GPU parity of the distribution-exact tree mode (spec_verify_tree with
stochastic = 2) with the oracle's orc_verify_tree_exact_u, through the C
ABI: small trees in both dtypes with ragged vocabularies, chain trees (equal
to the linear mode), input errors, the tree workload at full size, and a
chi-square of the GPU's own outputs against the target distribution on
trees whose children are independent draws from the draft rows ("Speculative
decoding explained", section "Draft and verification loop": the output keeps
the target's distribution)."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_87_b200 import workloads as wl
from parity import (FlagTally, TreeOnDevice, compare_linear, compare_tree_exact, oracle_tree_many,
                    run_linear_gpu)

pytestmark = pytest.mark.gpu
EXACT = 2


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from speculative_decoding_verification_87_b200 import binding, build
    build.build()
    binding.load_library()
    return binding


def _check(sv, orc, w, seed, offsets, min_trials=0):
    gpu = TreeOnDevice(sv, w).run_many(EXACT, seed, offsets)
    orcs = oracle_tree_many(orc, w, True, seed, offsets, exact=True)
    tally = FlagTally()
    for g, o in zip(gpu, orcs):
        assert g["status"] == int(np.bitwise_or.reduce(o["err"])), (g["status"], o["err"])
        tally.add(compare_tree_exact(g["out"], g["acc"], g["path"], o))
    return tally.check(min_trials=min_trials), gpu


@pytest.mark.parametrize("dtype,pad", [("f32", 3), ("bf16", 0), ("bf16", 8)])
def test_small_trees(sv, orc, dtype, pad):
    for seed in range(3):
        w = wl.draft_tree(seed=seed, batch=24, vocab=777 + 40 * seed, level_widths=(1, 3, 4, 2),
                          topk=3, dtype=dtype, pad=pad)
        t, gpu = _check(sv, orc, w, seed, range(6))
    print("small trees", dtype, t)


def test_chain_tree_equals_linear(sv, orc):
    w = wl.peaked_linear(seed=8, batch=48, k=6, vocab=3000, temperature=0.9, sigma=(0.5, 2.0))
    c = wl.chain_tree_from_linear(w)
    _check(sv, orc, c, 4, range(3))
    tally = FlagTally()
    gpu = TreeOnDevice(sv, c).run_many(EXACT, 4, range(3))
    for off, g in enumerate(gpu):
        lin = run_linear_gpu(sv, w, seed=4, offset=off, dbg=False)
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 4, off)
        tally.add(compare_linear(lin, o, w.k, check_logp=False))
        flagged = (o["smp_margin"] < 1e-5) | (o["acc_margin"] < 1e-5).any(axis=1)
        same = (g["acc"] == lin["acc"]) & np.all(g["out"][:, :w.k + 1] == lin["out"], axis=1)
        assert np.all(same | flagged)
    tally.check()


def test_errors_match_the_oracle(sv, orc):
    base = wl.draft_tree(seed=2, batch=6, vocab=40, level_widths=(1, 2, 1), dtype="f32")
    parents = base.parents.copy()
    tokens = base.node_tokens.copy()
    target = base.target.copy()
    parents[1, 2] = 2       # not before itself
    parents[2, 0] = 0       # root parent must be -1
    tokens[3, 1] = 40       # token out of range
    target[4, 1, 5] = np.nan
    w = wl.TreeWorkload("bad", target, base.draft, tokens, parents, base.max_depth, 40, 1.0, "f32")
    gpu = TreeOnDevice(sv, w).run_many(EXACT, 0, [0])[0]
    o = orc.verify_tree_exact(w.target, w.draft, tokens, parents, w.max_depth, 40, 1.0, 0, 0)
    assert gpu["status"] == int(np.bitwise_or.reduce(o["err"])) == 1 | 2 | 4
    assert np.array_equal(gpu["acc"], o["acc"]) and np.array_equal(gpu["out"], o["out"])
    assert np.array_equal(gpu["path"], o["path"])
    assert np.all(gpu["acc"][1:5] == -1) and gpu["acc"][0] >= 0 and gpu["acc"][5] >= 0


def test_tree_workload_full_size(sv, orc):
    """B=32, N=60, depth 6, V=128256 bf16, T=1 at 60 offsets."""
    w = wl.config_tree(seed=0)
    t, gpu = _check(sv, orc, w, 5, range(60), min_trials=3000)
    depths = np.concatenate([g["acc"] for g in gpu])
    print("exact tree full size", t, "mean depth", depths.mean())


def test_emitted_tokens_follow_the_target_distribution(sv, orc):
    """1e6 trees (depth 2, children i.i.d. from the draft rows): the GPU's
    own outputs pass the chi-square of the oracle's test, and equal the
    oracle's outputs under the margin rules."""
    from test_oracle_tree_exact import V, _emitted_chi2, _tables, _trials
    rng = np.random.default_rng(12345)
    tabs = _tables(rng)
    outs, accs = [], []
    tally = FlagTally()
    for c in range(5):
        tl, dl, tok, par = _trials(rng, tabs, 200_000)
        pad = np.zeros(tl.shape[:2] + (8 - V,), np.float32)   # 32-byte rows
        tl = np.ascontiguousarray(np.concatenate([tl, pad], axis=2))
        dl = np.ascontiguousarray(np.concatenate([dl, pad], axis=2))
        w = wl.TreeWorkload("iid", tl, dl, tok, par, 2, V, 1.0, "f32")
        (g,) = TreeOnDevice(sv, w).run_many(EXACT, 77, [c])
        (o,) = oracle_tree_many(orc, w, True, 77, [c], exact=True)
        assert g["status"] == 0
        tally.add(compare_tree_exact(g["out"], g["acc"], g["path"], o))
        outs.append(g["out"])
        accs.append(g["acc"])
    print("iid trees", tally.check(min_trials=1_000_000))
    out, acc = np.concatenate(outs), np.concatenate(accs)
    pval, dof = _emitted_chi2(out, acc, tabs)
    assert dof > 50 and pval > 1e-3, (pval, dof)
