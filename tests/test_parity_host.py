"""Host-side checks of the parity helpers (no GPU): the threaded oracle
calls equal one oracle call over the whole batch, the flag budget is strict,
and the log-probability rule treats -inf as a value that must match."""
import numpy as np
import pytest

from speculative_decoding_verification_87_b200 import workloads as wl
from parity import FlagTally, _check_logp, compare_linear, oracle_linear_many, oracle_tree_many


def _same(a, b):
    assert a.keys() == b.keys()
    for key in a:
        assert np.array_equal(a[key], b[key], equal_nan=True), key


def test_sliced_linear_oracle_equals_one_call(orc):
    w = wl.peaked_linear(seed=5, batch=11, k=3, vocab=700, temperature=0.8, sigma=(0.5, 2.0))
    many = oracle_linear_many(orc, w, 9, [0, 3], parts=4)
    for off, r in zip([0, 3], many):
        _same(r, orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 9, off))


def test_sliced_tree_oracle_equals_one_call(orc):
    w = wl.draft_tree(seed=3, batch=7, vocab=300, level_widths=(1, 3, 4, 2), topk=3)
    for stochastic in (False, True):
        (r,) = oracle_tree_many(orc, w, stochastic, 4, [2], parts=3)
        _same(r, orc.verify_tree(w.target, w.draft, w.node_tokens, w.parents, w.max_depth,
                                 w.vocab, stochastic, w.temperature, 4, 2))
    (r,) = oracle_tree_many(orc, w, True, 4, [2], exact=True, parts=3)
    _same(r, orc.verify_tree_exact(w.target, w.draft, w.node_tokens, w.parents, w.max_depth,
                                   w.vocab, w.temperature, 4, 2))


def test_flag_budget_has_no_slack():
    t = FlagTally()
    t.add(dict(trials=9999, flagged_trials=1))
    with pytest.raises(AssertionError):
        t.check()
    t.add(dict(trials=1, flagged_trials=0))
    t.check()  # 1 flagged of 10000 trials: exactly at the budget
    t.add(dict(unflagged_mismatch=1))
    with pytest.raises(AssertionError):
        t.check()


def test_log_prob_rule_treats_minus_inf_as_a_value():
    o = np.array([-1.0, -np.inf, -3.0])
    _check_logp(np.array([-1.0, -np.inf, -3.0 + 5e-6]), o, "ok")
    with pytest.raises(AssertionError):
        _check_logp(np.array([-1.0, -200.0, -3.0]), o, "finite where the oracle has -inf")
    with pytest.raises(AssertionError):
        _check_logp(np.array([-1.0, -np.inf, -np.inf]), o, "-inf where the oracle is finite")
    with pytest.raises(AssertionError):
        _check_logp(np.array([np.nan, -np.inf, -3.0]), o, "NaN")


def test_unflagged_mismatch_is_an_error(orc):
    w = wl.tiny_linear(seed=3, batch=8, k=3, vocab=16)
    o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 1, 0)
    g = dict(out=o["out"].copy(), acc=o["acc"].copy(), logp=o["logp"].astype(np.float32),
             logq=o["logq"].astype(np.float32))
    compare_linear(g, o, w.k)
    g["out"][0, 0] = (g["out"][0, 0] + 1) % 16
    with pytest.raises(AssertionError):
        compare_linear(g, o, w.k)
