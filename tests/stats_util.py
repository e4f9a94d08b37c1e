"""Statistical helpers shared by the oracle and GPU distribution tests."""
import itertools

import numpy as np
from scipy import stats


def chisquare_pvalue(observed, expected_prob, min_expected=5.0):
    """Pearson chi-square of observed counts against exact probabilities.

    Bins whose expected count is below ``min_expected`` are pooled into one
    bin.  Returns (p_value, impossible_hits) where impossible_hits counts
    observations that fell on zero-probability outcomes.
    """
    observed = np.asarray(observed, dtype=np.float64).ravel()
    p = np.asarray(expected_prob, dtype=np.float64).ravel()
    assert observed.shape == p.shape
    n = observed.sum()
    impossible = int(observed[p <= 0].sum())
    exp = p * n
    big = exp >= min_expected
    obs_b = list(observed[big])
    exp_b = list(exp[big])
    rest_o = observed[~big].sum()
    rest_e = exp[~big].sum()
    if rest_e > 0:
        obs_b.append(rest_o)
        exp_b.append(rest_e)
    obs_b = np.array(obs_b)
    exp_b = np.array(exp_b)
    if len(obs_b) < 2:
        return 1.0, impossible
    stat = float(((obs_b - exp_b) ** 2 / exp_b).sum())
    return float(stats.chi2.sf(stat, len(obs_b) - 1)), impossible


def softmax64(logits, temperature):
    """fp64 softmax used only to build exact expected distributions."""
    z = np.asarray(logits, dtype=np.float64) / temperature
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def brute_force_linear(p, q, k):
    """Exact distribution of (n, emitted tokens) by enumerating all drafts."""
    V = p.shape[-1]
    dist = {}
    for xs in itertools.product(range(V), repeat=k):
        wx = np.prod([q[j, xs[j]] for j in range(k)])
        if wx == 0:
            continue
        r = [min(1.0, p[j, xs[j]] / q[j, xs[j]]) for j in range(k)]
        reach = wx
        for m in range(k + 1):
            if m < k:
                pm = reach * (1 - r[m])
                res = np.maximum(p[m] - q[m], 0)
                res = res / res.sum() if res.sum() > 0 else p[m]
            else:
                pm = reach
                res = p[k]
            for y in range(V):
                if pm * res[y] > 0:
                    key = (m,) + tuple(xs[:m]) + (y,)
                    dist[key] = dist.get(key, 0.0) + pm * res[y]
            if m < k:
                reach *= r[m]
    return dist
