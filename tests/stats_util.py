"""Statistical helpers shared by the oracle and GPU distribution tests."""
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
