"""Parity helpers: run a workload through the C ABI and through the oracle,
and compare them under the margin rules.

Rules (per request):
  * greedy and tree-greedy: outputs identical, element by element;
  * stochastic: accepted length and every emitted token identical, except
    on requests where one of the oracle's decisions that was actually taken
    has |u - p/q| < 1e-5, or the final draw lies within 1e-5 of a bucket
    edge relative to that bucket's width.  Such trials are counted; their
    share must stay under 1e-4 of all trials (decisions plus draws), and
    unflagged mismatches must be zero.  The share is a rate, so it is
    asserted over a test's whole sample (``FlagTally.check``), never with
    any slack;
  * log p and log q of the drafts agree to 1e-5 (absolute in log space,
    i.e. 1e-5 relative in probability), and a log probability the oracle
    finds to be -inf (a token of probability zero) is -inf on the GPU too.

The oracle is single-threaded C; ``oracle_map`` spreads independent oracle
calls (offsets, request slices) over the host's cores with threads (ctypes
releases the interpreter lock during a call, and the oracle keeps no global
state).
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

MARGIN = 1e-5
FLAG_BUDGET = 1e-4
LOGP_TOL = 1e-5


def to_device(arr: np.ndarray, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if arr.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.to(device)


# ------------------------------------------------------------ oracle pool
def oracle_threads():
    return max(1, min(32, os.cpu_count() or 1))


def oracle_map(fn, jobs):
    """[fn(*job) for job in jobs], run on the host's cores."""
    jobs = list(jobs)
    if len(jobs) <= 1:
        return [fn(*j) for j in jobs]
    with ThreadPoolExecutor(max_workers=oracle_threads()) as ex:
        return list(ex.map(lambda j: fn(*j), jobs))


def _slices(n, parts):
    parts = max(1, min(parts, n))
    edges = np.linspace(0, n, parts + 1).astype(int)
    return [slice(int(a), int(b)) for a, b in zip(edges[:-1], edges[1:]) if b > a]


def _concat(dicts):
    return {key: np.concatenate([d[key] for d in dicts], axis=0) for key in dicts[0]}


def oracle_linear_many(orc, w, seed, offsets, parts=None):
    """The oracle's linear verification of workload w at each offset, as a
    list of result dicts.  Requests are split into slices, each verified
    with the uniforms of its own request indices (so the slices together
    equal one call over the whole batch)."""
    offsets = list(offsets)
    B, k = w.batch, w.k
    parts = parts or max(1, oracle_threads() // max(1, len(offsets)) + 1)
    sl = _slices(B, parts)
    jobs = []
    for off in offsets:
        ua = orc.uniforms(seed, off, orc.ACCEPT, B, k)
        us = orc.uniforms(seed, off, orc.SAMPLE, B, k + 1)
        for s in sl:
            jobs.append((w.target[s], w.draft[s], w.tokens[s], ua[s], us[s]))
    res = oracle_map(lambda t, d, x, ua, us: orc.verify_linear_u(t, d, x, w.temperature, ua, us,
                                                                 vocab=w.vocab), jobs)
    n = len(sl)
    return [_concat(res[i * n:(i + 1) * n]) for i in range(len(offsets))]


def oracle_tree_many(orc, w, stochastic, seed, offsets, exact=False, parts=None):
    """The oracle's tree verification of workload w at each offset (the
    independent-test mode, or the distribution-exact mode when exact)."""
    offsets = list(offsets)
    B, N = w.batch, w.num_nodes
    parts = parts or max(1, oracle_threads() // max(1, len(offsets)) + 1)
    sl = _slices(B, parts)
    jobs = []
    for off in offsets:
        ua, us = orc.tree_uniforms(seed, off, B, N)
        for s in sl:
            jobs.append((w.target[s], w.draft[s], w.node_tokens[s], w.parents[s], ua[s], us[s]))

    def one(t, d, tk, pa, ua, us):
        if exact:
            return orc.verify_tree_exact_u(t, d, tk, pa, w.max_depth, w.vocab, w.temperature,
                                           ua, us)
        return orc.verify_tree_u(t, d, tk, pa, w.max_depth, w.vocab, stochastic, w.temperature,
                                 ua, us)

    res = oracle_map(one, jobs)
    n = len(sl)
    return [_concat(res[i * n:(i + 1) * n]) for i in range(len(offsets))]


# ------------------------------------------------------------ GPU runs
class LinearOnDevice:
    """A linear workload's inputs resident on the device; ``run`` verifies it
    at one (seed, offset) and returns the outputs as numpy arrays."""

    def __init__(self, binding, w):
        self.sv, self.w = binding, w
        self.tl, self.dl = to_device(w.target), to_device(w.draft)
        self.x = to_device(w.tokens.astype(np.int32))

    def run_many(self, seed, offsets, dbg=True):
        """One call per offset, outputs kept on the device until the end."""
        offsets = list(offsets)
        B, k, n = self.w.batch, self.w.k, len(offsets)
        out = torch.empty((n, B, k + 1), dtype=torch.int32, device="cuda")
        acc = torch.empty((n, B), dtype=torch.int32, device="cuda")
        lp = torch.full((n, B, k), float("nan"), device="cuda") if dbg else None
        lq = torch.full((n, B, k), float("nan"), device="cuda") if dbg else None
        status = torch.zeros(n, dtype=torch.int32, device="cuda")
        for i, off in enumerate(offsets):
            self.sv.spec_verify_linear(self.tl, self.dl, self.x, self.w.vocab, self.w.temperature,
                                       seed, off, out_tokens=out[i], accepted_len=acc[i],
                                       dbg_logp=lp[i] if dbg else None,
                                       dbg_logq=lq[i] if dbg else None, status=status[i:i + 1])
        torch.cuda.synchronize()
        out, acc, status = out.cpu().numpy(), acc.cpu().numpy(), status.cpu().numpy()
        res = []
        for i in range(n):
            r = dict(out=out[i], acc=acc[i], status=int(status[i]))
            if dbg:
                r["logp"] = lp[i].cpu().numpy()
                r["logq"] = lq[i].cpu().numpy()
            res.append(r)
        return res

    def run(self, seed, offset, dbg=True):
        return self.run_many(seed, [offset], dbg)[0]


class TreeOnDevice:
    """A tree workload's inputs resident on the device; ``run_many`` verifies
    it at each offset (outputs read back once, at the end)."""

    def __init__(self, binding, w):
        self.sv, self.w = binding, w
        self.tl, self.dl = to_device(w.target), to_device(w.draft)
        self.tk = to_device(w.node_tokens.astype(np.int32))
        self.pa = to_device(w.parents.astype(np.int32))

    def run_many(self, stochastic, seed, offsets):
        offsets = list(offsets)
        B, W, n = self.w.batch, self.w.max_depth + 1, len(offsets)
        out = torch.empty((n, B, W), dtype=torch.int32, device="cuda")
        acc = torch.empty((n, B), dtype=torch.int32, device="cuda")
        path = torch.empty((n, B, W), dtype=torch.int32, device="cuda")
        status = torch.zeros(n, dtype=torch.int32, device="cuda")
        for i, off in enumerate(offsets):
            self.sv.spec_verify_tree(self.tl, self.dl if stochastic else None, self.tk, self.pa,
                                     self.w.max_depth, self.w.vocab, stochastic,
                                     self.w.temperature, seed, off, out_tokens=out[i],
                                     accepted_len=acc[i], out_path_nodes=path[i],
                                     status=status[i:i + 1])
        torch.cuda.synchronize()
        out, acc, path, status = (out.cpu().numpy(), acc.cpu().numpy(), path.cpu().numpy(),
                                  status.cpu().numpy())
        return [dict(out=out[i], acc=acc[i], path=path[i], status=int(status[i]))
                for i in range(n)]


def run_linear_gpu(binding, w, seed=None, offset=None, dbg=True):
    seed = w.seed if seed is None else seed
    offset = w.offset if offset is None else offset
    return LinearOnDevice(binding, w).run(seed, offset, dbg)


# ------------------------------------------------------------ comparisons
class FlagTally:
    """Trials, flagged trials and mismatches summed over a test's calls."""

    KEYS = ("requests", "trials", "flagged_trials", "accept_flags", "sample_flags",
            "flagged_mismatch", "unflagged_mismatch")

    def __init__(self):
        self.tot = {key: 0 for key in self.KEYS}

    def add(self, res):
        for key in self.KEYS:
            self.tot[key] += int(res.get(key, 0))
        return res

    def check(self, min_trials=0):
        """The budget over the whole sample, strictly: flagged trials at most
        1e-4 of all trials (with fewer than 1e4 trials that means none)."""
        t = self.tot
        assert t["unflagged_mismatch"] == 0, t
        assert t["trials"] >= min_trials, t
        assert t["flagged_trials"] <= FLAG_BUDGET * t["trials"], t
        return t


def _check_logp(gpu_lp, orc_lp, what):
    """|gpu - oracle| <= LOGP_TOL where the oracle's log p is finite; -inf
    exactly where the oracle's is -inf."""
    g = np.asarray(gpu_lp, dtype=np.float64)
    o = np.asarray(orc_lp, dtype=np.float64)
    zero = np.isneginf(o)
    assert np.all(np.isneginf(g[zero])), (what, g[zero][~np.isneginf(g[zero])][:5])
    fin = np.isfinite(o)
    if not fin.any():
        return 0.0
    d = np.abs(g[fin] - o[fin])
    assert np.all(d <= LOGP_TOL), (what, float(np.nanmax(d)) if np.isfinite(d).any() else d[:5])
    return float(d.max())


def compare_linear(gpu, orc_res, k, check_logp=True):
    """Returns a dict of counts; raises AssertionError on an unflagged
    mismatch or a log-probability violation.  The flag budget is a rate:
    callers sum the counts with FlagTally and check the whole sample."""
    acc_o = orc_res["acc"]
    B = acc_o.shape[0]
    ok_req = orc_res["err"] == 0
    # decisions actually taken by the oracle: j <= n (all k when n == k)
    j = np.arange(k)[None, :]
    taken = (j <= acc_o[:, None]) & ok_req[:, None]
    dec_flag = taken & (orc_res["acc_margin"] < MARGIN)
    smp_flag = ok_req & (orc_res["smp_margin"] < MARGIN)
    req_flag = dec_flag.any(axis=1) | smp_flag
    trials = int(taken.sum() + ok_req.sum())
    flagged_trials = int(dec_flag.sum() + smp_flag.sum())
    same = (gpu["acc"] == acc_o) & np.all(gpu["out"] == orc_res["out"], axis=1)
    mism = ~same
    unflagged = mism & ~req_flag
    res = dict(requests=B, trials=trials, flagged_trials=flagged_trials,
               flagged_mismatch=int((mism & req_flag).sum()), unflagged_mismatch=int(unflagged.sum()),
               accept_flags=int(dec_flag.sum()), sample_flags=int(smp_flag.sum()))
    if unflagged.any():
        bad = np.nonzero(unflagged)[0][:5]
        detail = [(int(b), gpu["acc"][b], acc_o[b], gpu["out"][b].tolist(),
                   orc_res["out"][b].tolist()) for b in bad]
        raise AssertionError(f"unflagged mismatches {res}: {detail}")
    if check_logp and "logp" in gpu:
        m = ok_req
        res["max_dlogp"] = max(_check_logp(gpu["logp"][m], orc_res["logp"][m], "log p"),
                               _check_logp(gpu["logq"][m], orc_res["logq"][m], "log q"))
    return res


def compare_tree_stochastic(gpu_out, gpu_acc, gpu_path, orc_res):
    """Same rules for trees.  Both sides evaluate the test of every node
    (N-1 decisions) and one final draw per request, so a request has N
    trials; it is flagged when any of them lies within the margin."""
    B, N = orc_res["acc_margin"].shape
    ok_req = orc_res["err"] == 0
    dec_flag = (orc_res["acc_margin"][:, 1:] < MARGIN) & ok_req[:, None]
    smp_flag = (orc_res["smp_margin"] < MARGIN) & ok_req
    req_flag = dec_flag.any(axis=1) | smp_flag
    same = (gpu_acc == orc_res["acc"]) & np.all(gpu_out == orc_res["out"], axis=1)
    if gpu_path is not None:
        same &= np.all(gpu_path == orc_res["path"], axis=1)
    mism = ~same
    res = dict(requests=B, trials=int(ok_req.sum()) * N,
               flagged_trials=int(dec_flag.sum() + smp_flag.sum()),
               accept_flags=int(dec_flag.sum()), sample_flags=int(smp_flag.sum()),
               flagged_mismatch=int((mism & req_flag).sum()),
               unflagged_mismatch=int((mism & ~req_flag).sum()))
    assert res["unflagged_mismatch"] == 0, res
    return res


def compare_tree_exact(gpu_out, gpu_acc, gpu_path, orc_res):
    """The rules for the distribution-exact tree mode: a request's trials
    are the children the oracle actually tested (finite margin) and its one
    draw; the request is flagged when any of them lies within the margin."""
    ok_req = orc_res["err"] == 0
    m = orc_res["acc_margin"][:, 1:]
    tested = np.isfinite(m) & ok_req[:, None]
    dec_flag = tested & (m < MARGIN)
    smp_flag = (orc_res["smp_margin"] < MARGIN) & ok_req
    req_flag = dec_flag.any(axis=1) | smp_flag
    same = (gpu_acc == orc_res["acc"]) & np.all(gpu_out == orc_res["out"], axis=1)
    if gpu_path is not None:
        same &= np.all(gpu_path == orc_res["path"], axis=1)
    mism = ~same
    res = dict(requests=len(ok_req), trials=int(tested.sum() + ok_req.sum()),
               flagged_trials=int(dec_flag.sum() + smp_flag.sum()),
               accept_flags=int(dec_flag.sum()), sample_flags=int(smp_flag.sum()),
               flagged_mismatch=int((mism & req_flag).sum()),
               unflagged_mismatch=int((mism & ~req_flag).sum()))
    if res["unflagged_mismatch"]:
        bad = np.nonzero(mism & ~req_flag)[0][:5]
        detail = [(int(b), int(gpu_acc[b]), int(orc_res["acc"][b]), gpu_out[b].tolist(),
                   orc_res["out"][b].tolist()) for b in bad]
        raise AssertionError(f"unflagged mismatches {res}: {detail}")
    return res
