"""Parity helpers: run a workload through the C ABI and through the oracle,
and compare them under the margin rules.

Rules (per request):
  * greedy and tree-greedy: outputs identical, element by element;
  * stochastic: accepted length and every emitted token identical, except
    on requests where one of the oracle's decisions that was actually taken
    has |u - p/q| < 1e-5, or the final draw lies within 1e-5 of a bucket
    edge relative to that bucket's width.  Such trials are counted; their
    share must stay under 1e-4 of all trials (decisions plus draws), and
    unflagged mismatches must be zero;
  * log p and log q of the drafts agree to 1e-5 (absolute in log space,
    i.e. 1e-5 relative in probability).
"""
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


def run_linear_gpu(binding, w, seed=None, offset=None, dbg=True):
    seed = w.seed if seed is None else seed
    offset = w.offset if offset is None else offset
    tl, dl = to_device(w.target), to_device(w.draft)
    x = to_device(w.tokens.astype(np.int32))
    B, k = w.batch, w.k
    lp = torch.full((B, k), float("nan"), device="cuda") if dbg else None
    lq = torch.full((B, k), float("nan"), device="cuda") if dbg else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, acc = binding.spec_verify_linear(tl, dl, x, w.vocab, w.temperature, seed, offset,
                                          dbg_logp=lp, dbg_logq=lq, status=status)
    torch.cuda.synchronize()
    r = dict(out=out.cpu().numpy(), acc=acc.cpu().numpy(), status=int(status.item()))
    if dbg:
        r["logp"] = lp.cpu().numpy()
        r["logq"] = lq.cpu().numpy()
    return r


def compare_linear(gpu, orc_res, k, check_logp=True):
    """Returns a dict of counts; raises AssertionError on a rule violation."""
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
    if trials:
        assert flagged_trials <= FLAG_BUDGET * trials + 2, res
    if check_logp and "logp" in gpu:
        m = ok_req
        dp = np.abs(gpu["logp"][m].astype(np.float64) - orc_res["logp"][m])
        dq = np.abs(gpu["logq"][m].astype(np.float64) - orc_res["logq"][m])
        fin = np.isfinite(orc_res["logp"][m])
        assert np.all(dp[fin] <= LOGP_TOL), float(dp[fin].max())
        finq = np.isfinite(orc_res["logq"][m])
        assert np.all(dq[finq] <= LOGP_TOL), float(dq[finq].max())
        res["max_dlogp"] = float(dp[fin].max()) if fin.any() else 0.0
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
               flagged_mismatch=int((mism & req_flag).sum()),
               unflagged_mismatch=int((mism & ~req_flag).sum()))
    assert res["unflagged_mismatch"] == 0, res
    assert res["flagged_trials"] <= FLAG_BUDGET * res["trials"] + 2, res
    return res
