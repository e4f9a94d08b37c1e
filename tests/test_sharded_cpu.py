"""The multi-rank protocol of vocabulary-sharded verification on two gloo
ranks (CPU processes): every rank holds a column range of every logit row,
the ranks exchange statistics, masses and the drawn token, and both end
with the outputs of single-rank verification under the parity rules
(greedy: identical; stochastic: identical except on trials within the
margins).  The per-rank steps run in a CPU stand-in of the kernels
(tests/shard_ops_cpu.py); the kernels themselves are checked on a GPU in
test_gpu_sharded.py.  Unmeasured on multi-GPU hardware."""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CHILD = textwrap.dedent("""
    import datetime, os, sys
    sys.path.insert(0, {root!r}); sys.path.insert(0, os.path.join({root!r}, "tests"))
    import numpy as np, torch
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    rank = dist.get_rank()
    import oracle
    from speculative_decoding_verification_87_b200 import workloads as wl
    from speculative_decoding_verification_87_b200.sharded import ShardedVerifier, TorchComm
    from shard_ops_cpu import CpuShardOps
    from parity import FlagTally, compare_linear

    def cols(a, lo, hi):
        x = np.ascontiguousarray(a[..., lo:hi])
        t = torch.from_numpy(x)
        return t.view(torch.bfloat16) if x.dtype == np.uint16 else t

    def same_everywhere(t):
        parts = [torch.empty_like(t) for _ in range(2)]
        dist.all_gather(parts, t.contiguous())
        assert torch.equal(parts[0], parts[1])

    bounds = [0, 1100, 3000]
    lo, hi = bounds[rank], bounds[rank + 1]
    sv = ShardedVerifier(bounds, rank, comm=TorchComm(), ops=CpuShardOps())
    tally = FlagTally()
    for dtype in ("bf16", "f32"):
        w = wl.peaked_linear(seed=3, batch=12, k=4, vocab=3000, temperature=0.8, sigma=(0.5, 2.0),
                             dtype=dtype)
        x = torch.from_numpy(w.tokens.astype(np.int32))
        for off in range(3):
            out, acc = sv.verify_linear(cols(w.target, lo, hi), cols(w.draft, lo, hi), x,
                                        w.temperature, seed=7, offset=off)
            same_everywhere(out); same_everywhere(acc)
            o = oracle.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 7, off)
            tally.add(compare_linear(dict(out=out.numpy(), acc=acc.numpy()), o, w.k))
    tally.check()
    # a request with a NaN in one rank's columns and one with a bad token
    w = wl.peaked_linear(seed=4, batch=6, k=3, vocab=3000, temperature=1.0, dtype="f32")
    t = w.target.copy(); t[1, 2, 2500] = np.nan
    xt = w.tokens.astype(np.int32).copy(); xt[3, 0] = 3000
    st = torch.zeros(1, dtype=torch.int32)
    out, acc = sv.verify_linear(cols(t, lo, hi), cols(w.draft, lo, hi), torch.from_numpy(xt), 1.0,
                                seed=1, offset=0, status=st)
    o = oracle.verify_linear(t, w.draft, xt, 3000, 1.0, 1, 0)
    assert np.array_equal(acc.numpy(), o["acc"]) and np.array_equal(out.numpy(), o["out"])
    assert int(st.item()) == int(np.bitwise_or.reduce(o["err"]))
    # greedy
    g = wl.greedy_linear(seed=5, batch=16, k=4, vocab=3000, dtype="bf16")
    out, acc = sv.verify_greedy(cols(g.target, lo, hi), torch.from_numpy(g.tokens.astype(np.int32)))
    og = oracle.verify_greedy(g.target, g.tokens, g.vocab)
    assert np.array_equal(out.numpy(), og["out"]) and np.array_equal(acc.numpy(), og["acc"])
    dist.destroy_process_group()
    print("rank", rank, "ok", tally.tot)
""")


@pytest.mark.timeout(300)
def test_two_gloo_ranks_match_the_oracle():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    outs = []
    for pr in procs:
        try:
            out, _ = pr.communicate(timeout=240)
        except subprocess.TimeoutExpired:
            pr.kill()
            out, _ = pr.communicate()
        outs.append(out)
    for rank, (pr, out) in enumerate(zip(procs, outs)):
        assert pr.returncode == 0, out
        assert f"rank {rank} ok" in out, out
