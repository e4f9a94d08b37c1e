"""The vocabulary-sharded verification kernels (spec_shard_*) on one GPU:
W ranks emulated by W host threads that share the device, each holding its
column range of the logits, exchanging through an in-process stand-in of the
collectives.  Outputs are compared with the oracle's single-rank
verification (greedy: identical; stochastic: identical except on trials
within the margins).  The same protocol runs over gloo on CPU in
test_sharded_cpu.py; on several GPUs it would run over NCCL (unmeasured)."""
import threading

import numpy as np
import pytest
import torch

from speculative_decoding_verification_87_b200 import workloads as wl
from parity import FlagTally, compare_linear, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from speculative_decoding_verification_87_b200 import binding, build
    build.build()
    binding.load_library()
    return binding


class ThreadComm:
    """All-gather and all-reduce among W threads of one process (the device
    work of every thread goes to the same stream, in order)."""

    def __init__(self, W):
        self.W = W
        self.slots = [None] * W
        self.bar = threading.Barrier(W, timeout=120)

    def bind(self, rank):
        comm = self

        class Bound:
            def all_gather(self, t):
                comm.slots[rank] = t
                comm.bar.wait()
                r = torch.stack(list(comm.slots))
                comm.bar.wait()
                return r

            def all_reduce_max(self, t):
                comm.slots[rank] = t
                comm.bar.wait()
                m = comm.slots[0].clone()
                for o in comm.slots[1:]:
                    m = torch.maximum(m, o)
                comm.bar.wait()
                t.copy_(m)
                return t

        return Bound()


def _cols(a, lo, hi, vec):
    """Columns [lo, hi) of every row, in a fresh array with a 16-byte pitch."""
    n = hi - lo
    stride = (n + vec - 1) // vec * vec
    out = np.zeros(a.shape[:-1] + (stride,), a.dtype)
    out[..., :n] = a[..., lo:hi]
    return to_device(out)


def _run_ranks(bounds, fn):
    W = len(bounds) - 1
    comm = ThreadComm(W)
    res, errs = [None] * W, []

    def body(r):
        try:
            res[r] = fn(r, comm.bind(r))
        except BaseException as e:  # noqa: BLE001 - reported below
            errs.append(e)
            comm.bar.abort()

    th = [threading.Thread(target=body, args=(r,)) for r in range(W)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    if errs:
        raise errs[0]
    torch.cuda.synchronize()
    return res


@pytest.mark.parametrize("bounds,dtype", [([0, 64128, 128256], "bf16"),
                                          ([0, 30000, 70000, 100000, 128256], "bf16"),
                                          ([0, 1001, 2003, 3000], "f32")])
def test_sharded_linear_matches_oracle(sv, orc, bounds, dtype):
    from speculative_decoding_verification_87_b200.sharded import ShardedVerifier
    V = bounds[-1]
    w = wl.peaked_linear(seed=V % 97, batch=16, k=6, vocab=V, temperature=0.7, sigma=(0.5, 2.0),
                         dtype=dtype)
    vec = 8 if dtype == "bf16" else 4
    x = to_device(w.tokens.astype(np.int32))
    tally = FlagTally()
    for off in range(4):
        def rank_fn(r, comm):
            lo, hi = bounds[r], bounds[r + 1]
            v = ShardedVerifier(bounds, r, comm=comm)
            out, acc = v.verify_linear(_cols(w.target, lo, hi, vec), _cols(w.draft, lo, hi, vec), x,
                                       w.temperature, seed=11, offset=off)
            return out.cpu().numpy(), acc.cpu().numpy()
        res = _run_ranks(bounds, rank_fn)
        for out, acc in res[1:]:
            assert np.array_equal(out, res[0][0]) and np.array_equal(acc, res[0][1])
        o = orc.verify_linear(w.target, w.draft, w.tokens, w.vocab, w.temperature, 11, off)
        tally.add(compare_linear(dict(out=res[0][0], acc=res[0][1]), o, w.k))
    print("sharded", bounds, tally.check())


def test_sharded_greedy_and_errors(sv, orc):
    from speculative_decoding_verification_87_b200.sharded import ShardedVerifier
    bounds = [0, 40000, 80000, 129280]
    g = wl.greedy_linear(seed=9, batch=32, k=4, vocab=129280, dtype="bf16")
    x = to_device(g.tokens.astype(np.int32))

    def rank_fn(r, comm):
        v = ShardedVerifier(bounds, r, comm=comm)
        out, acc = v.verify_greedy(_cols(g.target, bounds[r], bounds[r + 1], 8), x)
        return out.cpu().numpy(), acc.cpu().numpy()
    res = _run_ranks(bounds, rank_fn)
    og = orc.verify_greedy(g.target, g.tokens, g.vocab)
    for out, acc in res:
        assert np.array_equal(out, og["out"]) and np.array_equal(acc, og["acc"])
    # NaN in one rank's columns, a token out of range
    w = wl.peaked_linear(seed=4, batch=6, k=3, vocab=3000, temperature=1.0, dtype="f32")
    t = w.target.copy()
    t[1, 2, 2500] = np.nan
    xt = w.tokens.astype(np.int32).copy()
    xt[3, 0] = 3000
    b3 = [0, 1100, 3000]

    def rank_fn2(r, comm):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        v = ShardedVerifier(b3, r, comm=comm)
        out, acc = v.verify_linear(_cols(t, b3[r], b3[r + 1], 4), _cols(w.draft, b3[r], b3[r + 1], 4),
                                   to_device(xt), 1.0, seed=1, offset=0, status=st)
        return out.cpu().numpy(), acc.cpu().numpy(), int(st.item())
    res = _run_ranks(b3, rank_fn2)
    o = orc.verify_linear(t, w.draft, xt, 3000, 1.0, 1, 0)
    for out, acc, st in res:
        assert np.array_equal(acc, o["acc"]) and np.array_equal(out, o["out"])
        assert st == int(np.bitwise_or.reduce(o["err"]))
