"""GPU parity of spec_verify_greedy and spec_verify_tree against the oracle."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_87_b200 import workloads as wl
from parity import FlagTally, TreeOnDevice, compare_tree_stochastic, oracle_tree_many, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from speculative_decoding_verification_87_b200 import binding, build
    build.build()
    binding.load_library()
    return binding


# the two forms of spec_verify_greedy: streamed (workspace) and cluster (none)
FORMS = pytest.mark.parametrize("workspace_free", [False, True], ids=["streamed", "cluster"])


def run_greedy(sv, target, tokens, vocab, workspace_free=False):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, acc = sv.spec_verify_greedy(to_device(target), to_device(tokens.astype(np.int32)), vocab,
                                     status=status, workspace_free=workspace_free)
    torch.cuda.synchronize()
    return out.cpu().numpy(), acc.cpu().numpy(), int(status.item())


def run_tree(sv, w, stochastic, seed=0, offset=0, target=None, draft=None):
    target = w.target if target is None else target
    draft = w.draft if draft is None else draft
    B, N = w.batch, w.num_nodes
    path = torch.empty((B, w.max_depth + 1), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, acc, path = sv.spec_verify_tree(
        to_device(target), to_device(draft) if stochastic else None,
        to_device(w.node_tokens), to_device(w.parents), w.max_depth, w.vocab, stochastic,
        w.temperature, seed, offset, out_path_nodes=path, status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy(), acc.cpu().numpy(), path.cpu().numpy(), int(status.item())


@FORMS
def test_greedy_full_size_bit_exact(sv, orc, workspace_free):
    w = wl.config_greedy(seed=0)
    out, acc, st = run_greedy(sv, w.target, w.tokens, w.vocab, workspace_free)
    o = orc.verify_greedy(w.target, w.tokens, w.vocab)
    assert st == 0
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
    assert len(set(acc.tolist())) >= 3


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("batch,k,vocab,pad", [(1, 4, 128256, 0), (3, 32, 1000, 5),
                                               (37, 2, 77, 3), (5, 1, 1, 0), (300, 3, 4100, 0)])
@FORMS
def test_greedy_shapes_bit_exact(sv, orc, dtype, batch, k, vocab, pad, workspace_free):
    w = wl.greedy_linear(seed=batch + k, batch=batch, k=k, vocab=vocab, dtype=dtype, pad=pad)
    t = w.target.copy()
    if t.shape[-1] > vocab:
        t[..., vocab:] = np.uint16(0x7FC0) if dtype == "bf16" else np.float32(np.nan)
    out, acc, st = run_greedy(sv, t, w.tokens, vocab, workspace_free)
    o = orc.verify_greedy(t, w.tokens, vocab)
    assert st == 0
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])


@FORMS
def test_greedy_ties_and_errors(sv, orc, workspace_free):
    # heavy ties: logits drawn from 3 values, argmax ties resolved to the lowest index
    rng = np.random.default_rng(0)
    B, k, V = 64, 4, 3000
    t = rng.integers(0, 3, size=(B, k + 1, V)).astype(np.float32)
    x = np.zeros((B, k), np.int32)
    for b in range(B):
        for j in range(k):
            x[b, j] = int(np.argmax(t[b, j])) if rng.random() < 0.8 else int(rng.integers(V))
    out, acc, st = run_greedy(sv, t, x, V, workspace_free)
    o = orc.verify_greedy(t, x, V)
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
    # NaN logits and bad tokens
    t2 = t.copy()
    t2[3, 2, 17] = np.nan
    x2 = x.copy()
    x2[5, 0] = V
    out, acc, st = run_greedy(sv, t2, x2, V, workspace_free)
    o = orc.verify_greedy(t2, x2, V)
    assert st == (1 | 4)
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
    # a fully -inf row: argmax is index 0
    t3 = t.copy()
    t3[7, 0, :] = -np.inf
    out, acc, st = run_greedy(sv, t3, x, V, workspace_free)
    o = orc.verify_greedy(t3, x, V)
    assert st == 0 and np.array_equal(out, o["out"])


def test_tree_greedy_full_size_bit_exact(sv, orc):
    w = wl.config_tree(seed=0)
    out, acc, path, st = run_tree(sv, w, False)
    o = orc.verify_tree(w.target, None, w.node_tokens, w.parents, w.max_depth, w.vocab, False,
                        1.0, 0, 0)
    assert st == 0
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
    assert np.array_equal(path, o["path"])


def test_tree_stochastic_full_size(sv, orc):
    """B=32, N=60, depth 6, V=128256 bf16, T=1 at 200 offsets: 6400
    requests of 60 trials each (59 node tests and one draw)."""
    w = wl.config_tree(seed=0)
    offsets = range(200)
    gpu = TreeOnDevice(sv, w).run_many(True, 5, offsets)
    orcs = oracle_tree_many(orc, w, True, 5, offsets)
    tally = FlagTally()
    depths = []
    for g, o in zip(gpu, orcs):
        assert g["status"] == 0
        tally.add(compare_tree_stochastic(g["out"], g["acc"], g["path"], o))
        depths.extend(g["acc"].tolist())
    print("tree stochastic", tally.check(min_trials=100_000), "mean depth", np.mean(depths))


def test_chain_tree_equals_linear_greedy_on_gpu(sv):
    w = wl.greedy_linear(seed=11, batch=40, k=5, vocab=2000)
    out_l, acc_l, _ = run_greedy(sv, w.target, w.tokens, w.vocab)
    c = wl.chain_tree_from_linear(w)
    out_t, acc_t, path, st = run_tree(sv, c, False)
    assert st == 0
    assert np.array_equal(out_l, out_t) and np.array_equal(acc_l, acc_t)


def test_chain_tree_stochastic_accept_length_equals_linear(sv, orc):
    from parity import run_linear_gpu
    w = wl.peaked_linear(seed=8, batch=48, k=6, vocab=3000, temperature=0.9, sigma=(0.5, 2.0))
    c = wl.chain_tree_from_linear(w)
    for off in range(3):
        g = run_linear_gpu(sv, w, seed=4, offset=off, dbg=False)
        out_t, acc_t, path, st = run_tree(sv, c, True, seed=4, offset=off)
        assert np.array_equal(g["acc"], acc_t)


def test_tree_errors(sv, orc):
    V, N = 40, 4
    base = wl.draft_tree(seed=2, batch=4, vocab=V, level_widths=(1, 2, 1))
    parents = base.parents.copy()
    tokens = base.node_tokens.copy()
    parents[1, 2] = 2      # not before itself
    parents[2, 0] = 0      # root parent must be -1
    tokens[3, 1] = V       # token out of range
    w = wl.TreeWorkload("bad", base.target, base.draft, tokens, parents, base.max_depth, V, 1.0,
                        base.dtype)
    for stochastic in (False, True):
        out, acc, path, st = run_tree(sv, w, stochastic)
        o = orc.verify_tree(w.target, w.draft, tokens, parents, w.max_depth, V, stochastic, 1.0,
                            0, 0)
        assert st & 2 and st & 1
        assert np.array_equal(acc, o["acc"]) and np.array_equal(out, o["out"])
        assert np.array_equal(path, o["path"])
        assert acc[0] >= 0 and np.all(acc[1:] == -1)


def test_small_trees_both_modes(sv, orc):
    tally = FlagTally()
    for seed in range(4):
        w = wl.draft_tree(seed=seed, batch=16, vocab=777, level_widths=(1, 3, 4, 2), topk=3,
                          dtype="f32", pad=3)
        for stochastic in (False, True):
            out, acc, path, st = run_tree(sv, w, stochastic, seed=seed, offset=1)
            o = orc.verify_tree(w.target, w.draft, w.node_tokens, w.parents, w.max_depth,
                                w.vocab, stochastic, 1.0, seed, 1)
            assert st == 0
            if stochastic:
                tally.add(compare_tree_stochastic(out, acc, path, o))
            else:
                assert np.array_equal(out, o["out"]) and np.array_equal(path, o["path"])
    tally.check()
