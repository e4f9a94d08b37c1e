"""GPU parity of the walking greedy calls (spec_verify_greedy_walk,
spec_verify_tree_greedy_walk) against the oracle: bit-exact outputs,
accepted lengths, paths and per-request error bits, on the greedy and tree
workloads at full size, ragged shapes, heavy ties, sibling nodes with equal
tokens (several kept nodes per level), a 1024-node chain kept to the end,
and malformed inputs."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_87_b200 import workloads as wl
from parity import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from speculative_decoding_verification_87_b200 import binding, build
    build.build()
    binding.load_library()
    return binding


def walk_linear(sv, target, tokens, vocab):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, acc = sv.spec_verify_greedy_walk(to_device(target), to_device(tokens.astype(np.int32)),
                                          vocab, status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy(), acc.cpu().numpy(), int(status.item())


def walk_tree(sv, target, tokens, parents, max_depth, vocab):
    B = target.shape[0]
    path = torch.empty((B, max_depth + 1), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, acc, path = sv.spec_verify_tree_greedy_walk(
        to_device(target), to_device(tokens.astype(np.int32)), to_device(parents.astype(np.int32)),
        max_depth, vocab, out_path_nodes=path, status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy(), acc.cpu().numpy(), path.cpu().numpy(), int(status.item())


def oracle_tree(orc, target, tokens, parents, max_depth, vocab):
    return orc.verify_tree(target, None, tokens, parents, max_depth, vocab, False, 1.0, 0, 0)


def random_tree(rng, B, N, max_depth, V, keep=0.7, values=3):
    """Random trees (parents[i] < i, depth <= max_depth) over integer-valued
    rows; a node's token is its parent's argmax with probability ``keep``,
    so siblings often share a token and several nodes per level are kept."""
    parents = np.full((B, N), -1, np.int32)
    depth = np.zeros((B, N), np.int64)
    for b in range(B):
        for i in range(1, N):
            while True:
                p = int(rng.integers(0, i))
                if depth[b, p] < max_depth:
                    break
            parents[b, i] = p
            depth[b, i] = depth[b, p] + 1
    target = rng.integers(0, values, size=(B, N, V)).astype(np.float32)
    am = np.argmax(target, axis=-1)
    tokens = np.zeros((B, N), np.int32)
    for b in range(B):
        for i in range(1, N):
            tokens[b, i] = am[b, parents[b, i]] if rng.random() < keep else int(rng.integers(V))
    return target, tokens, parents


def test_greedy_walk_full_size_bit_exact(sv, orc):
    w = wl.config_greedy(seed=0)
    out, acc, st = walk_linear(sv, w.target, w.tokens, w.vocab)
    o = orc.verify_greedy(w.target, w.tokens, w.vocab)
    assert st == 0
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
    assert len(set(acc.tolist())) >= 3
    # the same as the full greedy call
    t = to_device(w.target)
    x = to_device(w.tokens.astype(np.int32))
    out_f, acc_f = sv.spec_verify_greedy(t, x, w.vocab)
    assert np.array_equal(out_f.cpu().numpy(), out) and np.array_equal(acc_f.cpu().numpy(), acc)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("batch,k,vocab,pad", [(1, 4, 128256, 0), (3, 32, 1000, 5),
                                               (37, 2, 77, 3), (5, 1, 1, 0), (300, 3, 4100, 0),
                                               (700, 6, 515, 1)])
def test_greedy_walk_shapes_bit_exact(sv, orc, dtype, batch, k, vocab, pad):
    w = wl.greedy_linear(seed=batch + k, batch=batch, k=k, vocab=vocab, dtype=dtype, pad=pad)
    t = w.target.copy()
    if t.shape[-1] > vocab:  # padding past V is never read
        t[..., vocab:] = np.uint16(0x7FC0) if dtype == "bf16" else np.float32(np.nan)
    out, acc, st = walk_linear(sv, t, w.tokens, vocab)
    o = orc.verify_greedy(t, w.tokens, vocab)
    assert st == 0
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])


def test_greedy_walk_ties_long_chains_and_errors(sv, orc):
    rng = np.random.default_rng(3)
    B, k, V = 96, 32, 3000
    t = rng.integers(0, 3, size=(B, k + 1, V)).astype(np.float32)
    x = np.zeros((B, k), np.int32)
    for b in range(B):
        for j in range(k):  # most requests keep many drafts
            x[b, j] = int(np.argmax(t[b, j])) if rng.random() < 0.95 else int(rng.integers(V))
    out, acc, st = walk_linear(sv, t, x, V)
    clean = orc.verify_greedy(t, x, V)
    assert st == 0
    assert np.array_equal(out, clean["out"]) and np.array_equal(acc, clean["acc"])
    assert acc.max() == k

    # a NaN in a row the walk reads (row 0) and an out-of-range token
    t2 = t.copy()
    t2[3, 0, 17] = np.nan
    x2 = x.copy()
    x2[5, 0] = V
    out, acc, st = walk_linear(sv, t2, x2, V)
    o = orc.verify_greedy(t2, x2, V)
    assert st == (1 | 4)
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])

    # a NaN after the first mismatch is never read: the result is the one of
    # the clean input
    b = int(np.flatnonzero(clean["acc"] < k - 1)[0])
    n = int(clean["acc"][b])
    t3 = t.copy()
    t3[b, n + 1, 5] = np.nan
    out, acc, st = walk_linear(sv, t3, x, V)
    assert st == 0
    assert np.array_equal(out, clean["out"]) and np.array_equal(acc, clean["acc"])

    # a fully -inf row: argmax is index 0
    t4 = t.copy()
    t4[7, 0, :] = -np.inf
    out, acc, st = walk_linear(sv, t4, x, V)
    o = orc.verify_greedy(t4, x, V)
    assert st == 0 and np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])


def test_tree_walk_full_size_bit_exact(sv, orc):
    w = wl.config_tree(seed=0)
    out, acc, path, st = walk_tree(sv, w.target, w.node_tokens, w.parents, w.max_depth, w.vocab)
    o = oracle_tree(orc, w.target, w.node_tokens, w.parents, w.max_depth, w.vocab)
    assert st == 0
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
    assert np.array_equal(path, o["path"])
    # the same as the full tree call
    outf, accf, pathf = sv.spec_verify_tree(
        to_device(w.target), None, to_device(w.node_tokens), to_device(w.parents), w.max_depth,
        w.vocab, False, out_path_nodes=torch.empty_like(torch.from_numpy(path)).cuda())
    assert np.array_equal(outf.cpu().numpy(), out) and np.array_equal(pathf.cpu().numpy(), path)


@pytest.mark.parametrize("B,N,max_depth,V,dtype", [(5, 7, 3, 40, "f32"), (40, 60, 6, 300, "f32"),
                                                   (9, 200, 12, 1000, "bf16"),
                                                   (3, 1024, 30, 64, "f32"),
                                                   (70, 33, 32, 129, "bf16")])
def test_tree_walk_shared_sibling_tokens(sv, orc, B, N, max_depth, V, dtype):
    rng = np.random.default_rng(B * 1000 + N)
    t, tokens, parents = random_tree(rng, B, N, max_depth, V)
    if dtype == "bf16":  # small integers are exact in bf16
        t = wl._pack(t, "bf16", wl._stride_for(V, "bf16"))
    out, acc, path, st = walk_tree(sv, t, tokens, parents, max_depth, V)
    o = oracle_tree(orc, t, tokens, parents, max_depth, V)
    assert st == 0
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
    assert np.array_equal(path, o["path"])


def test_tree_walk_1024_node_chain_kept_to_the_end(sv, orc):
    B, N, V = 2, 1024, 36  # fp32 rows of 144 bytes (a multiple of 16)
    t = np.zeros((B, N, V), np.float32)
    t[:, :, 11] = 1.0
    parents = np.tile(np.arange(-1, N - 1, dtype=np.int32), (B, 1))
    tokens = np.full((B, N), 11, np.int32)
    tokens[1, 700] = 12  # request 1 stops at depth 699
    out, acc, path, st = walk_tree(sv, t, tokens, parents, N - 1, V)
    o = oracle_tree(orc, t, tokens, parents, N - 1, V)
    assert st == 0 and acc.tolist() == [N - 1, 699]
    assert np.array_equal(out, o["out"]) and np.array_equal(path, o["path"])


def test_chain_tree_walk_equals_linear_walk(sv):
    w = wl.greedy_linear(seed=11, batch=40, k=5, vocab=2000)
    out_l, acc_l, _ = walk_linear(sv, w.target, w.tokens, w.vocab)
    c = wl.chain_tree_from_linear(w)
    out_t, acc_t, path, st = walk_tree(sv, c.target, c.node_tokens, c.parents, c.max_depth, c.vocab)
    assert st == 0
    assert np.array_equal(out_l, out_t) and np.array_equal(acc_l, acc_t)


def test_tree_walk_errors(sv, orc):
    rng = np.random.default_rng(5)
    B, N, V = 8, 12, 8  # fp32 rows of 32 bytes
    t, tokens, _ = random_tree(rng, B, N, 4, V, keep=1.0)
    parents = np.tile(np.array([-1, 0, 0, 1, 1, 2, 3, 4, 5, 6, 7, 8], np.int32), (B, 1))
    am = np.argmax(t, axis=-1)
    for b in range(B):
        for i in range(1, N):
            tokens[b, i] = am[b, parents[b, i]]
    parents[1, 5] = 7          # not before itself
    parents[2, 0] = 0          # the root's parent must be -1
    tokens[3, 4] = V           # out of range
    t[4, 0, 2] = np.nan        # the root row is always read
    tokens[5, 1] = (am[5, 0] + 1) % V
    tokens[5, 2] = (am[5, 0] + 1) % V
    t[5, 5, 1] = np.nan        # row of node 5, a child of rejected node 2: never read
    out, acc, path, st = walk_tree(sv, t, tokens, parents, 4, V)
    clean = t.copy()
    clean[5, 5, 1] = 0.0
    o = oracle_tree(orc, clean, tokens, parents, 4, V)
    assert st == (1 | 2 | 4)
    assert acc.tolist()[:6] == [4, -1, -1, -1, -1, 0]
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
    assert np.array_equal(path, o["path"])
    assert np.array_equal(np.flatnonzero(acc < 0), np.flatnonzero(o["err"] != 0))
    # a node deeper than max_depth makes the tree malformed
    out, acc, path, st = walk_tree(sv, clean, tokens, parents, 3, V)
    o = oracle_tree(orc, clean, tokens, parents, 3, V)
    assert st & 2 and (acc == -1).all() and (out == -1).all()
    assert np.array_equal(out, o["out"]) and np.array_equal(acc, o["acc"])
