"""Seeded synthetic inputs for the verification sampler.

This module draws logits, draft tokens and draft trees.  It holds none of the
verification arithmetic (no softmax normaliser, no accept test, no inverse
CDF): drafts are drawn by the Gumbel-max trick (argmax of logit/T plus
Gumbel noise, an exact sample of softmax(logit/T)), and greedy drafts are
the row argmax.  The same bytes feed the CUDA path and the fp64 oracle.

Recipes (numpy PCG64 streams, one per workload seed):
  * tiny:    fp32, target ~ N(0, 2^2) i.i.d., draft = target + N(0, 0.5^2).
  * peaked:  target ~ N(0, 3^2) with 20 random "peak" tokens per row raised
             by +8; draft = target + N(0, sigma_b^2) with sigma_b per
             request; both rounded to bf16 (round-to-nearest-even).
  * tree:    per-node target/draft rows from the peaked recipe; the tree is
             grown level by level by top-4 expansion of each frontier node's
             draft row, the candidates reranked by cumulative draft
             log-probability, keeping a fixed number per level.
Logits are returned as float32 arrays or as uint16 arrays of raw bf16 bits,
shaped [B][rows][stride] with stride >= vocab (pad columns hold -inf for
fp32 inputs and the bf16 pattern of -inf for bf16 inputs; they are never
read as vocabulary).
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

PEAKS_PER_ROW = 20
PEAK_LIFT = 8.0
BASE_SIGMA = 3.0


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> raw bf16 bits with round-to-nearest-even (torch's cast)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _stride_for(vocab: int, dtype: str, pad: int = 0) -> int:
    align = 8 if dtype == "bf16" else 4  # 16-byte rows
    s = vocab + pad
    return (s + align - 1) // align * align


def _pack(values: np.ndarray, dtype: str, stride: int) -> np.ndarray:
    """[..., V] float32 -> [..., stride] in the requested storage dtype."""
    V = values.shape[-1]
    shape = values.shape[:-1] + (stride,)
    if dtype == "f32":
        out = np.full(shape, -np.inf, dtype=np.float32)
        out[..., :V] = values
        return out
    out = np.full(shape, 0xFF80, dtype=np.uint16)  # bf16 -inf
    out[..., :V] = _bf16_bits(values)
    return out


def as_f32(logits: np.ndarray, vocab: int) -> np.ndarray:
    """Stored logits -> float32 values [..., vocab] (exact widening)."""
    if logits.dtype == np.uint16:
        return bf16_bits_to_f32(logits[..., :vocab])
    return logits[..., :vocab].astype(np.float32)


def gumbel_max(rng: np.random.Generator, logits: np.ndarray, temperature: float,
               chunk_rows: int = 1 << 14) -> np.ndarray:
    """One exact sample of softmax(logits/T) per row, by argmax(l/T + G)."""
    flat = logits.reshape(-1, logits.shape[-1])
    out = np.empty(flat.shape[0], dtype=np.int32)
    for s in range(0, flat.shape[0], chunk_rows):
        rows = flat[s:s + chunk_rows].astype(np.float64) / temperature
        g = -np.log(-np.log(rng.random(rows.shape)))
        out[s:s + chunk_rows] = np.argmax(rows + g, axis=1)
    return out.reshape(logits.shape[:-1])


@dataclass
class LinearWorkload:
    """Inputs of one linear verification call."""
    name: str
    target: np.ndarray            # [B][k+1][stride]
    draft: np.ndarray             # [B][k][stride]
    tokens: np.ndarray            # [B][k] int32
    vocab: int
    temperature: float
    dtype: str                    # "f32" or "bf16"
    seed: int = 0                 # Philox seed of the verify call
    offset: int = 0               # Philox offset of the verify call
    sigma: Optional[np.ndarray] = None

    @property
    def batch(self):
        return self.target.shape[0]

    @property
    def k(self):
        return self.target.shape[1] - 1

    @property
    def stride(self):
        return self.target.shape[2]


@dataclass
class TreeWorkload:
    name: str
    target: np.ndarray            # [B][N][stride]
    draft: np.ndarray             # [B][N][stride]
    node_tokens: np.ndarray       # [B][N] int32 (entry 0 = -1, the root)
    parents: np.ndarray           # [B][N] int32 (entry 0 = -1)
    max_depth: int
    vocab: int
    temperature: float
    dtype: str
    seed: int = 0
    offset: int = 0
    level_widths: tuple = field(default_factory=tuple)

    @property
    def batch(self):
        return self.target.shape[0]

    @property
    def num_nodes(self):
        return self.target.shape[1]

    @property
    def stride(self):
        return self.target.shape[2]


def _peaked_rows(rng, n_rows, vocab):
    base = rng.standard_normal((n_rows, vocab), dtype=np.float32) * np.float32(BASE_SIGMA)
    for r in range(n_rows):
        idx = rng.choice(vocab, size=min(PEAKS_PER_ROW, vocab), replace=False)
        base[r, idx] += np.float32(PEAK_LIFT)
    return base


def tiny_linear(seed=0, batch=4, k=4, vocab=32, temperature=1.0, pad=0) -> LinearWorkload:
    """fp32, target N(0, 2^2), draft = target + N(0, 0.5^2), drafts ~ q."""
    rng = np.random.default_rng([seed, 1])
    t = rng.standard_normal((batch, k + 1, vocab)).astype(np.float32) * np.float32(2.0)
    d = t[:, :k, :] + rng.standard_normal((batch, k, vocab)).astype(np.float32) * np.float32(0.5)
    stride = _stride_for(vocab, "f32", pad)
    x = gumbel_max(rng, d, temperature)
    return LinearWorkload("tiny", _pack(t, "f32", stride), _pack(d, "f32", stride),
                          x.astype(np.int32), vocab, temperature, "f32", seed, 0)


def peaked_linear(seed=0, batch=1, k=4, vocab=128256, temperature=1.0, sigma=(1.0, 1.0),
                  dtype="bf16", pad=0, name="peaked") -> LinearWorkload:
    """Peaked target rows; draft = target + N(0, sigma_b^2), sigma_b ~ U[sigma]."""
    rng = np.random.default_rng([seed, 2])
    sig = rng.uniform(sigma[0], sigma[1], size=batch).astype(np.float32)
    t = _peaked_rows(rng, batch * (k + 1), vocab).reshape(batch, k + 1, vocab)
    noise = rng.standard_normal((batch, k, vocab), dtype=np.float32) * sig[:, None, None]
    d = t[:, :k, :] + noise
    stride = _stride_for(vocab, dtype, pad)
    tp = _pack(t, dtype, stride)
    dp = _pack(d, dtype, stride)
    x = gumbel_max(rng, as_f32(dp, vocab), temperature)
    return LinearWorkload(name, tp, dp, x.astype(np.int32), vocab, temperature, dtype, seed, 0,
                          sig)


def greedy_linear(seed=0, batch=256, k=4, vocab=129280, dtype="bf16", pad=0) -> LinearWorkload:
    """Peaked rows; the draft emits its own top token (argmax of its row)."""
    rng = np.random.default_rng([seed, 3])
    t = _peaked_rows(rng, batch * (k + 1), vocab).reshape(batch, k + 1, vocab)
    d = t[:, :k, :] + rng.standard_normal((batch, k, vocab), dtype=np.float32)
    stride = _stride_for(vocab, dtype, pad)
    tp = _pack(t, dtype, stride)
    dp = _pack(d, dtype, stride)
    x = np.argmax(as_f32(dp, vocab), axis=-1).astype(np.int32)
    return LinearWorkload("greedy", tp, dp, x, vocab, 1.0, dtype, seed, 0)


EAGLE_LEVEL_WIDTHS = (1, 4, 16, 16, 12, 8, 3)


def draft_tree(seed=0, batch=32, vocab=128256, level_widths=EAGLE_LEVEL_WIDTHS, topk=4,
               temperature=1.0, dtype="bf16", pad=0) -> TreeWorkload:
    """Tree of drafts grown by top-``topk`` expansion of draft rows.

    Level 0 is the root.  Every node of level L is expanded into the top-k
    tokens of its draft row; the candidates are reranked by cumulative
    draft log-probability and the best ``level_widths[L+1]`` are kept.
    Nodes are numbered level by level (best first), so parents[i] < i.
    """
    rng = np.random.default_rng([seed, 5])
    N = int(sum(level_widths))
    D = len(level_widths) - 1
    t = _peaked_rows(rng, batch * N, vocab).reshape(batch, N, vocab)
    d = t + rng.standard_normal((batch, N, vocab), dtype=np.float32)
    stride = _stride_for(vocab, dtype, pad)
    tp = _pack(t, dtype, stride)
    dp = _pack(d, dtype, stride)
    dvals = torch.from_numpy(as_f32(dp, vocab))
    tokens = np.full((batch, N), -1, dtype=np.int32)
    parents = np.full((batch, N), -1, dtype=np.int32)
    for b in range(batch):
        frontier = [(0, 0.0)]  # (node, cumulative draft log-prob)
        next_id = 1
        for level in range(1, len(level_widths)):
            cands = []
            for node, score in frontier:
                lp = torch.log_softmax(dvals[b, node].double() / temperature, dim=0)
                top = torch.topk(lp, topk)
                for val, tok in zip(top.values.tolist(), top.indices.tolist()):
                    cands.append((score + val, node, tok))
            cands.sort(key=lambda c: (-c[0], c[1], c[2]))
            frontier = []
            for score, par, tok in cands[:level_widths[level]]:
                tokens[b, next_id] = tok
                parents[b, next_id] = par
                frontier.append((next_id, score))
                next_id += 1
    return TreeWorkload("tree", tp, dp, tokens, parents, D, vocab, temperature, dtype, seed, 0,
                        tuple(level_widths))


def chain_tree_from_linear(w: LinearWorkload) -> TreeWorkload:
    """A chain tree (parents[i] = i-1) with the same rows as a linear call:
    node i's target row is linear target row i, node i's draft row is linear
    draft row i (the leaf's draft row is unused), node i's token is draft
    i-1."""
    B, k = w.batch, w.k
    N = k + 1
    draft = np.concatenate([w.draft, w.draft[:, :1, :]], axis=1)
    tokens = np.full((B, N), -1, dtype=np.int32)
    tokens[:, 1:] = w.tokens
    parents = np.tile(np.arange(-1, N - 1, dtype=np.int32), (B, 1))
    return TreeWorkload("chain", w.target, np.ascontiguousarray(draft), tokens, parents, k,
                        w.vocab, w.temperature, w.dtype, w.seed, w.offset, tuple([1] * N))


def replicate_requests(w: LinearWorkload, copies: int, draft_rng_seed: int) -> LinearWorkload:
    """Repeat each request ``copies`` times (request-major) with fresh drafts
    drawn from the same draft rows: independent trials of the same logits."""
    rng = np.random.default_rng([draft_rng_seed, 7])
    t = np.repeat(w.target, copies, axis=0)
    d = np.repeat(w.draft, copies, axis=0)
    x = gumbel_max(rng, as_f32(d, w.vocab), w.temperature).astype(np.int32)
    return LinearWorkload(w.name + f"x{copies}", t, d, x, w.vocab, w.temperature, w.dtype,
                          w.seed, w.offset)


# The five workloads the sampler is measured and checked on.
def config_tiny(seed=0):
    return tiny_linear(seed=seed)


def config_single(seed=0):
    return peaked_linear(seed=seed, batch=1, k=4, vocab=128256, temperature=1.0,
                         sigma=(1.0, 1.0), name="single")


def config_batched(seed=0):
    return peaked_linear(seed=seed, batch=64, k=8, vocab=128256, temperature=0.7,
                         sigma=(0.5, 2.0), name="batched")


def config_greedy(seed=0):
    return greedy_linear(seed=seed, batch=256, k=4, vocab=129280)


def config_tree(seed=0, temperature=1.0):
    return draft_tree(seed=seed, batch=32, vocab=128256, temperature=temperature)
