"""fp64 CPU oracle of the speculative-decoding verification sampler.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports this package.  The arithmetic lives in ``specverify_oracle.c``
(plain single-threaded fp64 C); this module only marshals numpy arrays.

Sources: Leviathan, Kalman & Matias, "Fast inference from transformers via
speculative decoding" (accept with min(1, p/q), resample from
norm(max(0, p-q))); "Accelerating Sonar through speculation" (sections
"Speculative decoding", "Target-Draft", "EAGLE"); "Speculative decoding
explained" (section "Draft and verification loop"); Salmon et al., SC'11
(Philox4x32-10).

Logit arrays: ``float32`` arrays (dtype code 0) or ``uint16`` arrays holding
raw bf16 bits (dtype code 1), shaped ``[B][rows][stride]``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

ACCEPT, SAMPLE, DRAFT = 0, 1, 2
ERR_TOKEN, ERR_TREE, ERR_LOGIT, ERR_CAPACITY = 1, 2, 4, 16

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_D = ctypes.c_double
_U32 = ctypes.c_uint32
_U64 = ctypes.c_uint64


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_philox4x32_10.argtypes = [_P, _P, _P]
        L.orc_philox4x32_10.restype = None
        L.orc_uniform.argtypes = [_U64, _U32, _U32, _U32, _U32]
        L.orc_uniform.restype = _D
        L.orc_fill_uniforms.argtypes = [_U64, _U32, _U32, _I, _I, _I, _P]
        L.orc_fill_uniforms.restype = None
        L.orc_verify_linear_u.argtypes = [_P, _P, _I, _I64, _P, _I, _I, _I, _D, _P, _P,
                                          _P, _P, _P, _P, _P, _P, _P]
        L.orc_verify_linear_u.restype = _I
        L.orc_verify_greedy.argtypes = [_P, _I, _I64, _P, _I, _I, _I, _P, _P, _P]
        L.orc_verify_greedy.restype = _I
        L.orc_verify_tree_u.argtypes = [_P, _P, _I, _I64, _P, _P, _I, _I, _I, _I, _I, _D,
                                        _P, _P, _P, _P, _P, _P, _P, _P]
        L.orc_verify_tree_u.restype = _I
        L.orc_verify_tree_exact_u.argtypes = [_P, _P, _I, _I64, _P, _P, _I, _I, _I, _I, _D,
                                              _P, _P, _P, _P, _P, _P, _P, _P]
        L.orc_verify_tree_exact_u.restype = _I
        L.orc_log_softmax_row.argtypes = [_P, _I, _I, _D, _P]
        L.orc_log_softmax_row.restype = _I
        L.orc_plug_tokens.argtypes = [_P, _P, _P, _I, _I, _P, _P, _P, _I]
        L.orc_plug_tokens.restype = _I
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _logits(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, 0
    if a.dtype == np.uint16:
        return a, 1
    raise TypeError("logits must be float32 or uint16 (raw bf16 bits)")


def philox4x32_10(counter, key):
    """Raw Philox4x32-10 block: 4 counter words, 2 key words -> 4 words."""
    c = np.ascontiguousarray(np.asarray(counter, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    o = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(o))
    return o


def uniform(seed, request, position, purpose, offset):
    return lib().orc_uniform(seed, request, position, purpose, offset)


def uniforms(seed, offset, purpose, batch, count, first_position=0):
    """[batch][count] array of U(seed, b, first_position + i, purpose, offset)."""
    out = np.zeros((batch, count), dtype=np.float64)
    if batch > 0 and count > 0:
        lib().orc_fill_uniforms(seed, offset, purpose, batch, count, first_position, _ptr(out))
    return out


def verify_linear_u(target, draft, tokens, temperature, u_accept, u_sample, vocab=None):
    """Linear stochastic verification with explicit uniforms.

    target [B][k+1][stride], draft [B][k][stride], tokens [B][k] int32,
    u_accept [B][k], u_sample [B][k+1].  Returns a dict of numpy arrays.
    """
    t, dt = _logits(target)
    d, dd = _logits(draft)
    assert dt == dd
    B, R, stride = t.shape
    k = R - 1
    assert d.shape == (B, k, stride)
    x = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, k)
    ua = np.ascontiguousarray(u_accept, dtype=np.float64).reshape(B, k)
    us = np.ascontiguousarray(u_sample, dtype=np.float64).reshape(B, k + 1)
    return _run_linear(t, d, dt, stride, x, B, k, temperature, ua, us, vocab)


def _run_linear(t, d, dt, stride, x, B, k, temperature, ua, us, vocab=None):
    V = stride if vocab is None else vocab
    r = dict(out=np.zeros((B, k + 1), np.int32), acc=np.zeros(B, np.int32),
             logp=np.zeros((B, k)), logq=np.zeros((B, k)), acc_margin=np.zeros((B, k)),
             smp_margin=np.zeros(B), err=np.zeros(B, np.int32))
    rc = lib().orc_verify_linear_u(_ptr(t), _ptr(d), dt, stride, _ptr(x), B, k, V,
                                   float(temperature), _ptr(ua), _ptr(us), _ptr(r["out"]),
                                   _ptr(r["acc"]), _ptr(r["logp"]), _ptr(r["logq"]),
                                   _ptr(r["acc_margin"]), _ptr(r["smp_margin"]), _ptr(r["err"]))
    if rc != 0:
        raise ValueError(f"oracle verify_linear rejected its arguments ({rc})")
    return r


def verify_linear(target, draft, tokens, vocab, temperature, seed, offset):
    """Linear stochastic verification; uniforms from Philox (seed, b, j, purpose, offset)."""
    t, dt = _logits(target)
    d, dd = _logits(draft)
    assert dt == dd
    B, R, stride = t.shape
    k = R - 1
    x = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, k)
    ua = uniforms(seed, offset, ACCEPT, B, k)
    us = uniforms(seed, offset, SAMPLE, B, k + 1)
    return _run_linear(t, d, dt, stride, x, B, k, temperature, ua, us, vocab)


def verify_greedy(target, tokens, vocab):
    t, dt = _logits(target)
    B, R, stride = t.shape
    k = R - 1
    x = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, k)
    r = dict(out=np.zeros((B, k + 1), np.int32), acc=np.zeros(B, np.int32),
             err=np.zeros(B, np.int32))
    rc = lib().orc_verify_greedy(_ptr(t), dt, stride, _ptr(x), B, k, vocab, _ptr(r["out"]),
                                 _ptr(r["acc"]), _ptr(r["err"]))
    if rc != 0:
        raise ValueError(f"oracle verify_greedy rejected its arguments ({rc})")
    return r


def verify_tree_u(target, draft, node_tokens, parents, max_depth, vocab, stochastic,
                  temperature, u_accept, u_sample):
    t, dt = _logits(target)
    B, N, stride = t.shape
    if draft is None:
        d, dd = t, dt
    else:
        d, dd = _logits(draft)
        assert dd == dt and d.shape == t.shape
    tk = np.ascontiguousarray(node_tokens, dtype=np.int32).reshape(B, N)
    pa = np.ascontiguousarray(parents, dtype=np.int32).reshape(B, N)
    ua = np.ascontiguousarray(u_accept, dtype=np.float64).reshape(B, N)
    us = np.ascontiguousarray(u_sample, dtype=np.float64).reshape(B, N)
    W = max_depth + 1
    r = dict(out=np.zeros((B, W), np.int32), acc=np.zeros(B, np.int32),
             path=np.zeros((B, W), np.int32), acc_margin=np.zeros((B, N)),
             smp_margin=np.zeros(B), err=np.zeros(B, np.int32))
    rc = lib().orc_verify_tree_u(_ptr(t), _ptr(d), dt, stride, _ptr(tk), _ptr(pa), B, N,
                                 max_depth, vocab, int(bool(stochastic)), float(temperature),
                                 _ptr(ua), _ptr(us), _ptr(r["out"]), _ptr(r["acc"]),
                                 _ptr(r["path"]), _ptr(r["acc_margin"]), _ptr(r["smp_margin"]),
                                 _ptr(r["err"]))
    if rc != 0:
        raise ValueError(f"oracle verify_tree rejected its arguments ({rc})")
    return r


def tree_uniforms(seed, offset, batch, num_nodes):
    """Uniforms of the tree test: node i >= 1 uses position i-1 (its draft
    index, so a chain tree draws exactly the linear mode's numbers); the
    bonus at node d uses position d."""
    ua = np.zeros((batch, num_nodes))
    if num_nodes > 1:
        ua[:, 1:] = uniforms(seed, offset, ACCEPT, batch, num_nodes - 1, 0)
    us = uniforms(seed, offset, SAMPLE, batch, num_nodes, 0)
    return ua, us


def verify_tree(target, draft, node_tokens, parents, max_depth, vocab, stochastic,
                temperature, seed, offset):
    B, N = np.asarray(target).shape[:2]
    ua, us = tree_uniforms(seed, offset, B, N)
    return verify_tree_u(target, draft, node_tokens, parents, max_depth, vocab, stochastic,
                         temperature, ua, us)


def verify_tree_exact_u(target, draft, node_tokens, parents, max_depth, vocab, temperature,
                        u_accept, u_sample):
    """Distribution-exact tree verification (recursive rejection over
    siblings) with given uniforms: u_accept [B][N] (entry c tests node c),
    u_sample [B][N] (entry d draws at node d).  Same outputs as
    verify_tree_u."""
    t, dt = _logits(target)
    d, dd = _logits(draft)
    assert dd == dt and d.shape == t.shape
    B, N, stride = t.shape
    tk = np.ascontiguousarray(node_tokens, dtype=np.int32).reshape(B, N)
    pa = np.ascontiguousarray(parents, dtype=np.int32).reshape(B, N)
    ua = np.ascontiguousarray(u_accept, dtype=np.float64).reshape(B, N)
    us = np.ascontiguousarray(u_sample, dtype=np.float64).reshape(B, N)
    W = max_depth + 1
    r = dict(out=np.zeros((B, W), np.int32), acc=np.zeros(B, np.int32),
             path=np.zeros((B, W), np.int32), acc_margin=np.zeros((B, N)),
             smp_margin=np.zeros(B), err=np.zeros(B, np.int32))
    rc = lib().orc_verify_tree_exact_u(_ptr(t), _ptr(d), dt, stride, _ptr(tk), _ptr(pa), B, N,
                                       max_depth, vocab, float(temperature), _ptr(ua), _ptr(us),
                                       _ptr(r["out"]), _ptr(r["acc"]), _ptr(r["path"]),
                                       _ptr(r["acc_margin"]), _ptr(r["smp_margin"]),
                                       _ptr(r["err"]))
    if rc != 0:
        raise ValueError(f"oracle verify_tree_exact rejected its arguments ({rc})")
    return r


def verify_tree_exact(target, draft, node_tokens, parents, max_depth, vocab, temperature, seed,
                      offset):
    B, N = np.asarray(target).shape[:2]
    ua, us = tree_uniforms(seed, offset, B, N)
    return verify_tree_exact_u(target, draft, node_tokens, parents, max_depth, vocab,
                               temperature, ua, us)


def log_softmax_row(row, temperature):
    r, dt = _logits(np.asarray(row).reshape(-1))
    out = np.zeros(r.shape[0])
    rc = lib().orc_log_softmax_row(_ptr(r), dt, r.shape[0], float(temperature), _ptr(out))
    if rc != 0:
        raise ValueError("row has no finite normaliser")
    return out


def plug_tokens(in_tokens, out_tokens, accepted_len, seq_tokens=None, seq_len=None,
                want_next=True):
    """Device-side token plug of the next step's inputs (see the C source).
    in_tokens, out_tokens [B][k+1]; accepted_len [B]; seq_tokens [B][cap]
    and seq_len [B] are copied, updated and returned.  Returns a dict with
    next [B][k+1] (or None), seq, len and the error bits."""
    a = np.ascontiguousarray(in_tokens, dtype=np.int32)
    B, W = a.shape
    k = W - 1
    o = np.ascontiguousarray(out_tokens, dtype=np.int32).reshape(B, W)
    n = np.ascontiguousarray(accepted_len, dtype=np.int32).reshape(B)
    nxt = np.zeros((B, W), np.int32) if want_next else None
    seq = None if seq_tokens is None else np.array(seq_tokens, dtype=np.int32, copy=True)
    ln = None if seq_len is None else np.array(seq_len, dtype=np.int32, copy=True).reshape(B)
    cap = 0 if seq is None else seq.shape[1]
    bits = lib().orc_plug_tokens(_ptr(a), _ptr(o), _ptr(n), B, k, _ptr(nxt), _ptr(seq), _ptr(ln),
                                 cap)
    return dict(next=nxt, seq=seq, len=ln, err=int(bits))
