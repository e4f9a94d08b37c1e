"""ctypes binding of libspecverify.so: argument marshalling only.

Each function takes torch CUDA tensors, checks their shapes and dtypes,
passes raw device pointers and the current CUDA stream to the C ABI of the
same name (declared in include/specverify.h) and returns the output
tensors.  Every step of the computation runs in the library's kernels; there
is no fallback.  If the library has not been built, the first call raises.

Build it with ``python -m speculative_decoding_verification_87_b200.build``.
"""
import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspecverify.so")

SPEC_F32, SPEC_BF16 = 0, 1
SPEC_OK = 0
STATUS_TOKEN, STATUS_TREE, STATUS_LOGIT, STATUS_TIMEOUT, STATUS_CAPACITY = 1, 2, 4, 8, 16
MAX_K, MAX_NODES = 32, 1024
SYMBOLS = ("spec_verify_workspace_size", "spec_verify_strerror", "spec_verify_linear",
           "spec_verify_greedy", "spec_verify_tree", "spec_verify_debug_uniforms",
           "spec_verify_linear_noalloc", "spec_verify_debug_exp2", "spec_verify_greedy_walk",
           "spec_verify_tree_greedy_walk", "spec_verify_debug_wait_expiry", "spec_plug_tokens",
           "spec_shard_row_stats", "spec_shard_decide", "spec_shard_decide_greedy",
           "spec_shard_draw_sums", "spec_shard_draw_pick", "spec_shard_emit")
NOALLOC_SCRATCH_BYTES = 8 << 20

_lib = None
_lock = threading.Lock()
_ws_cache = {}

_P, _I, _I64, _U32, _U64, _F, _SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                     ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float,
                                     ctypes.c_size_t)


class SpecVerifyError(RuntimeError):
    pass


def load_library(path: str = LIB_PATH):
    """Load libspecverify.so and declare its C signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise SpecVerifyError(
                f"{path} is missing: build it with "
                "`python -m speculative_decoding_verification_87_b200.build`")
        L = ctypes.CDLL(path)
        L.spec_verify_workspace_size.argtypes = [_I, _I, _I]
        L.spec_verify_workspace_size.restype = _SZ
        L.spec_verify_strerror.argtypes = [_I]
        L.spec_verify_strerror.restype = ctypes.c_char_p
        L.spec_verify_linear.argtypes = [_P, _P, _I, _I64, _P, _I, _I, _I, _F, _U64, _U32, _P, _P,
                                         _P, _P, _P, _P, _SZ, _P]
        L.spec_verify_linear.restype = _I
        L.spec_verify_greedy.argtypes = [_P, _I, _I64, _P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]
        L.spec_verify_greedy.restype = _I
        L.spec_verify_tree.argtypes = [_P, _P, _I, _I64, _P, _P, _I, _I, _I, _I, _I, _F, _U64,
                                       _U32, _P, _P, _P, _P, _P, _SZ, _P]
        L.spec_verify_tree.restype = _I
        L.spec_verify_debug_uniforms.argtypes = [_U64, _U32, _U32, _I, _I, _I, _P, _P]
        L.spec_verify_debug_uniforms.restype = _I
        L.spec_verify_linear_noalloc.argtypes = [_P, _P, _I, _I64, _P, _I, _I, _I, _F, _U64, _U32,
                                                 _P, _P, _P, _P, _P, _P]
        L.spec_verify_linear_noalloc.restype = _I
        L.spec_verify_greedy_walk.argtypes = [_P, _I, _I64, _P, _I, _I, _I, _P, _P, _P, _P]
        L.spec_verify_greedy_walk.restype = _I
        L.spec_verify_tree_greedy_walk.argtypes = [_P, _I, _I64, _P, _P, _I, _I, _I, _I, _P, _P,
                                                   _P, _P, _P]
        L.spec_verify_tree_greedy_walk.restype = _I
        L.spec_verify_debug_exp2.argtypes = [_P, _P, _I, _I, _P]
        L.spec_verify_debug_exp2.restype = _I
        L.spec_verify_debug_wait_expiry.argtypes = [_P, _P, _I, _I64, _P, _I, _I, _I, _F, _U32,
                                                    _P, _P, _P, _P, _SZ, _P]
        L.spec_verify_debug_wait_expiry.restype = _I
        L.spec_plug_tokens.argtypes = [_P, _P, _P, _I, _I, _P, _P, _P, _I, _P, _P]
        L.spec_plug_tokens.restype = _I
        L.spec_shard_row_stats.argtypes = [_P, _P, _I, _I64, _P, _I, _I, _I, _I, _F, _P, _P, _P, _P,
                                           _P]
        L.spec_shard_row_stats.restype = _I
        L.spec_shard_decide.argtypes = [_P, _P, _P, _P, _I, _P, _I, _I, _I, _F, _U64, _U32, _P, _P,
                                        _P, _P, _P]
        L.spec_shard_decide.restype = _I
        L.spec_shard_decide_greedy.argtypes = [_P, _P, _I, _P, _I, _I, _I, _P, _P, _P, _P]
        L.spec_shard_decide_greedy.restype = _I
        L.spec_shard_draw_sums.argtypes = [_P, _P, _I, _I64, _I, _I, _I, _I, _F, _P, _P, _I, _P, _P]
        L.spec_shard_draw_sums.restype = _I
        L.spec_shard_draw_pick.argtypes = [_P, _P, _I, _I64, _I, _I, _I, _I, _F, _P, _P, _P, _I, _I,
                                           _P, _P]
        L.spec_shard_draw_pick.restype = _I
        L.spec_shard_emit.argtypes = [_P, _P, _I, _I, _P, _P]
        L.spec_shard_emit.restype = _I
        _lib = L
        return L


def _check(rc: int, what: str):
    if rc != SPEC_OK:
        msg = load_library().spec_verify_strerror(rc).decode()
        raise SpecVerifyError(f"{what} failed ({rc}): {msg}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SPEC_BF16
    if t.dtype == torch.float32:
        return SPEC_F32
    raise TypeError(f"logits must be bfloat16 or float32, got {t.dtype}")


def _need_cuda(name, t, dtype=None, shape=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def workspace_size(batch: int, rows_per_req: int, vocab: int) -> int:
    return int(load_library().spec_verify_workspace_size(batch, rows_per_req, vocab))


def workspace(batch: int, rows_per_req: int, vocab: int, device=None) -> torch.Tensor:
    """A cached uint8 device buffer large enough for the call (256-byte aligned)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    need = workspace_size(batch, rows_per_req, vocab)
    if need == 0:
        raise ValueError("invalid workspace request")
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.empty(need + 256, dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    off = (-buf.data_ptr()) % 256
    return buf[off:off + need]


def spec_verify_linear(target_logits, draft_logits, draft_tokens, vocab, temperature, seed=0,
                       offset=0, out_tokens=None, accepted_len=None, dbg_logp=None,
                       dbg_logq=None, status=None, workspace_buf=None, stream=None):
    """target_logits [B][k+1][stride], draft_logits [B][k][stride] (bf16/fp32),
    draft_tokens [B][k] int32.  Returns (out_tokens [B][k+1], accepted_len [B])."""
    _need_cuda("target_logits", target_logits)
    B, R, stride = target_logits.shape
    k = R - 1
    _need_cuda("draft_logits", draft_logits, target_logits.dtype, (B, k, stride))
    _need_cuda("draft_tokens", draft_tokens, torch.int32, (B, k))
    dev = target_logits.device
    if out_tokens is None:
        out_tokens = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    if accepted_len is None:
        accepted_len = torch.empty((B,), dtype=torch.int32, device=dev)
    _need_cuda("out_tokens", out_tokens, torch.int32, (B, k + 1))
    _need_cuda("accepted_len", accepted_len, torch.int32, (B,))
    for name, t in (("dbg_logp", dbg_logp), ("dbg_logq", dbg_logq)):
        if t is not None:
            _need_cuda(name, t, torch.float32, (B, k))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    if workspace_buf is None:
        workspace_buf = workspace(B, 2 * k + 1, vocab, dev) if B > 0 else None
    ws_bytes = 0 if workspace_buf is None else workspace_buf.numel()
    rc = load_library().spec_verify_linear(
        _ptr(target_logits), _ptr(draft_logits), _dtype_code(target_logits), stride,
        _ptr(draft_tokens), B, k, vocab, float(temperature), int(seed), int(offset),
        _ptr(out_tokens), _ptr(accepted_len), _ptr(dbg_logp), _ptr(dbg_logq), _ptr(status),
        _ptr(workspace_buf), ws_bytes, _stream(stream))
    _check(rc, "spec_verify_linear")
    return out_tokens, accepted_len


def spec_verify_greedy(target_logits, draft_tokens, vocab, out_tokens=None, accepted_len=None,
                       status=None, workspace_buf=None, stream=None, workspace_free=False):
    """target_logits [B][k+1][stride], draft_tokens [B][k] int32.  By default
    the streamed form runs in a cached workspace (or workspace_buf);
    workspace_free=True runs the cluster form, which needs none."""
    _need_cuda("target_logits", target_logits)
    B, R, stride = target_logits.shape
    k = R - 1
    _need_cuda("draft_tokens", draft_tokens, torch.int32, (B, k))
    dev = target_logits.device
    if out_tokens is None:
        out_tokens = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    if accepted_len is None:
        accepted_len = torch.empty((B,), dtype=torch.int32, device=dev)
    _need_cuda("out_tokens", out_tokens, torch.int32, (B, k + 1))
    _need_cuda("accepted_len", accepted_len, torch.int32, (B,))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    if workspace_free:
        workspace_buf = None
    elif workspace_buf is None and B > 0:
        workspace_buf = workspace(B, k + 1, vocab, dev)
    ws_bytes = 0 if workspace_buf is None else workspace_buf.numel()
    rc = load_library().spec_verify_greedy(
        _ptr(target_logits), _dtype_code(target_logits), stride, _ptr(draft_tokens), B, k, vocab,
        _ptr(out_tokens), _ptr(accepted_len), _ptr(status), _ptr(workspace_buf), ws_bytes,
        _stream(stream))
    _check(rc, "spec_verify_greedy")
    return out_tokens, accepted_len


def spec_verify_greedy_walk(target_logits, draft_tokens, vocab, out_tokens=None,
                            accepted_len=None, status=None, stream=None):
    """As spec_verify_greedy, reading only target rows 0..n of each request."""
    _need_cuda("target_logits", target_logits)
    B, R, stride = target_logits.shape
    k = R - 1
    _need_cuda("draft_tokens", draft_tokens, torch.int32, (B, k))
    dev = target_logits.device
    if out_tokens is None:
        out_tokens = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    if accepted_len is None:
        accepted_len = torch.empty((B,), dtype=torch.int32, device=dev)
    _need_cuda("out_tokens", out_tokens, torch.int32, (B, k + 1))
    _need_cuda("accepted_len", accepted_len, torch.int32, (B,))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    rc = load_library().spec_verify_greedy_walk(
        _ptr(target_logits), _dtype_code(target_logits), stride, _ptr(draft_tokens), B, k, vocab,
        _ptr(out_tokens), _ptr(accepted_len), _ptr(status), _stream(stream))
    _check(rc, "spec_verify_greedy_walk")
    return out_tokens, accepted_len


def spec_verify_tree_greedy_walk(target_logits, node_tokens, parents, max_depth, vocab,
                                 out_tokens=None, accepted_len=None, out_path_nodes=None,
                                 status=None, stream=None):
    """As spec_verify_tree with stochastic=False, reading only the rows of
    kept nodes.  Returns (out_tokens [B][D+1], accepted_len [B],
    out_path_nodes [B][D+1] or None)."""
    _need_cuda("target_logits", target_logits)
    B, N, stride = target_logits.shape
    _need_cuda("node_tokens", node_tokens, torch.int32, (B, N))
    _need_cuda("parents", parents, torch.int32, (B, N))
    dev = target_logits.device
    W = max_depth + 1
    if out_tokens is None:
        out_tokens = torch.empty((B, W), dtype=torch.int32, device=dev)
    if accepted_len is None:
        accepted_len = torch.empty((B,), dtype=torch.int32, device=dev)
    _need_cuda("out_tokens", out_tokens, torch.int32, (B, W))
    _need_cuda("accepted_len", accepted_len, torch.int32, (B,))
    if out_path_nodes is not None:
        _need_cuda("out_path_nodes", out_path_nodes, torch.int32, (B, W))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    rc = load_library().spec_verify_tree_greedy_walk(
        _ptr(target_logits), _dtype_code(target_logits), stride, _ptr(node_tokens),
        _ptr(parents), B, N, max_depth, vocab, _ptr(out_tokens), _ptr(accepted_len),
        _ptr(out_path_nodes), _ptr(status), _stream(stream))
    _check(rc, "spec_verify_tree_greedy_walk")
    return out_tokens, accepted_len, out_path_nodes


def spec_verify_tree(target_logits, draft_logits, node_tokens, parents, max_depth, vocab,
                     stochastic, temperature=1.0, seed=0, offset=0, out_tokens=None,
                     accepted_len=None, out_path_nodes=None, status=None, workspace_buf=None,
                     stream=None):
    """target_logits [B][N][stride]; draft_logits [B][N][stride] or None (greedy);
    node_tokens, parents [B][N] int32.  stochastic: 0 (or False) greedy, 1 (or
    True) an independent test per node, 2 distribution-exact (siblings tested
    in turn against the residual).  Returns (out_tokens [B][D+1],
    accepted_len [B], out_path_nodes [B][D+1] or None)."""
    stochastic = int(stochastic)
    if stochastic not in (0, 1, 2):
        raise ValueError("stochastic must be 0, 1 or 2")
    _need_cuda("target_logits", target_logits)
    B, N, stride = target_logits.shape
    if stochastic:
        _need_cuda("draft_logits", draft_logits, target_logits.dtype, (B, N, stride))
    _need_cuda("node_tokens", node_tokens, torch.int32, (B, N))
    _need_cuda("parents", parents, torch.int32, (B, N))
    dev = target_logits.device
    W = max_depth + 1
    if out_tokens is None:
        out_tokens = torch.empty((B, W), dtype=torch.int32, device=dev)
    if accepted_len is None:
        accepted_len = torch.empty((B,), dtype=torch.int32, device=dev)
    _need_cuda("out_tokens", out_tokens, torch.int32, (B, W))
    _need_cuda("accepted_len", accepted_len, torch.int32, (B,))
    if out_path_nodes is not None:
        _need_cuda("out_path_nodes", out_path_nodes, torch.int32, (B, W))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    if workspace_buf is None:
        workspace_buf = workspace(B, 2 * N, vocab, dev) if B > 0 else None
    ws_bytes = 0 if workspace_buf is None else workspace_buf.numel()
    rc = load_library().spec_verify_tree(
        _ptr(target_logits), _ptr(draft_logits if stochastic else None),
        _dtype_code(target_logits), stride, _ptr(node_tokens), _ptr(parents), B, N, max_depth,
        vocab, int(stochastic), float(temperature), int(seed), int(offset), _ptr(out_tokens),
        _ptr(accepted_len), _ptr(out_path_nodes), _ptr(status), _ptr(workspace_buf), ws_bytes,
        _stream(stream))
    _check(rc, "spec_verify_tree")
    return out_tokens, accepted_len, out_path_nodes


def spec_verify_debug_uniforms(seed, offset, purpose, batch, count, first_position=0,
                               device=None, stream=None):
    """[batch][count] float64 device tensor of the kernels' uniforms."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    out = torch.empty((batch, count), dtype=torch.float64, device=device)
    rc = load_library().spec_verify_debug_uniforms(int(seed), int(offset), int(purpose), batch,
                                                   count, first_position, _ptr(out),
                                                   _stream(stream))
    _check(rc, "spec_verify_debug_uniforms")
    return out


def spec_verify_debug_exp2(z, kind=0, stream=None):
    """2^z (z <= 0) from one of the kernels' exponentials (kind 0: fp64
    table driven; 1: fp32 FMA-pipe polynomial; 2: fp32 special-function
    unit); z a float64 CUDA tensor."""
    _need_cuda("z", z, torch.float64)
    out = torch.empty_like(z)
    rc = load_library().spec_verify_debug_exp2(_ptr(z), _ptr(out), z.numel(), int(kind),
                                               _stream(stream))
    _check(rc, "spec_verify_debug_exp2")
    return out


def spec_verify_debug_wait_expiry(target_logits, draft_logits, draft_tokens, vocab, temperature,
                                  poll_limit, status, out_tokens=None, accepted_len=None,
                                  workspace_buf=None, stream=None):
    """spec_verify_linear with its waits made to expire after poll_limit polls
    (diagnostic: pass 1 stores nothing, so every decide step gives up and
    reports SPEC_STATUS_TIMEOUT into status; the outputs stay -1)."""
    _need_cuda("target_logits", target_logits)
    B, R, stride = target_logits.shape
    k = R - 1
    _need_cuda("draft_logits", draft_logits, target_logits.dtype, (B, k, stride))
    _need_cuda("draft_tokens", draft_tokens, torch.int32, (B, k))
    _need_cuda("status", status, torch.int32)
    dev = target_logits.device
    if out_tokens is None:
        out_tokens = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    if accepted_len is None:
        accepted_len = torch.empty((B,), dtype=torch.int32, device=dev)
    if workspace_buf is None:
        workspace_buf = workspace(B, 2 * k + 1, vocab, dev) if B > 0 else None
    ws_bytes = 0 if workspace_buf is None else workspace_buf.numel()
    rc = load_library().spec_verify_debug_wait_expiry(
        _ptr(target_logits), _ptr(draft_logits), _dtype_code(target_logits), stride,
        _ptr(draft_tokens), B, k, vocab, float(temperature), int(poll_limit), _ptr(out_tokens),
        _ptr(accepted_len), _ptr(status), _ptr(workspace_buf), ws_bytes, _stream(stream))
    _check(rc, "spec_verify_debug_wait_expiry")
    return out_tokens, accepted_len


def spec_verify_linear_noalloc(target_logits, draft_logits, draft_tokens, vocab, temperature,
                               seed, offset, out_tokens, accepted_len, dbg_logp=None,
                               dbg_logq=None, status=None, stream=None):
    """Linear verification through the entry point that allocates nothing.

    For callers that cannot allocate device memory (a plugin whose host
    framework owns the device pool, a serving loop that forbids cudaMalloc
    while running): the outputs must be passed in, no workspace is taken,
    and the library uses its own static 8 MiB device scratch.  Calls that
    overlap on the GPU share that scratch and must not be issued
    concurrently."""
    _need_cuda("target_logits", target_logits)
    B, R, stride = target_logits.shape
    k = R - 1
    _need_cuda("draft_logits", draft_logits, target_logits.dtype, (B, k, stride))
    _need_cuda("draft_tokens", draft_tokens, torch.int32, (B, k))
    _need_cuda("out_tokens", out_tokens, torch.int32, (B, k + 1))
    _need_cuda("accepted_len", accepted_len, torch.int32, (B,))
    for name, t in (("dbg_logp", dbg_logp), ("dbg_logq", dbg_logq)):
        if t is not None:
            _need_cuda(name, t, torch.float32, (B, k))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    rc = load_library().spec_verify_linear_noalloc(
        _ptr(target_logits), _ptr(draft_logits), _dtype_code(target_logits), stride,
        _ptr(draft_tokens), B, k, vocab, float(temperature), int(seed), int(offset),
        _ptr(out_tokens), _ptr(accepted_len), _ptr(dbg_logp), _ptr(dbg_logq), _ptr(status),
        _stream(stream))
    _check(rc, "spec_verify_linear_noalloc")
    return out_tokens, accepted_len


def spec_plug_tokens(in_tokens, out_tokens, accepted_len, next_tokens=None, seq_tokens=None,
                     seq_len=None, status=None, stream=None):
    """Write the next step's input tokens from a verification's outputs on
    the device (no host synchronisation).  in_tokens, out_tokens [B][k+1],
    accepted_len [B] int32; next_tokens [B][k+1] (output, allocated when
    None and want); seq_tokens [B][cap] and seq_len [B] updated in place.
    Returns next_tokens."""
    _need_cuda("out_tokens", out_tokens, torch.int32)
    B, W = out_tokens.shape
    k = W - 1
    _need_cuda("in_tokens", in_tokens, torch.int32, (B, W))
    _need_cuda("accepted_len", accepted_len, torch.int32, (B,))
    if next_tokens is None:
        next_tokens = torch.empty((B, W), dtype=torch.int32, device=out_tokens.device)
    _need_cuda("next_tokens", next_tokens, torch.int32, (B, W))
    cap = 0
    if seq_tokens is not None or seq_len is not None:
        _need_cuda("seq_tokens", seq_tokens, torch.int32)
        if seq_tokens.dim() != 2 or seq_tokens.shape[0] != B:
            raise ValueError("seq_tokens must be [B][capacity]")
        cap = seq_tokens.shape[1]
        _need_cuda("seq_len", seq_len, torch.int32, (B,))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    rc = load_library().spec_plug_tokens(_ptr(in_tokens), _ptr(out_tokens), _ptr(accepted_len), B,
                                         k, _ptr(next_tokens), _ptr(seq_tokens), _ptr(seq_len), cap,
                                         _ptr(status), _stream(stream))
    _check(rc, "spec_plug_tokens")
    return next_tokens


# ------------------------------------------------------------ vocabulary-sharded steps
SHARD_DRAW_WORDS = 6


def spec_shard_row_stats(target_logits, draft_logits, draft_tokens, vocab_lo, vocab_hi,
                         temperature=1.0, stream=None):
    """Per-row statistics of this rank's columns [vocab_lo, vocab_hi).
    Stochastic (draft_logits given): dict(max [B][2k+1] f32, sum [B][2k+1]
    f64, probe [B][k][2] f32); greedy (draft_logits None): dict(max
    [B][k+1] f32, arg [B][k+1] int32)."""
    _need_cuda("target_logits", target_logits)
    B, R1, stride = target_logits.shape
    k = R1 - 1
    _need_cuda("draft_tokens", draft_tokens, torch.int32, (B, k))
    dev = target_logits.device
    stoch = draft_logits is not None
    if stoch:
        _need_cuda("draft_logits", draft_logits, target_logits.dtype, (B, k, stride))
    R = 2 * k + 1 if stoch else k + 1
    mx = torch.empty((B, R), dtype=torch.float32, device=dev)
    sm = torch.empty((B, R), dtype=torch.float64, device=dev) if stoch else None
    arg = None if stoch else torch.empty((B, R), dtype=torch.int32, device=dev)
    probe = torch.empty((B, k, 2), dtype=torch.float32, device=dev) if stoch else None
    rc = load_library().spec_shard_row_stats(
        _ptr(target_logits), _ptr(draft_logits), _dtype_code(target_logits), stride,
        _ptr(draft_tokens), B, k, int(vocab_lo), int(vocab_hi), float(temperature), _ptr(mx),
        _ptr(sm), _ptr(arg), _ptr(probe), _stream(stream))
    _check(rc, "spec_shard_row_stats")
    return dict(max=mx, sum=sm, arg=arg, probe=probe)


def spec_shard_decide(max_all, sum_all, probe_all, bounds, draft_tokens, vocab, temperature,
                      seed=0, offset=0, status=None, stream=None):
    """Merge the ranks' statistics (rank order) and run the accept tests.
    Returns (out_tokens [B][k+1] with the drawn slot still -1,
    accepted_len [B], draw [B][6] f64)."""
    _need_cuda("max_all", max_all, torch.float32)
    W, B, R = max_all.shape
    k = (R - 1) // 2
    _need_cuda("sum_all", sum_all, torch.float64, (W, B, R))
    _need_cuda("probe_all", probe_all, torch.float32, (W, B, k, 2))
    _need_cuda("bounds", bounds, torch.int32, (W + 1,))
    _need_cuda("draft_tokens", draft_tokens, torch.int32, (B, k))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    dev = max_all.device
    out = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    acc = torch.empty((B,), dtype=torch.int32, device=dev)
    draw = torch.empty((B, SHARD_DRAW_WORDS), dtype=torch.float64, device=dev)
    rc = load_library().spec_shard_decide(
        _ptr(max_all), _ptr(sum_all), _ptr(probe_all), _ptr(bounds), W, _ptr(draft_tokens), B, k,
        int(vocab), float(temperature), int(seed), int(offset), _ptr(out), _ptr(acc), _ptr(draw),
        _ptr(status), _stream(stream))
    _check(rc, "spec_shard_decide")
    return out, acc, draw


def spec_shard_decide_greedy(max_all, arg_all, draft_tokens, vocab, status=None, stream=None):
    """Greedy verification from the ranks' (max, lowest argmax) per target row."""
    _need_cuda("max_all", max_all, torch.float32)
    W, B, R = max_all.shape
    k = R - 1
    _need_cuda("arg_all", arg_all, torch.int32, (W, B, R))
    _need_cuda("draft_tokens", draft_tokens, torch.int32, (B, k))
    if status is not None:
        _need_cuda("status", status, torch.int32)
    dev = max_all.device
    out = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    acc = torch.empty((B,), dtype=torch.int32, device=dev)
    rc = load_library().spec_shard_decide_greedy(_ptr(max_all), _ptr(arg_all), W, _ptr(draft_tokens),
                                                 B, k, int(vocab), _ptr(out), _ptr(acc),
                                                 _ptr(status), _stream(stream))
    _check(rc, "spec_shard_decide_greedy")
    return out, acc


def spec_shard_draw_sums(target_logits, draft_logits, vocab_lo, vocab_hi, temperature, draw,
                         norm_parts=None, stream=None):
    """fp64 sums over this rank's columns of each request's draw rows:
    without norm_parts (sum e, sum f); with the ranks' gathered first sums
    [W][B][2] (the draw mass, sum e).  Returns [B][2] f64."""
    _need_cuda("target_logits", target_logits)
    B, R1, stride = target_logits.shape
    k = R1 - 1
    _need_cuda("draft_logits", draft_logits, target_logits.dtype, (B, k, stride))
    _need_cuda("draw", draw, torch.float64, (B, SHARD_DRAW_WORDS))
    W = 1
    if norm_parts is not None:
        _need_cuda("norm_parts", norm_parts, torch.float64)
        W = norm_parts.shape[0]
    sums = torch.empty((B, 2), dtype=torch.float64, device=target_logits.device)
    rc = load_library().spec_shard_draw_sums(
        _ptr(target_logits), _ptr(draft_logits), _dtype_code(target_logits), stride, B, k,
        int(vocab_lo), int(vocab_hi), float(temperature), _ptr(draw), _ptr(norm_parts), W,
        _ptr(sums), _stream(stream))
    _check(rc, "spec_shard_draw_sums")
    return sums


def spec_shard_draw_pick(target_logits, draft_logits, vocab_lo, vocab_hi, temperature, draw,
                         norm_parts, mass_parts, shard_index, stream=None):
    """The token of each request if this rank owns the part of the running
    mass that holds u * Z (drawn inside its columns), else -1.  [B] int32."""
    _need_cuda("target_logits", target_logits)
    B, R1, stride = target_logits.shape
    k = R1 - 1
    _need_cuda("draft_logits", draft_logits, target_logits.dtype, (B, k, stride))
    _need_cuda("draw", draw, torch.float64, (B, SHARD_DRAW_WORDS))
    _need_cuda("norm_parts", norm_parts, torch.float64)
    W = norm_parts.shape[0]
    _need_cuda("mass_parts", mass_parts, torch.float64, (W, B, 2))
    token = torch.empty((B,), dtype=torch.int32, device=target_logits.device)
    rc = load_library().spec_shard_draw_pick(
        _ptr(target_logits), _ptr(draft_logits), _dtype_code(target_logits), stride, B, k,
        int(vocab_lo), int(vocab_hi), float(temperature), _ptr(draw), _ptr(norm_parts),
        _ptr(mass_parts), W, int(shard_index), _ptr(token), _stream(stream))
    _check(rc, "spec_shard_draw_pick")
    return token


def spec_shard_emit(token, draw, out_tokens, stream=None):
    """out_tokens[b][n] = token[b] for every request that draws one."""
    _need_cuda("out_tokens", out_tokens, torch.int32)
    B, W1 = out_tokens.shape
    _need_cuda("token", token, torch.int32, (B,))
    _need_cuda("draw", draw, torch.float64, (B, SHARD_DRAW_WORDS))
    rc = load_library().spec_shard_emit(_ptr(token), _ptr(draw), B, W1 - 1, _ptr(out_tokens),
                                        _stream(stream))
    _check(rc, "spec_shard_emit")
    return out_tokens
