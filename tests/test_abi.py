"""The C-ABI library builds for sm_100a, loads without a GPU, exports every
symbol include/specverify.h declares, and rejects bad arguments on the host
before touching the device (these calls return before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "specverify.h")

SPEC_OK, SPEC_EINVAL, SPEC_EALIGN, SPEC_EUNSUPPORTED, SPEC_ECUDA, SPEC_EWORKSPACE = 0, -1, -2, -3, -4, -5


@pytest.fixture(scope="module")
def lib():
    from speculative_decoding_verification_87_b200 import binding, build
    build.build()
    return binding.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"SPECVERIFY_API\s+[\w\s\*]+?\b(spec_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    assert {"spec_verify_linear", "spec_verify_greedy", "spec_verify_tree",
            "spec_verify_workspace_size", "spec_verify_strerror"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    from speculative_decoding_verification_87_b200 import binding
    assert set(declared_symbols()) == set(binding.SYMBOLS)


def test_workspace_size(lib):
    a = lib.spec_verify_workspace_size(64, 17, 128256)
    b = lib.spec_verify_workspace_size(128, 17, 128256)
    assert a > 0 and b > a and a % 256 == 0
    assert lib.spec_verify_workspace_size(0, 17, 100) > 0
    assert lib.spec_verify_workspace_size(4, 0, 100) == 0
    assert lib.spec_verify_workspace_size(4, 9, 0) == 0
    assert lib.spec_verify_workspace_size(-1, 9, 10) == 0


def test_strerror(lib):
    for code in (SPEC_OK, SPEC_EINVAL, SPEC_EALIGN, SPEC_EUNSUPPORTED, SPEC_ECUDA,
                 SPEC_EWORKSPACE, 12345):
        assert isinstance(lib.spec_verify_strerror(code), bytes)
    assert lib.spec_verify_strerror(SPEC_OK) == b"ok"


def _linear(lib, tl=0x1000, dl=0x2000, dtype=1, stride=128, tokens=0x3000, batch=2, k=3,
            vocab=100, temperature=1.0, ws=0x10000, ws_bytes=1 << 30):
    P = ctypes.c_void_p
    return lib.spec_verify_linear(P(tl), P(dl), dtype, stride, P(tokens), batch, k, vocab,
                                  temperature, 0, 0, P(0x4000), P(0x5000), None, None, None,
                                  P(ws), ws_bytes, None)


def test_linear_host_validation(lib):
    assert _linear(lib, k=0) == SPEC_EINVAL
    assert _linear(lib, k=33) == SPEC_EUNSUPPORTED
    assert _linear(lib, batch=-1) == SPEC_EINVAL
    assert _linear(lib, temperature=0.0) == SPEC_EINVAL
    assert _linear(lib, temperature=float("nan")) == SPEC_EINVAL
    assert _linear(lib, temperature=float("inf")) == SPEC_EINVAL
    assert _linear(lib, vocab=0) == SPEC_EINVAL
    assert _linear(lib, vocab=129) == SPEC_EINVAL            # stride < vocab
    assert _linear(lib, dtype=7) == SPEC_EINVAL
    assert _linear(lib, tl=0) == SPEC_EINVAL
    assert _linear(lib, dl=0) == SPEC_EINVAL
    assert _linear(lib, tokens=0) == SPEC_EINVAL
    assert _linear(lib, stride=100) == SPEC_EALIGN           # 200-byte bf16 rows
    assert _linear(lib, tl=0x1008) == SPEC_EALIGN
    assert _linear(lib, ws=0) == SPEC_EWORKSPACE
    assert _linear(lib, ws=0x10010) == SPEC_EWORKSPACE
    assert _linear(lib, ws_bytes=16) == SPEC_EWORKSPACE
    assert _linear(lib, batch=0) == SPEC_OK                  # nothing to enqueue
    assert _linear(lib, batch=0, tl=0, dl=0, tokens=0) == SPEC_OK


def test_noalloc_checks_arguments_before_the_scratch_size(lib):
    # too large for the static scratch: SPEC_EUNSUPPORTED, unless an argument
    # is invalid, which keeps the code spec_verify_linear gives it
    P = ctypes.c_void_p

    def na(**kw):
        return lib.spec_verify_linear_noalloc(
            P(kw.get("tl", 0x1000)), P(0x2000), 1, 128256, P(0x3000), kw.get("batch", 5000), 8,
            128256, kw.get("temp", 1.0), 0, 0, P(0x4000), P(0x5000), None, None, None, None)
    assert na() == SPEC_EUNSUPPORTED
    assert na(temp=0.0) == SPEC_EINVAL
    assert na(tl=0) == SPEC_EINVAL
    assert na(tl=0x1008) == SPEC_EALIGN


def test_debug_wait_expiry_host_validation(lib):
    P = ctypes.c_void_p

    def d(**kw):
        return lib.spec_verify_debug_wait_expiry(
            P(0x1000), P(0x2000), 1, 128, P(0x3000), 2, 3, 100, 1.0, kw.get("polls", 16),
            P(0x4000), P(0x5000), P(kw.get("status", 0x6000)), P(kw.get("ws", 0x10000)),
            kw.get("ws_bytes", 1 << 30), None)
    assert d(polls=0) == SPEC_EINVAL
    assert d(polls=4097) == SPEC_EINVAL
    assert d(status=0) == SPEC_EINVAL     # the expiry is reported through status
    assert d(ws=0) == SPEC_EWORKSPACE


def test_plug_host_validation(lib):
    P = ctypes.c_void_p

    def pl(**kw):
        return lib.spec_plug_tokens(P(kw.get("inp", 0x1000)), P(kw.get("out", 0x2000)),
                                    P(kw.get("acc", 0x3000)), kw.get("batch", 4), kw.get("k", 3),
                                    P(kw.get("nxt", 0x4000)), P(kw.get("seq", 0)),
                                    P(kw.get("ln", 0)), kw.get("cap", 0), None, None)
    assert pl(k=0) == SPEC_EINVAL and pl(k=33) == SPEC_EUNSUPPORTED
    assert pl(batch=-1) == SPEC_EINVAL and pl(cap=-1) == SPEC_EINVAL
    assert pl(seq=0x5000) == SPEC_EINVAL          # seq_tokens without seq_len
    assert pl(ln=0x5000) == SPEC_EINVAL           # seq_len without seq_tokens
    assert pl(out=0) == SPEC_EINVAL and pl(acc=0) == SPEC_EINVAL
    assert pl(inp=0) == SPEC_EINVAL               # next_tokens needs the inputs
    assert pl(nxt=0) == SPEC_OK                   # nothing asked for: nothing enqueued
    assert pl(batch=0, out=0, acc=0) == SPEC_OK


def test_greedy_and_tree_host_validation(lib):
    P = ctypes.c_void_p
    g = lambda **kw: lib.spec_verify_greedy(P(kw.get("tl", 0x1000)), kw.get("dtype", 0),
                                            kw.get("stride", 64), P(0x2000), kw.get("batch", 3),
                                            kw.get("k", 2), kw.get("vocab", 50), P(0x3000),
                                            P(0x4000), None, P(kw.get("ws", 0)),
                                            kw.get("ws_bytes", 0), None)
    assert g(k=0) == SPEC_EINVAL and g(k=40) == SPEC_EUNSUPPORTED
    assert g(stride=63) == SPEC_EALIGN and g(vocab=65) == SPEC_EINVAL
    assert g(batch=0) == SPEC_OK
    # the streamed form: an aligned workspace of spec_verify_workspace_size(B, k+1, V) bytes
    need = lib.spec_verify_workspace_size(3, 3, 50)
    assert need > 0
    assert g(ws=0x10000, ws_bytes=need - 1) == SPEC_EWORKSPACE
    assert g(ws=0x10010, ws_bytes=need) == SPEC_EWORKSPACE   # not 256-byte aligned
    assert g(ws=0x10000, ws_bytes=need, batch=0) == SPEC_OK

    def t(**kw):
        return lib.spec_verify_tree(P(0x1000), P(kw.get("dl", 0x2000)), 1, 64, P(0x3000),
                                    P(0x3800), kw.get("batch", 2), kw.get("nodes", 60),
                                    kw.get("depth", 6), 60, kw.get("stoch", 1),
                                    kw.get("temp", 1.0), 0, 0, P(0x4000), P(0x5000), None, None,
                                    P(0x10000), kw.get("ws_bytes", 1 << 30), None)
    assert t(nodes=0) == SPEC_EINVAL and t(nodes=1025) == SPEC_EUNSUPPORTED
    assert t(depth=0) == SPEC_EINVAL
    assert t(dl=0) == SPEC_EINVAL                 # stochastic trees read draft rows
    assert t(dl=0, batch=0) == SPEC_OK            # an empty batch reads nothing
    assert t(temp=-1.0) == SPEC_EINVAL
    assert t(stoch=3) == SPEC_EINVAL and t(stoch=-1) == SPEC_EINVAL
    assert t(stoch=2, dl=0) == SPEC_EINVAL        # the exact mode reads draft rows too
    assert t(ws_bytes=8) == SPEC_EWORKSPACE
    assert t(batch=0) == SPEC_OK


def test_walk_host_validation(lib):
    P = ctypes.c_void_p
    g = lambda **kw: lib.spec_verify_greedy_walk(P(kw.get("tl", 0x1000)), kw.get("dtype", 0),
                                                 kw.get("stride", 64), P(kw.get("tok", 0x2000)),
                                                 kw.get("batch", 3), kw.get("k", 2),
                                                 kw.get("vocab", 50), P(0x3000), P(0x4000), None,
                                                 None)
    assert g(k=0) == SPEC_EINVAL and g(k=33) == SPEC_EUNSUPPORTED
    assert g(batch=-1) == SPEC_EINVAL
    assert g(stride=63) == SPEC_EALIGN and g(vocab=65) == SPEC_EINVAL and g(vocab=0) == SPEC_EINVAL
    assert g(tl=0x1004) == SPEC_EALIGN and g(tl=0) == SPEC_EINVAL and g(tok=0) == SPEC_EINVAL
    assert g(dtype=3) == SPEC_EINVAL
    assert g(batch=0) == SPEC_OK and g(batch=0, tl=0, tok=0) == SPEC_OK

    def t(**kw):
        return lib.spec_verify_tree_greedy_walk(P(kw.get("tl", 0x1000)), 1, 64, P(0x3000),
                                                P(kw.get("par", 0x3800)), kw.get("batch", 2),
                                                kw.get("nodes", 60), kw.get("depth", 6), 60,
                                                P(0x4000), P(0x5000), None, None, None)
    assert t(nodes=0) == SPEC_EINVAL and t(nodes=1025) == SPEC_EUNSUPPORTED
    assert t(depth=0) == SPEC_EINVAL and t(batch=-2) == SPEC_EINVAL
    assert t(par=0) == SPEC_EINVAL and t(tl=0x1002) == SPEC_EALIGN
    assert t(batch=0) == SPEC_OK and t(batch=0, tl=0, par=0) == SPEC_OK


def test_binding_fails_loudly_without_the_library(tmp_path):
    # the product path has no fallback: a missing library is an error, and
    # the binding never imports the oracle
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from speculative_decoding_verification_87_b200 import binding\n"
        "try:\n"
        "    binding.load_library(%r)\n"
        "except binding.SpecVerifyError as e:\n"
        "    print('raised', 'missing' in str(e))\n"
        "print('oracle' in sys.modules)\n" % (ROOT, str(tmp_path / "absent.so")))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         timeout=120).stdout.split()
    assert out == ["raised", "True", "False"], out
