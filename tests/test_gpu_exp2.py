"""Accuracy of the kernels' fp64 2^z (Tang's table-driven method) against
the host math library's exp2, through the diagnostic C-ABI entry point."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from speculative_decoding_verification_87_b200 import binding, build
    build.build()
    binding.load_library()
    return binding


def test_exp2_fp64_relative_error(sv):
    rng = np.random.default_rng(0)
    z = np.concatenate([
        -rng.random(1 << 20) * 1.0,              # the dense range near the maximum
        -rng.random(1 << 20) * 60.0,             # typical (l - m) / T * log2 e
        -rng.random(1 << 16) * 1019.0,           # the whole normal range
        -np.arange(0, 64) / 64.0,                # table points
        np.array([0.0, -0.0, -1e-300, -1.0 / 128, -1.0 / 128 + 1e-17]),
    ])
    got = sv.spec_verify_debug_exp2(torch.from_numpy(z).cuda()).cpu().numpy()
    ref = np.exp2(z)
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-15, (rel.max(), z[np.argmax(rel)])
    assert got[np.where(z == 0.0)[0][0]] == 1.0


@pytest.mark.parametrize("kind", [1, 2])
def test_exp2_fp32_relative_error(sv, kind):
    """The fp32 exponentials of the streaming pass: the FMA-pipe polynomial
    (kind 1) and the special-function unit (kind 2), on fp32 inputs."""
    rng = np.random.default_rng(1)
    z = np.concatenate([-rng.random(1 << 20) * 124.0, -rng.random(1 << 16),
                        np.array([0.0, -0.5, -1.5, -124.5])]).astype(np.float32).astype(np.float64)
    got = sv.spec_verify_debug_exp2(torch.from_numpy(z).cuda(), kind=kind).cpu().numpy()
    ref = np.exp2(z)
    rel = np.abs(got - ref) / ref
    assert rel.max() < 4e-7, (kind, rel.max(), z[np.argmax(rel)])


def test_exp2_fma_flushes_below_range(sv):
    z = np.array([-125.5, -200.0, -np.inf])
    got = sv.spec_verify_debug_exp2(torch.from_numpy(z).cuda(), kind=1).cpu().numpy()
    assert np.all(got == 0.0)


def test_exp2_fp64_tiny_results_are_zero(sv):
    z = np.array([-1020.5, -1100.0, -np.inf, -3000.0])
    got = sv.spec_verify_debug_exp2(torch.from_numpy(z).cuda()).cpu().numpy()
    assert np.all(got == 0.0)
