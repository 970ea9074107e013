"""CPU-only checks of libtq.so: it loads, exports every entry point that
include/tq.h declares, its host math matches the oracle, and argument
validation / host fault injection behave (no GPU work is launched here)."""

import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

from oracle import codebook, rotation

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    m = build_lib()
    return m


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(tq):
    names = _declared_functions()
    assert len(names) >= 20
    for name in names:
        assert hasattr(tq._lib.lib, name), name
    assert set(names) == set(tq._lib.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", tq._lib.LIB_PATH], capture_output=True, text=True).stdout
    for name in names:
        assert re.search(rf"\bT {name}\b", out), name


@pytest.mark.parametrize("d,bits", [(3, 1), (3, 3), (16, 2), (128, 1), (128, 2), (128, 3), (128, 4), (1536, 2),
                                    (1536, 4)])
def test_host_codebook_matches_oracle(tq, d, bits):
    c, b = tq.tq_codebook_host(d, bits)
    co, bo = codebook.lloyd_max(d, bits)
    assert np.allclose(c, co, rtol=0, atol=1e-12)
    assert np.allclose(b, bo, rtol=0, atol=1e-12)
    assert np.array_equal(c, -c[::-1])


@pytest.mark.parametrize("level,bits", [(1, 4), (1, 3), (2, 1), (2, 2), (3, 2), (4, 3), (5, 4), (7, 2), (8, 2)])
def test_host_polar_codebook_matches_oracle(tq, level, bits):
    from oracle import polar
    c, b = tq.tq_polar_codebook_host(level, bits)
    co, bo = polar.lloyd_max(level, bits)
    # the oracle's cell moments come from a cumulative table (about 1e-12 relative); the library
    # integrates each cell by Gauss-Legendre quadrature
    assert np.allclose(c, co, rtol=0, atol=2e-10)
    assert np.allclose(b, bo, rtol=0, atol=2e-10)
    if level > 1:   # symmetric about pi/4
        assert np.allclose(c + c[::-1], np.pi / 2, atol=1e-15)


@pytest.mark.parametrize("d,m,seed", [(32, 32, 0), (128, 128, 2), (128, 0, 3), (256, 64, 9)])
def test_host_rotation_matches_oracle(tq, d, m, seed):
    Pi, S = tq.tq_rotation_host(d, m, seed)
    Po, So = rotation.rotation(d, seed, m)
    assert np.abs(Pi - Po).max() <= 1e-12
    if m:
        assert np.abs(S - So).max() <= 1e-12
    assert np.abs(Pi.T @ Pi - np.eye(d)).max() <= 1e-13


def test_host_rotation_large_d(tq):
    Pi, _ = tq.tq_rotation_host(1536, 0, 0)
    Po, _ = rotation.rotation(1536, 0)
    assert np.abs(Pi - Po).max() <= 1e-12


def test_argument_validation_without_gpu(tq):
    h = ctypes.c_void_p()
    lib = tq._lib.lib
    assert lib.tq_create(100, 3, 0, ctypes.byref(h)) == tq.TQ_EUNSUPPORTED      # d % 32 != 0
    assert "multiple of 32" in tq.tq_last_error()
    assert lib.tq_create(128, 5, 0, ctypes.byref(h)) == tq.TQ_EUNSUPPORTED      # MSE bits > 4
    assert lib.tq_create_prod(128, 3, 48, 0, ctypes.byref(h)) == tq.TQ_EUNSUPPORTED  # m % 32 != 0
    assert lib.tq_create_prod(256, 3, 128, 0, ctypes.byref(h)) == tq.TQ_EUNSUPPORTED  # prod d > 128
    assert lib.tq_create(128, 3, 0, None) == tq.TQ_EINVAL
    assert lib.tq_encode(None, None, 0, 0, None, None, None, None, None) == tq.TQ_EINVAL
    assert lib.tq_codebook_host(2, 3, None, None) == tq.TQ_EINVAL
    assert lib.tq_score_workspace_bytes(None, 1, 1) == 0
    assert lib.tq_last_status(None, None) == tq.TQ_EINVAL
    with pytest.raises(tq.TQError):
        tq.tq_codebook_host(2, 1)


def test_fault_injection_alloc_is_host_side(tq):
    code = ("import ctypes, embedding_vector_quantization_b200 as t;"
            "h = ctypes.c_void_p();"
            "print(t._lib.lib.tq_create(128, 3, 0, ctypes.byref(h)), t.tq_last_error())")
    env = dict(os.environ, TQ_FAULT="alloc", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=ROOT)
    assert out.stdout.startswith(str(tq.TQ_ENOMEM)), out.stdout + out.stderr
    assert "TQ_FAULT=alloc" in out.stdout


def test_without_gpu_create_reports_cuda_error(tq):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(tq.TQError) as e:
        tq.tq_create(128, 3, 0)
    assert e.value.status == tq.TQ_ECUDA
