"""The C-ABI library loads and exports every entry point its header declares;
host-side argument checks answer without touching a GPU."""
import ctypes

import pytest

from speculative_decoding_verification_86_b200 import binding, build


@pytest.fixture(scope="module")
def L():
    build.build()
    return binding.lib()


def test_every_declared_symbol_is_exported(L):
    names = binding.declared_symbols()
    assert "spec_verify_run" in names and "spec_verify_greedy" in names
    assert "spec_verify_init" in names and "spec_conf_budget" in names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for s in range(7):
        assert binding.status_string(s)
    assert binding.status_string(0) == "ok"


def test_null_context_is_rejected(L):
    args = [None, None, None, 1, None, None, None, None, 1, 1, 8, 0, 0, 0,
            None, None, None, None, None, None]
    assert L.spec_verify_run(*args) == binding.SPEC_ERR_INVALID_ARG
    assert L.spec_verify_greedy(None, None, 1, None, None, 1, 1, 8, None, None, None, None) == \
        binding.SPEC_ERR_INVALID_ARG
    assert L.spec_conf_budget(None, None, None, 0.5, 1, 1, 8, 0.3, None, None, None) == \
        binding.SPEC_ERR_INVALID_ARG
    assert L.spec_verify_destroy(None) == binding.SPEC_OK


def test_init_argument_checks(L):
    h = ctypes.c_void_p()
    assert L.spec_verify_init(None, 0, 1, 1, 8) == binding.SPEC_ERR_INVALID_ARG
    assert L.spec_verify_init(ctypes.byref(h), 0, 0, 1, 8) == binding.SPEC_ERR_INVALID_ARG
    assert L.spec_verify_init(ctypes.byref(h), 0, 1, 17, 8) == binding.SPEC_ERR_INVALID_ARG
    assert L.spec_verify_init(ctypes.byref(h), 0, 1, 1, 0) == binding.SPEC_ERR_INVALID_ARG
    assert not h.value


def test_init_without_a_gpu_reports_an_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    st = L.spec_verify_init(ctypes.byref(h), 0, 4, 5, 1000)
    assert st in (binding.SPEC_ERR_CUDA, binding.SPEC_ERR_INVALID_ARG)
    assert not h.value


def test_error_bound_constant(L):
    b = L.spec_verify_ex2_error_bound()
    assert 1e-7 < b < 1e-6
