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


_SCALARS = {"int": ctypes.c_int, "int64_t": ctypes.c_int64, "uint32_t": ctypes.c_uint32,
            "uint64_t": ctypes.c_uint64, "float": ctypes.c_float, "spec_dtype": ctypes.c_int,
            "spec_status": ctypes.c_int}


def _prototypes():
    import re
    text = open(binding.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    for name, params in re.findall(r"\b(spec_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        ps = [" ".join(p.split()) for p in params.split(",")]
        yield name, [] if ps == ["void"] or ps == [""] else ps


def test_binding_marshals_every_parameter_with_its_c_type(L):
    """The ctypes declarations have the header's arity and, parameter by
    parameter, a pointer where the header has one and the same scalar width."""
    protos = list(_prototypes())
    assert {n for n, _ in protos} == set(binding.declared_symbols())
    for name, params in protos:
        argtypes = getattr(L, name).argtypes
        assert argtypes is not None and len(argtypes) == len(params), name
        for c_param, ct in zip(params, argtypes):
            if "*" in c_param or "[" in c_param or c_param.split()[0] == "cudaStream_t":
                assert ct is ctypes.c_void_p or issubclass(ct, (ctypes._Pointer, ctypes.c_char_p)), \
                    (name, c_param, ct)
            else:
                base = c_param.replace("const ", "").rsplit(" ", 1)[0]
                assert ctypes.sizeof(ct) == ctypes.sizeof(_SCALARS[base]), (name, c_param, ct)
                assert (ct is ctypes.c_float) == (base == "float"), (name, c_param, ct)
                if base.startswith("uint"):
                    assert ct in (ctypes.c_uint32, ctypes.c_uint64), (name, c_param, ct)


def test_null_lmhead_and_shard_handles_are_rejected(L):
    assert L.spec_lmhead_destroy(None) == binding.SPEC_OK
    assert L.spec_lmhead_set_cta_pairs(None, 1) == binding.SPEC_ERR_INVALID_ARG
    assert L.spec_lmhead_errors(None, None) == binding.SPEC_ERR_INVALID_ARG
    assert L.spec_lmhead_logits(None, None, 1, None, 64, 1000, None, None) == \
        binding.SPEC_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert L.spec_lmhead_init(ctypes.byref(h), None, 2560) == binding.SPEC_ERR_INVALID_ARG
    assert not h.value
    assert L.spec_shard_stats(None, 0, 2, None, None, 1, None, None, None, None, 4, 3, 1000,
                              None, None) == binding.SPEC_ERR_INVALID_ARG
    assert L.spec_shard_finish(None, None, 4, 3, None, None, None) == binding.SPEC_ERR_INVALID_ARG
    assert L.spec_shard_refine_finish(None, None, 4, 3, None, None, None) == \
        binding.SPEC_ERR_INVALID_ARG
