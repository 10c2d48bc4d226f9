"""Python access to the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports this package, and nothing here imports the CUDA package.

``build()`` compiles ``oracle.c`` with gcc into ``liboracle.so`` beside it
(no fast-math, no FMA contraction, so the arithmetic is the plain fp64 the
source spells out).

``ORACLE_LIB_OVERRIDE`` (environment) names another build of the same source
to load instead; the mutation tests use it to check that the pins fail on a
copy of the oracle with one planted mistake.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPE_F32 = 0
DTYPE_BF16 = 1

ERR_BAD_TOKEN = 1
ERR_NONFINITE = 2
ERR_BAD_TEMPERATURE = 4


def compile_source(src: str, out: str) -> str:
    """gcc with the oracle's flags: ``src`` (C) -> shared library ``out``."""
    tmp = out + ".tmp.%d" % os.getpid()
    subprocess.check_call([
        "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
        "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, src, "-lm",
    ])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


class _Inputs(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("target", ctypes.c_void_p),
        ("draft", ctypes.c_void_p),
        ("draft_tokens", ctypes.c_void_p),
        ("verify_len", ctypes.c_void_p),
        ("temperature", ctypes.c_void_p),
        ("conf_hidden", ctypes.c_void_p),
        ("conf_w", ctypes.c_void_p),
        ("conf_bias", ctypes.c_float),
        ("conf_threshold", ctypes.c_float),
        ("conf_kb", ctypes.c_int),
        ("conf_H", ctypes.c_int),
        ("conf_total", ctypes.c_int64),
        ("B", ctypes.c_int),
        ("k", ctypes.c_int),
        ("V", ctypes.c_int64),
        ("seed", ctypes.c_uint64),
        ("step", ctypes.c_uint32),
        ("request_offset", ctypes.c_uint32),
        ("u_override", ctypes.c_void_p),
    ]


class _Outputs(ctypes.Structure):
    _fields_ = [
        ("accepted", ctypes.c_void_p),
        ("tokens", ctypes.c_void_p),
        ("p_x", ctypes.c_void_p),
        ("q_x", ctypes.c_void_p),
        ("accept_margin", ctypes.c_void_p),
        ("sample_margin", ctypes.c_void_p),
        ("verify_len_used", ctypes.c_void_p),
        ("status", ctypes.c_void_p),
    ]


_lib = None
_lock = threading.Lock()


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(os.environ.get("ORACLE_LIB_OVERRIDE") or build())
            _lib.oracle_philox4x32_10.argtypes = [ctypes.c_void_p] * 3
            _lib.oracle_philox4x32_10.restype = None
            _lib.oracle_uniform.argtypes = [ctypes.c_uint64] + [ctypes.c_uint32] * 4
            _lib.oracle_uniform.restype = ctypes.c_double
            _lib.oracle_uniform_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                                 ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p]
            _lib.oracle_uniform_fill.restype = None
            _lib.oracle_budget_topn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int64, ctypes.c_void_p]
            _lib.oracle_budget_topn.restype = ctypes.c_int
            _lib.oracle_verify_lengths.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
            _lib.oracle_verify_lengths.restype = ctypes.c_int
            _lib.oracle_conf_budget.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
            _lib.oracle_conf_budget.restype = ctypes.c_int
            _lib.oracle_verify.argtypes = [ctypes.POINTER(_Inputs), ctypes.POINTER(_Outputs)]
            _lib.oracle_verify.restype = ctypes.c_int
            _lib.oracle_row_softmax.argtypes = [
                ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p]
            _lib.oracle_row_softmax.restype = ctypes.c_int
            _lib.oracle_row_argmax.argtypes = [
                ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p]
            _lib.oracle_row_argmax.restype = ctypes.c_int
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def philox(counter, key) -> np.ndarray:
    """Philox4x32-10 block for a 4-word counter and 2-word key."""
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def uniform(seed: int, request: int, position: int, draw: int, step: int = 0) -> float:
    return lib().oracle_uniform(seed, request, position, draw, step)


def uniform_grid(seed: int, requests: int, positions: int, draw: int, step: int = 0) -> np.ndarray:
    """U(seed, i, j, draw, step) for i < requests, j < positions, as [requests, positions]."""
    out = np.zeros((requests, positions), dtype=np.float64)
    lib().oracle_uniform_fill(seed, requests, positions, draw, step, _ptr(out))
    return out


def conf_budget(hidden: np.ndarray, w: np.ndarray, bias: float, threshold: float):
    """hidden: uint16 bf16 bits [B, kb, H]; w: uint16 [H]. Returns (len, s, prefix)."""
    hidden = np.ascontiguousarray(hidden, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint16)
    B, kb, H = hidden.shape
    out_len = np.zeros(B, dtype=np.int32)
    surv = np.zeros((B, kb), dtype=np.float64)
    pref = np.zeros((B, kb), dtype=np.float64)
    rc = lib().oracle_conf_budget(_ptr(hidden), _ptr(w), bias, B, kb, H, threshold,
                                  _ptr(out_len), _ptr(surv), _ptr(pref))
    assert rc == 0
    return out_len, surv, pref


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) widened exactly to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def lmhead_logits(hidden: np.ndarray, head: np.ndarray) -> np.ndarray:
    """Logits of the shared output head, l = h W^T ("Speculative decoding
    becomes standard: DSpark and multi-token drafters", section "What DSpark
    adds": the drafter shares the target's frozen output head), in fp64 from
    the bf16 inputs: hidden [..., H] and head [V, H] as uint16 bits ->
    float64 [..., V].  One library matmul is the whole step; every product of
    two bf16 values is exact in fp64."""
    h = bf16_to_f64(hidden)
    w = bf16_to_f64(head)
    return h @ w.T


def verify_lmhead(hidden_target, hidden_draft, head, draft_tokens, **kw):
    """Verification of the rows the shared head produces: the fp64 logits of
    ``lmhead_logits`` rounded to fp32 (the precision the fused path holds its
    accumulators in; on inputs whose partial sums are exact in fp32 the
    rounding is exact too), then ``verify`` with dtype fp32."""
    t = lmhead_logits(hidden_target, head).astype(np.float32)
    d = None if hidden_draft is None else lmhead_logits(hidden_draft, head).astype(np.float32)
    return verify(t, d, draft_tokens, dtype=DTYPE_F32, **kw)


def row_softmax(row: np.ndarray, dtype: int, T: float) -> np.ndarray:
    row = np.ascontiguousarray(row)
    out = np.zeros(row.shape[-1], dtype=np.float64)
    rc = lib().oracle_row_softmax(_ptr(row), dtype, row.shape[-1], T, _ptr(out))
    if rc:
        raise ValueError("row rejected by the oracle: error bits %d" % rc)
    return out


def row_argmax(row: np.ndarray, dtype: int) -> int:
    row = np.ascontiguousarray(row)
    out = np.zeros(1, dtype=np.int32)
    rc = lib().oracle_row_argmax(_ptr(row), dtype, row.shape[-1], _ptr(out))
    if rc:
        raise ValueError("row rejected by the oracle: error bits %d" % rc)
    return int(out[0])


def _verify_slice(d, lo, hi, res):
    B, k = hi - lo, d["k"]
    sl = lambda a: None if a is None else np.ascontiguousarray(a[lo:hi])
    keep = []
    def keepref(a):
        keep.append(a)
        return _ptr(a)
    inp = _Inputs()
    inp.dtype = d["dtype"]
    inp.target = keepref(sl(d["target"]))
    inp.draft = keepref(sl(d["draft"]))
    inp.draft_tokens = keepref(sl(d["draft_tokens"]))
    inp.verify_len = keepref(sl(d["verify_len"]))
    inp.temperature = keepref(sl(d["temperature"]))
    inp.conf_hidden = keepref(sl(d["conf_hidden"]))
    inp.conf_w = keepref(d["conf_w"])
    inp.conf_bias = d["conf_bias"]
    inp.conf_threshold = d["conf_threshold"]
    inp.conf_kb = d["conf_kb"]
    inp.conf_H = d["conf_H"]
    inp.conf_total = d.get("conf_total", 0)
    inp.B = B
    inp.k = k
    inp.V = d["V"]
    inp.seed = d["seed"]
    inp.step = d["step"]
    inp.request_offset = d["request_offset"] + lo
    inp.u_override = keepref(sl(d["u_override"]))
    out = _Outputs()
    out.accepted = _ptr(res["accepted"][lo:hi])
    out.tokens = _ptr(res["tokens"][lo:hi])
    out.p_x = _ptr(res["p_x"][lo:hi])
    out.q_x = _ptr(res["q_x"][lo:hi])
    out.accept_margin = _ptr(res["accept_margin"][lo:hi])
    out.sample_margin = _ptr(res["sample_margin"][lo:hi])
    out.verify_len_used = _ptr(res["verify_len_used"][lo:hi])
    out.status = _ptr(res["status"][lo:hi])
    rc = lib().oracle_verify(ctypes.byref(inp), ctypes.byref(out))
    assert rc == 0, rc


def _verify_lengths(d, B):
    keep = []
    def keepref(a):
        keep.append(a)
        return _ptr(a)
    inp = _Inputs()
    inp.verify_len = keepref(d["verify_len"])
    inp.conf_hidden = keepref(d["conf_hidden"])
    inp.conf_w = keepref(d["conf_w"])
    inp.conf_bias = d["conf_bias"]
    inp.conf_threshold = d["conf_threshold"]
    inp.conf_kb = d["conf_kb"]
    inp.conf_H = d["conf_H"]
    inp.conf_total = d["conf_total"]
    inp.B = B
    inp.k = d["k"]
    out = np.zeros(B, dtype=np.int32)
    rc = lib().oracle_verify_lengths(ctypes.byref(inp), _ptr(out))
    assert rc == 0, rc
    return out


def budget_topn(prefix: np.ndarray, cap: np.ndarray, total: int) -> np.ndarray:
    """Batch-wide verify budget: prefix [B, kb] fp64 survival products, cap [B]
    candidate positions per request, total budget -> L [B] int32."""
    prefix = np.ascontiguousarray(prefix, dtype=np.float64)
    B, kb = prefix.shape
    cap = np.ascontiguousarray(cap, dtype=np.int32)
    out = np.zeros(B, dtype=np.int32)
    rc = lib().oracle_budget_topn(_ptr(prefix), _ptr(cap), B, kb, int(total), _ptr(out))
    if rc:
        raise ValueError("oracle_budget_topn rejected its arguments (%d)" % rc)
    return out


def verify(target, draft, draft_tokens, *, dtype, verify_len=None, temperature=None,
           conf=None, seed=0, step=0, request_offset=0, u_override=None, threads=1):
    """Run the oracle over a batch.

    target: [B, k+1, V] float32 or uint16 (bf16 bits); draft: [B, k, V] same
    dtype or None; draft_tokens: [B, k] int32; verify_len: [B] int32 or None;
    temperature: [B] float32 or None; conf: dict(hidden=[B,kb,H] uint16,
    w=[H] uint16, bias=float, threshold=float[, total=int batch-wide verify
    budget]) or None; u_override:
    [B, k+1, 2] float64 or None.  ``threads`` > 1 runs contiguous request
    groups concurrently (each request is independent; the global request index
    keeps the random draws identical).
    """
    target = np.ascontiguousarray(target)
    B, kp1, V = target.shape
    k = kp1 - 1
    d = dict(
        dtype=dtype, target=target,
        draft=None if draft is None else np.ascontiguousarray(draft),
        draft_tokens=np.ascontiguousarray(draft_tokens, dtype=np.int32).reshape(B, k),
        verify_len=None if verify_len is None else np.ascontiguousarray(verify_len, dtype=np.int32),
        temperature=None if temperature is None else np.ascontiguousarray(temperature, dtype=np.float32),
        conf_hidden=None if conf is None else np.ascontiguousarray(conf["hidden"], dtype=np.uint16),
        conf_w=None if conf is None else np.ascontiguousarray(conf["w"], dtype=np.uint16),
        conf_bias=0.0 if conf is None else float(conf["bias"]),
        conf_threshold=0.0 if conf is None else float(conf["threshold"]),
        conf_kb=0 if conf is None else int(conf["hidden"].shape[1]),
        conf_H=0 if conf is None else int(conf["hidden"].shape[2]),
        conf_total=0 if conf is None else int(conf.get("total", 0)),
        k=k, V=V, seed=int(seed), step=int(step), request_offset=int(request_offset),
        u_override=None if u_override is None else np.ascontiguousarray(u_override, dtype=np.float64),
    )
    if dtype == DTYPE_BF16:
        assert target.dtype == np.uint16
    else:
        assert target.dtype == np.float32
    res = dict(
        accepted=np.zeros(B, dtype=np.int32),
        tokens=np.zeros((B, k + 1), dtype=np.int32),
        p_x=np.zeros((B, k), dtype=np.float64),
        q_x=np.zeros((B, k), dtype=np.float64),
        accept_margin=np.zeros((B, k), dtype=np.float64),
        sample_margin=np.zeros(B, dtype=np.float64),
        verify_len_used=np.zeros(B, dtype=np.int32),
        status=np.zeros(B, dtype=np.uint32),
    )
    if B == 0:
        return res
    threads = max(1, min(int(threads), B))
    if threads > 1 and d["conf_total"] > 0:
        # the batch-wide budget couples the requests: fix every L_i on the
        # whole batch first, then verify slices with those lengths
        lengths = _verify_lengths(d, B)
        d = dict(d, verify_len=lengths, conf_hidden=None, conf_total=0)
    if threads == 1:
        _verify_slice(d, 0, B, res)
    else:
        bounds = np.linspace(0, B, threads + 1).astype(int)
        with ThreadPoolExecutor(threads) as ex:
            futs = [ex.submit(_verify_slice, d, int(bounds[t]), int(bounds[t + 1]), res)
                    for t in range(threads) if bounds[t + 1] > bounds[t]]
            for f in futs:
                f.result()
    return res
