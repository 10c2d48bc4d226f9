"""Thin ctypes binding of ``libspecverify.so`` (the C ABI in include/spec_verify.h).

Only argument marshalling lives here: tensors become device pointers, the
current torch CUDA stream becomes the ``cudaStream_t``.  Every step of the
verification runs in the library's CUDA kernels.  There is no fallback: if
the library is missing or fails to load, :func:`lib` raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspecverify.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "spec_verify.h")

SPEC_OK = 0
SPEC_ERR_INVALID_ARG = 1
SPEC_ERR_UNSUPPORTED = 2
SPEC_ERR_CUDA = 3
SPEC_ERR_NOMEM = 4
SPEC_ERR_DEVICE_STATUS = 5
SPEC_ERR_TIMEOUT = 6

SPEC_F32 = 0
SPEC_BF16 = 1

SPEC_MODE_DENSE = 0
SPEC_MODE_PREFIX = 1
MODES = {"dense": SPEC_MODE_DENSE, "prefix": SPEC_MODE_PREFIX}

DEV_BAD_TOKEN = 1
DEV_NONFINITE = 2
DEV_BAD_TEMPERATURE = 4
DEV_INTERNAL = 16

TIMING_ENGINE, TIMING_CONF = 0, 3
TIMING_STATS = TIMING_ENGINE


class SpecVerifyError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (where, status_string(status), status))


class ConfArgs(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_void_p), ("w", ctypes.c_void_p), ("bias", ctypes.c_float),
                ("kb", ctypes.c_int), ("H", ctypes.c_int), ("threshold", ctypes.c_float),
                ("total_budget", ctypes.c_int64)]


_lib = None
_vp = ctypes.c_void_p
_i32 = ctypes.c_int
_i64 = ctypes.c_int64
_u32 = ctypes.c_uint32
_u64 = ctypes.c_uint64


def lib():
    """Load the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libspecverify.so is not built (%s); run "
                           "`python -m speculative_decoding_verification_86_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    L.spec_status_string.argtypes = [_i32]
    L.spec_status_string.restype = ctypes.c_char_p
    L.spec_verify_init.argtypes = [ctypes.POINTER(_vp), _i32, _i32, _i32, _i64]
    L.spec_verify_destroy.argtypes = [_vp]
    run_common = [_vp, _vp, _vp, _i32, _vp, _vp, _vp, ctypes.POINTER(ConfArgs), _i32, _i32, _i64]
    L.spec_verify_run.argtypes = run_common + [_u64, _u32, _u32, _vp, _vp, _vp, _vp, _vp, _vp]
    L.spec_verify_run_with_uniforms.argtypes = run_common + [_vp, _vp, _vp, _vp, _vp, _vp, _vp]
    L.spec_verify_run_host.argtypes = run_common + [_u64, _u32, _u32, _vp, _vp, _vp, _vp, _vp, _vp]
    L.spec_verify_greedy.argtypes = [_vp, _vp, _i32, _vp, _vp, _i32, _i32, _i64, _vp, _vp, _vp, _vp]
    L.spec_verify_greedy_noalloc.argtypes = [_vp, _i32, _vp, _vp, _i32, _i32, _i64, _vp, _vp, _vp, _vp]
    L.spec_conf_budget.argtypes = [_vp, _vp, _vp, ctypes.c_float, _i32, _i32, _i32,
                                   ctypes.c_float, _vp, _vp, _vp]
    L.spec_verify_lengths.argtypes = [_vp, ctypes.POINTER(ConfArgs), _vp, _i32, _i32, _vp, _vp, _vp]
    L.spec_verify_set_mode.argtypes = [_vp, _i32]
    L.spec_verify_timing_enable.argtypes = [_vp, _i32]
    L.spec_verify_timing_read.argtypes = [_vp, _i32, ctypes.POINTER(_i32), ctypes.POINTER(ctypes.c_double)]
    L.spec_verify_last_counters.argtypes = [_vp, _vp, ctypes.POINTER(_u32)]
    L.spec_verify_selfcheck_ex2.argtypes = [_i32, ctypes.c_float, ctypes.c_float,
                                            ctypes.POINTER(ctypes.c_double)]
    L.spec_verify_ex2_error_bound.argtypes = []
    L.spec_verify_ex2_error_bound.restype = ctypes.c_double
    for name in ("spec_verify_init", "spec_verify_destroy", "spec_verify_run",
                 "spec_verify_run_with_uniforms", "spec_verify_run_host", "spec_verify_greedy",
                 "spec_conf_budget", "spec_verify_lengths", "spec_verify_greedy_noalloc",
                 "spec_verify_set_mode",
                 "spec_verify_timing_enable", "spec_verify_timing_read",
                 "spec_verify_last_counters", "spec_verify_selfcheck_ex2"):
        getattr(L, name).restype = _i32
    _lib = L
    return L


def declared_symbols() -> list:
    """Entry points declared in include/spec_verify.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(spec_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().spec_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != SPEC_OK:
        raise SpecVerifyError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SPEC_BF16
    if t.dtype == torch.float32:
        return SPEC_F32
    raise TypeError("logits must be bfloat16 or float32, got %s" % t.dtype)


def _dev_ptr(t, dtype=None, device=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _stream_handle(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


class SpecVerifier:
    """A verification context (device workspace) on one GPU.

    ``run`` / ``greedy`` / ``conf_budget`` launch asynchronously on the given
    (default: current) torch stream and return output tensors.
    """

    def __init__(self, device=None, max_batch=1024, max_k=8, max_vocab=262144, mode="prefix"):
        dev = torch.device("cuda") if device is None else torch.device(device)
        if dev.type != "cuda":
            raise ValueError("SpecVerifier needs a CUDA device, got %s" % dev)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self.max_batch, self.max_k, self.max_vocab = max_batch, max_k, max_vocab
        h = _vp()
        _check(lib().spec_verify_init(ctypes.byref(h), self.device.index, max_batch, max_k,
                                      max_vocab), "spec_verify_init")
        self._h = h
        self.set_mode(mode)

    def set_mode(self, mode):
        """Statistics order: "prefix" (default: rows past the first rejection
        are never read) or "dense" (every verified position's rows)."""
        _check(lib().spec_verify_set_mode(self._h, MODES[mode]), "spec_verify_set_mode")
        self.mode = mode

    # -- lifecycle ------------------------------------------------------------
    def close(self):
        if getattr(self, "_h", None):
            lib().spec_verify_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # -- helpers --------------------------------------------------------------
    def _outputs(self, B, k, with_pq=True, out=None):
        if out is not None:
            return out
        d = self.device
        o = dict(accepted=torch.empty(B, dtype=torch.int32, device=d),
                 tokens=torch.empty((B, k + 1), dtype=torch.int32, device=d),
                 status=torch.empty(B, dtype=torch.int32, device=d))
        if with_pq:
            o["p"] = torch.empty((B, k), dtype=torch.float32, device=d)
            o["q"] = torch.empty((B, k), dtype=torch.float32, device=d)
        return o

    def _conf(self, conf):
        if conf is None:
            return None, None
        hidden, w = conf["hidden"], conf["w"]
        c = ConfArgs(_dev_ptr(hidden, torch.bfloat16, self.device, "conf.hidden"),
                     _dev_ptr(w, torch.bfloat16, self.device, "conf.w"), float(conf["bias"]),
                     int(hidden.shape[1]), int(hidden.shape[2]), float(conf["threshold"]),
                     int(conf.get("total", 0)))
        return ctypes.byref(c), c

    def _shape(self, target, draft, tokens):
        if target.dim() != 3:
            raise ValueError("target logits must be [B, k+1, V]")
        B, kp1, V = target.shape
        k = kp1 - 1
        if draft is not None and tuple(draft.shape) != (B, k, V):
            raise ValueError("draft logits must be [B, k, V] = %s" % ((B, k, V),))
        if tuple(tokens.shape) != (B, k):
            raise ValueError("draft tokens must be [B, k] = %s" % ((B, k),))
        return B, k, V

    # -- entry points ---------------------------------------------------------
    def run(self, target, draft, tokens, verify_len=None, temperature=None, conf=None, seed=0,
            step=0, request_offset=0, stream=None, out=None, uniforms=None):
        """spec_verify_run (or spec_verify_run_with_uniforms when ``uniforms`` is given)."""
        B, k, V = self._shape(target, draft, tokens)
        dt = _dtype_code(target)
        if draft is not None and draft.dtype != target.dtype:
            raise TypeError("draft logits must have the target's dtype")
        o = self._outputs(B, k, True, out)
        cref, _keep = self._conf(conf)
        args = [self._h, _dev_ptr(target, None, self.device, "target"),
                _dev_ptr(draft, None, self.device, "draft"), dt,
                _dev_ptr(tokens, torch.int32, self.device, "tokens"),
                _dev_ptr(verify_len, torch.int32, self.device, "verify_len"),
                _dev_ptr(temperature, torch.float32, self.device, "temperature"), cref, B, k, V]
        outs = [_dev_ptr(o["accepted"], torch.int32), _dev_ptr(o["tokens"], torch.int32),
                _dev_ptr(o.get("p")), _dev_ptr(o.get("q")), _dev_ptr(o["status"]),
                _stream_handle(stream, self.device)]
        if uniforms is not None:
            if tuple(uniforms.shape) != (B, k + 1, 2):
                raise ValueError("uniforms must be [B, k+1, 2]")
            st = lib().spec_verify_run_with_uniforms(
                *args, _dev_ptr(uniforms, torch.float64, self.device, "uniforms"), *outs)
            _check(st, "spec_verify_run_with_uniforms")
        else:
            st = lib().spec_verify_run(*args, int(seed), int(step), int(request_offset), *outs)
            _check(st, "spec_verify_run")
        return o

    def greedy(self, target, tokens, verify_len=None, stream=None, out=None):
        """spec_verify_greedy (temperature 0, no draft logits)."""
        B, k, V = self._shape(target, None, tokens)
        o = self._outputs(B, k, False, out)
        st = lib().spec_verify_greedy(
            self._h, _dev_ptr(target, None, self.device, "target"), _dtype_code(target),
            _dev_ptr(tokens, torch.int32, self.device, "tokens"),
            _dev_ptr(verify_len, torch.int32, self.device, "verify_len"), B, k, V,
            _dev_ptr(o["accepted"], torch.int32), _dev_ptr(o["tokens"], torch.int32),
            _dev_ptr(o["status"]), _stream_handle(stream, self.device))
        _check(st, "spec_verify_greedy")
        return o

    def conf_budget(self, hidden, w, bias, threshold, stream=None, with_survival=True):
        """spec_conf_budget: returns (lengths [B] int32, survival [B, kb] fp32 or None)."""
        B, kb, H = hidden.shape
        out_len = torch.empty(B, dtype=torch.int32, device=self.device)
        surv = torch.empty((B, kb), dtype=torch.float32, device=self.device) if with_survival else None
        st = lib().spec_conf_budget(
            self._h, _dev_ptr(hidden, torch.bfloat16, self.device, "hidden"),
            _dev_ptr(w, torch.bfloat16, self.device, "w"), float(bias), B, kb, H, float(threshold),
            _dev_ptr(out_len, torch.int32), _dev_ptr(surv), _stream_handle(stream, self.device))
        _check(st, "spec_conf_budget")
        return out_len, surv

    def lengths(self, conf, k, verify_len=None, stream=None, with_survival=False):
        """spec_verify_lengths: the verified lengths L [B] int32 that
        spec_verify_run would use (verify_len, threshold, conf["total"]), and
        optionally the survival [B, kb] fp32."""
        B, kb, _ = conf["hidden"].shape
        if verify_len is not None and tuple(verify_len.shape) != (B,):
            raise ValueError("verify_len must be [B]")
        cref, keep = self._conf(conf)
        out_len = torch.empty(B, dtype=torch.int32, device=self.device)
        surv = torch.empty((B, kb), dtype=torch.float32, device=self.device) if with_survival else None
        st = lib().spec_verify_lengths(
            self._h, cref, _dev_ptr(verify_len, torch.int32, self.device, "verify_len"), B, int(k),
            _dev_ptr(out_len, torch.int32), _dev_ptr(surv), _stream_handle(stream, self.device))
        del keep
        _check(st, "spec_verify_lengths")
        return out_len, surv

    def run_host(self, target, draft, tokens, verify_len=None, temperature=None, conf=None,
                 seed=0, step=0, request_offset=0, stream=None, out=None, allow_failed=True):
        """spec_verify_run_host: CPU tensors in (pinned for speed), CPU tensors out."""
        B, kp1, V = target.shape
        k = kp1 - 1
        dt = _dtype_code(target)

        def hp(t):
            if t is None:
                return None
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("run_host takes contiguous CPU tensors")
            return t.data_ptr()

        if out is None:
            out = dict(accepted=torch.empty(B, dtype=torch.int32), tokens=torch.empty((B, k + 1), dtype=torch.int32),
                       p=torch.empty((B, k), dtype=torch.float32), q=torch.empty((B, k), dtype=torch.float32),
                       status=torch.empty(B, dtype=torch.int32))
        keep = None
        cref = None
        if conf is not None:
            keep = ConfArgs(hp(conf["hidden"]), hp(conf["w"]), float(conf["bias"]),
                            int(conf["hidden"].shape[1]), int(conf["hidden"].shape[2]),
                            float(conf["threshold"]), int(conf.get("total", 0)))
            cref = ctypes.byref(keep)
        st = lib().spec_verify_run_host(
            self._h, hp(target), hp(draft), dt, hp(tokens), hp(verify_len), hp(temperature), cref,
            B, k, V, int(seed), int(step), int(request_offset), hp(out["accepted"]), hp(out["tokens"]),
            hp(out.get("p")), hp(out.get("q")), hp(out["status"]), _stream_handle(stream, self.device))
        if st == SPEC_ERR_DEVICE_STATUS and allow_failed:
            return out
        _check(st, "spec_verify_run_host")
        return out

    # -- diagnostics ----------------------------------------------------------
    def timing_enable(self, classes=(TIMING_STATS,)):
        """Bracket launches of the given kernel classes with CUDA events (empty: off)."""
        mask = 0
        for c in classes:
            mask |= 1 << int(c)
        _check(lib().spec_verify_timing_enable(self._h, mask), "spec_verify_timing_enable")

    def timing_read(self, which):
        n = _i32()
        ms = ctypes.c_double()
        _check(lib().spec_verify_timing_read(self._h, which, ctypes.byref(n), ctypes.byref(ms)),
               "spec_verify_timing_read")
        return n.value, ms.value

    def last_counters(self, stream=None):
        out = (_u32 * 5)()
        _check(lib().spec_verify_last_counters(self._h, _stream_handle(stream, self.device), out),
               "spec_verify_last_counters")
        return dict(accept_fp64=out[0], sample_fp64=out[1], sample_fp32=out[2], chunks_fp64=out[3],
                    engine_error=out[4])


def greedy_noalloc(target, tokens, verify_len=None, stream=None, out=None):
    """spec_verify_greedy_noalloc: greedy verification for callers that may not
    allocate device memory (the library's fixed scratch array is used; see the
    header for the size limits).  ``out`` lets the caller pass preallocated
    outputs (accepted [B], tokens [B, k+1], status [B], int32, on the device)."""
    if target.dim() != 3:
        raise ValueError("target logits must be [B, k+1, V]")
    B, kp1, V = target.shape
    dev = target.device
    if out is None:
        out = dict(accepted=torch.empty(B, dtype=torch.int32, device=dev),
                   tokens=torch.empty((B, kp1), dtype=torch.int32, device=dev),
                   status=torch.empty(B, dtype=torch.int32, device=dev))
    st = lib().spec_verify_greedy_noalloc(
        _dev_ptr(target, None, dev, "target"), _dtype_code(target),
        _dev_ptr(tokens, torch.int32, dev, "tokens"), _dev_ptr(verify_len, torch.int32, dev, "verify_len"),
        B, kp1 - 1, V, _dev_ptr(out["accepted"], torch.int32), _dev_ptr(out["tokens"], torch.int32),
        _dev_ptr(out["status"]), _stream_handle(stream, dev))
    _check(st, "spec_verify_greedy_noalloc")
    return out


def selfcheck_ex2(device=0, lo=-126.0, hi=0.0):
    """(measured max relative error of ex2.approx.ftz.f32 on [lo, hi], bound the kernels assume)."""
    v = ctypes.c_double()
    _check(lib().spec_verify_selfcheck_ex2(int(device), float(lo), float(hi), ctypes.byref(v)),
           "spec_verify_selfcheck_ex2")
    return v.value, lib().spec_verify_ex2_error_bound()


# C-ABI names, for callers who prefer the flat interface.
def spec_verify_init(device=0, max_batch=1024, max_k=8, max_vocab=262144):
    return SpecVerifier(device, max_batch, max_k, max_vocab)


def spec_verify_destroy(ctx: SpecVerifier):
    ctx.close()


def spec_verify_run(ctx: SpecVerifier, *a, **kw):
    return ctx.run(*a, **kw)


def spec_verify_greedy(ctx: SpecVerifier, *a, **kw):
    return ctx.greedy(*a, **kw)


def spec_conf_budget(ctx: SpecVerifier, *a, **kw):
    return ctx.conf_budget(*a, **kw)


def spec_verify_run_host(ctx: SpecVerifier, *a, **kw):
    return ctx.run_host(*a, **kw)
