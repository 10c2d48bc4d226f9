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
SPEC_MODE_AUTO = 2
MODES = {"dense": SPEC_MODE_DENSE, "prefix": SPEC_MODE_PREFIX, "auto": SPEC_MODE_AUTO}

DEV_BAD_TOKEN = 1
DEV_NONFINITE = 2
DEV_BAD_TEMPERATURE = 4
DEV_INTERNAL = 16

TIMING_ENGINE, TIMING_LM_STATS, TIMING_LM_ROWS, TIMING_CONF = 0, 1, 2, 3
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
    shard_common = [_vp, _i32, _i32]
    shard_inputs = [_vp, _vp, _i32, _vp, _vp, _vp, ctypes.POINTER(ConfArgs), _i32, _i32, _i64]
    L.spec_shard_layout.argtypes = [_i32, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _vp]
    L.spec_shard_refine_partials.argtypes = shard_common + shard_inputs + [_vp, _vp]
    L.spec_shard_refine_locate.argtypes = shard_common + [_vp] + shard_inputs + [_vp, _vp]
    L.spec_shard_refine_finish.argtypes = [_vp, _vp, _i32, _i32, _vp, _vp, _vp]
    L.spec_shard_stats.argtypes = shard_common + shard_inputs + [_vp, _vp]
    L.spec_shard_decide.argtypes = shard_common + [_vp] + shard_inputs + [
        _u64, _u32, _u32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    L.spec_shard_locate.argtypes = shard_common + [_vp] + shard_inputs + [_vp, _vp]
    L.spec_shard_finish.argtypes = [_vp, _vp, _i32, _i32, _vp, _vp, _vp]
    L.spec_lmhead_init.argtypes = [ctypes.POINTER(_vp), _vp, _i32]
    L.spec_lmhead_destroy.argtypes = [_vp]
    L.spec_lmhead_errors.argtypes = [_vp, ctypes.POINTER(_u32)]
    L.spec_lmhead_set_cta_pairs.argtypes = [_vp, _i32]
    L.spec_lmhead_logits.argtypes = [_vp, _vp, _i32, _vp, _i32, _i64, _vp, _vp]
    L.spec_lmhead_verify.argtypes = [_vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp,
                                     ctypes.POINTER(ConfArgs), _i32, _i32, _i64, _u64, _u32, _u32,
                                     _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    L.spec_verify_set_mode.argtypes = [_vp, _i32]
    L.spec_verify_set_prefix_tail.argtypes = [_vp, _i32]
    L.spec_verify_draws.argtypes = [_vp, _u64, _u32, _u32, _i32, _i32, _vp, _vp]
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
                 "spec_shard_layout", "spec_shard_stats", "spec_shard_decide", "spec_shard_locate",
                 "spec_shard_finish", "spec_shard_refine_partials", "spec_shard_refine_locate",
                 "spec_shard_refine_finish",
                 "spec_lmhead_init", "spec_lmhead_destroy", "spec_lmhead_errors",
                 "spec_lmhead_logits", "spec_lmhead_verify", "spec_lmhead_set_cta_pairs",
                 "spec_verify_set_mode", "spec_verify_set_prefix_tail", "spec_verify_draws",
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

    def __init__(self, device=None, max_batch=1024, max_k=8, max_vocab=262144, mode="auto"):
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
        """Statistics order: "auto" (default: dense when every row the batch
        may verify fits in one wave of the grid, else prefix), "prefix" (rows
        past the first rejection are never read) or "dense" (every verified
        position's rows)."""
        _check(lib().spec_verify_set_mode(self._h, MODES[mode]), "spec_verify_set_mode")
        self.mode = mode

    def set_prefix_tail(self, position):
        """Prefix order: read all remaining positions of a request at once
        after it accepted positions 0 .. position-1 (1..17; above k: one
        position at a time; 0, the default: chosen per run from the batch's
        size against the grid).  The outputs do not depend on it."""
        _check(lib().spec_verify_set_prefix_tail(self._h, int(position)), "spec_verify_set_prefix_tail")

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

    def draws(self, B, k, seed=0, step=0, request_offset=0, stream=None):
        """spec_verify_draws: the run's random draws, [B, k+1, 2] float64."""
        out = torch.empty((B, k + 1, 2), dtype=torch.float64, device=self.device)
        _check(lib().spec_verify_draws(self._h, int(seed), int(step), int(request_offset), int(B),
                                       int(k), _dev_ptr(out), _stream_handle(stream, self.device)),
               "spec_verify_draws")
        return out

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
        out = (_u32 * 6)()
        _check(lib().spec_verify_last_counters(self._h, _stream_handle(stream, self.device), out),
               "spec_verify_last_counters")
        return dict(accept_fp64=out[0], sample_fp64=out[1], sample_fp32=out[2], chunks_fp64=out[3],
                    engine_error=out[4], wait_fail=out[5])


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


# ----------------------------------------------------- vocabulary-parallel --

def shard_layout(B, k, V, dtype, n_shards):
    """Vocabulary split and exchange-block sizes: (bounds [n+1], block1, block2,
    block3 bytes).  Rank r holds tokens [bounds[r], bounds[r+1])."""
    bounds = (_i64 * (n_shards + 1))()
    b1, b2, b3 = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    code = SPEC_BF16 if dtype == torch.bfloat16 else SPEC_F32
    _check(lib().spec_shard_layout(B, k, int(V), code, n_shards, bounds, ctypes.byref(b1),
                                   ctypes.byref(b2), ctypes.byref(b3)), "spec_shard_layout")
    return list(bounds), b1.value, b2.value, b3.value


class ShardRank:
    """One rank of a vocabulary-parallel verification (its own context).  The
    phases follow include/spec_verify.h; `verify_vocab_parallel` runs them with
    torch.distributed collectives, `emulate_vocab_parallel` on one device."""

    def __init__(self, device, rank, n_shards, max_batch, max_k, max_vocab):
        self.ver = SpecVerifier(device, max_batch=max_batch, max_k=max_k, max_vocab=max_vocab,
                                mode="dense")
        self.device = self.ver.device
        self.rank, self.n = int(rank), int(n_shards)

    def _inputs(self, target, draft, tokens, verify_len, temperature, conf, V):
        B, kp1, _ = target.shape
        k = kp1 - 1
        cref, keep = self.ver._conf(conf)
        args = [_dev_ptr(target, None, self.device, "target shard"),
                _dev_ptr(draft, None, self.device, "draft shard"), _dtype_code(target),
                _dev_ptr(tokens, torch.int32, self.device, "tokens"),
                _dev_ptr(verify_len, torch.int32, self.device, "verify_len"),
                _dev_ptr(temperature, torch.float32, self.device, "temperature"), cref, B, k, int(V)]
        return args, keep

    def stats(self, target, draft, tokens, V, block1, verify_len=None, temperature=None, conf=None,
              stream=None):
        args, keep = self._inputs(target, draft, tokens, verify_len, temperature, conf, V)
        _check(lib().spec_shard_stats(self.ver._h, self.rank, self.n, *args, _dev_ptr(block1),
                                      _stream_handle(stream, self.device)), "spec_shard_stats")
        del keep

    def decide(self, blocks1, target, draft, tokens, V, out, block2, verify_len=None,
               temperature=None, conf=None, seed=0, step=0, request_offset=0, stream=None):
        args, keep = self._inputs(target, draft, tokens, verify_len, temperature, conf, V)
        _check(lib().spec_shard_decide(
            self.ver._h, self.rank, self.n, _dev_ptr(blocks1), *args, int(seed), int(step),
            int(request_offset), _dev_ptr(out["accepted"]), _dev_ptr(out["tokens"]),
            _dev_ptr(out.get("p")), _dev_ptr(out.get("q")), _dev_ptr(out["status"]),
            _dev_ptr(block2), _stream_handle(stream, self.device)), "spec_shard_decide")
        del keep

    def locate(self, blocks2, target, draft, tokens, V, votes, verify_len=None, temperature=None,
               conf=None, stream=None):
        args, keep = self._inputs(target, draft, tokens, verify_len, temperature, conf, V)
        _check(lib().spec_shard_locate(self.ver._h, self.rank, self.n, _dev_ptr(blocks2), *args,
                                       _dev_ptr(votes), _stream_handle(stream, self.device)),
               "spec_shard_locate")
        del keep

    def refine_partials(self, target, draft, tokens, V, block3, verify_len=None, temperature=None,
                        conf=None, stream=None):
        args, keep = self._inputs(target, draft, tokens, verify_len, temperature, conf, V)
        _check(lib().spec_shard_refine_partials(self.ver._h, self.rank, self.n, *args, _dev_ptr(block3),
                                                _stream_handle(stream, self.device)),
               "spec_shard_refine_partials")
        del keep

    def refine_locate(self, blocks3, target, draft, tokens, V, votes, verify_len=None,
                      temperature=None, conf=None, stream=None):
        args, keep = self._inputs(target, draft, tokens, verify_len, temperature, conf, V)
        _check(lib().spec_shard_refine_locate(self.ver._h, self.rank, self.n, _dev_ptr(blocks3),
                                              *args, _dev_ptr(votes),
                                              _stream_handle(stream, self.device)),
               "spec_shard_refine_locate")
        del keep

    def refine_finish(self, votes_max, out, stream=None):
        B, kp1 = out["tokens"].shape
        redo = torch.empty(B, dtype=torch.int32, device=self.device)
        _check(lib().spec_shard_refine_finish(self.ver._h, _dev_ptr(votes_max), B, kp1 - 1,
                                              _dev_ptr(out["tokens"]), _dev_ptr(redo),
                                              _stream_handle(stream, self.device)),
               "spec_shard_refine_finish")
        return redo

    def finish(self, votes_max, out, stream=None):
        B, kp1 = out["tokens"].shape
        redo = torch.empty(B, dtype=torch.int32, device=self.device)
        _check(lib().spec_shard_finish(self.ver._h, _dev_ptr(votes_max), B, kp1 - 1,
                                       _dev_ptr(out["tokens"]), _dev_ptr(redo),
                                       _stream_handle(stream, self.device)), "spec_shard_finish")
        return redo

    def close(self):
        self.ver.close()


def _redo_requests(ver, redo, rows_of, tokens, verify_len, temperature, conf, seed, step,
                   request_offset, out):
    """Requests flagged for an fp64 path: verified whole on their gathered rows
    (the single-rank path, same global request index and draws)."""
    idx = torch.nonzero(redo.cpu() == 1).flatten().tolist()
    for i in idx:
        t_full, d_full = rows_of(i)
        sl = slice(i, i + 1)
        c = None
        if conf is not None:
            c = dict(conf, hidden=conf["hidden"][sl])
        o = ver.run(t_full, d_full, tokens[sl].contiguous(),
                    verify_len=None if verify_len is None else verify_len[sl].contiguous(),
                    temperature=None if temperature is None else temperature[sl].contiguous(),
                    conf=c, seed=seed, step=step, request_offset=request_offset + i)
        for key in o:
            out[key][sl] = o[key]
        if "redo" in out:
            out["redo"][sl] = 0
    return idx


def verify_vocab_parallel(rank_obj, target, draft, tokens, V, verify_len=None, temperature=None,
                          conf=None, seed=0, step=0, request_offset=0, group=None, redo_whole=True):
    """Vocabulary-parallel verification on this rank's shard with
    torch.distributed collectives (all ranks call it with the same arguments
    apart from their shards).  Returns the outputs (identical on every rank).

    Every phase always runs, the fp64 refinement included (its kernels skip
    the requests that do not need it), so a step is kernel launches and
    collectives with no host round trip.  The one exception is a request whose
    decision needs rows of every rank (out["redo"] == 1 on the device: an
    accept draw inside the fp32 bound, about one decision in 10^5, or a
    refinement whose support was not settled).  With ``redo_whole`` (the
    default) such requests are found on the host and verified whole from
    gathered rows; ``redo_whole=False`` leaves that to the caller and keeps the
    step free of host synchronisation."""
    import torch.distributed as dist
    n, r = rank_obj.n, rank_obj.rank
    B, kp1, _ = target.shape
    k = kp1 - 1
    bounds, b1, b2, b3 = shard_layout(B, k, V, target.dtype, n)
    dev = rank_obj.device
    blk1 = torch.empty(b1, dtype=torch.uint8, device=dev)
    all1 = torch.empty(n * b1, dtype=torch.uint8, device=dev)
    blk2 = torch.empty(b2, dtype=torch.uint8, device=dev)
    all2 = torch.empty(n * b2, dtype=torch.uint8, device=dev)
    out = rank_obj.ver._outputs(B, k, True)
    votes = torch.empty(B, dtype=torch.int32, device=dev)
    kw = dict(verify_len=verify_len, temperature=temperature, conf=conf)
    rank_obj.stats(target, draft, tokens, V, blk1, **kw)
    dist.all_gather_into_tensor(all1, blk1, group=group)
    rank_obj.decide(all1, target, draft, tokens, V, out, blk2, seed=seed, step=step,
                    request_offset=request_offset, **kw)
    dist.all_gather_into_tensor(all2, blk2, group=group)
    rank_obj.locate(all2, target, draft, tokens, V, votes, **kw)
    dist.all_reduce(votes, op=dist.ReduceOp.MAX, group=group)
    rank_obj.finish(votes, out)
    # the fp64 refinement phase, a no-op for requests that do not need it
    blk3 = torch.empty(b3, dtype=torch.uint8, device=dev)
    all3 = torch.empty(n * b3, dtype=torch.uint8, device=dev)
    rank_obj.refine_partials(target, draft, tokens, V, blk3, **kw)
    dist.all_gather_into_tensor(all3, blk3, group=group)
    rank_obj.refine_locate(all3, target, draft, tokens, V, votes, **kw)
    dist.all_reduce(votes, op=dist.ReduceOp.MAX, group=group)
    redo = rank_obj.refine_finish(votes, out)
    out["redo"] = redo
    if not redo_whole:
        return out

    widths = [bounds[q + 1] - bounds[q] for q in range(n)]
    wmax = max(widths)

    def gather_rows(x):  # [1, rows, w_r] on every rank -> [1, rows, V]
        pad = torch.zeros((1, x.shape[1], wmax), dtype=x.dtype, device=dev)
        pad[:, :, :x.shape[2]] = x
        parts = [torch.empty_like(pad) for _ in range(n)]
        dist.all_gather(parts, pad, group=group)
        return torch.cat([parts[q][:, :, :widths[q]] for q in range(n)], dim=2).contiguous()

    def rows_of(i):
        t_full = gather_rows(target[i:i + 1])
        d_full = gather_rows(draft[i:i + 1]) if draft is not None else None
        return t_full, d_full

    _redo_requests(rank_obj.ver, redo, rows_of, tokens, verify_len, temperature, conf, seed, step,
                   request_offset, out)
    return out


def emulate_vocab_parallel(ranks, target, draft, tokens, verify_len=None, temperature=None,
                           conf=None, seed=0, step=0, request_offset=0):
    """The vocabulary-parallel protocol on ONE device: `ranks` are ShardRank
    objects (their own contexts), each given its slice of the full logits; the
    all-gathers become concatenations and the max a torch.max.  Returns
    (outputs of every rank, final outputs, {"redone", "refined"} request lists,
    the phase-3 votes)."""
    n = len(ranks)
    B, kp1, V = target.shape
    k = kp1 - 1
    bounds, b1, b2, b3 = shard_layout(B, k, V, target.dtype, n)
    dev = ranks[0].device
    shards = [(target[:, :, bounds[r]:bounds[r + 1]].contiguous(),
               None if draft is None else draft[:, :, bounds[r]:bounds[r + 1]].contiguous())
              for r in range(n)]
    kw = dict(verify_len=verify_len, temperature=temperature, conf=conf)
    all1 = torch.empty(n * b1, dtype=torch.uint8, device=dev)
    for r, rk in enumerate(ranks):
        rk.stats(shards[r][0], shards[r][1], tokens, V, all1[r * b1:(r + 1) * b1], **kw)
    all2 = torch.empty(n * b2, dtype=torch.uint8, device=dev)
    outs = []
    for r, rk in enumerate(ranks):
        o = rk.ver._outputs(B, k, True)
        rk.decide(all1, shards[r][0], shards[r][1], tokens, V, o, all2[r * b2:(r + 1) * b2],
                  seed=seed, step=step, request_offset=request_offset, **kw)
        outs.append(o)
    votes = torch.empty((n, B), dtype=torch.int32, device=dev)
    for r, rk in enumerate(ranks):
        rk.locate(all2, shards[r][0], shards[r][1], tokens, V, votes[r], **kw)
    vmax = votes.max(dim=0).values.contiguous()
    redos = [rk.finish(vmax, outs[r]) for r, rk in enumerate(ranks)]
    redo = redos[0]
    refined = []
    if bool((redo == 2).any()):
        refined = torch.nonzero(redo == 2).flatten().tolist()
        all3 = torch.empty(n * b3, dtype=torch.uint8, device=dev)
        for r, rk in enumerate(ranks):
            rk.refine_partials(shards[r][0], shards[r][1], tokens, V, all3[r * b3:(r + 1) * b3], **kw)
        votes3 = torch.empty((n, B), dtype=torch.int32, device=dev)
        for r, rk in enumerate(ranks):
            rk.refine_locate(all3, shards[r][0], shards[r][1], tokens, V, votes3[r], **kw)
        vmax3 = votes3.max(dim=0).values.contiguous()
        redos = [rk.refine_finish(vmax3, outs[r]) for r, rk in enumerate(ranks)]
        redo = redos[0]
    for other in redos[1:]:
        assert torch.equal(other, redo), "ranks disagree on the requests to redo"
    final = {key: v.clone() for key, v in outs[0].items()}

    def rows_of(i):
        return (target[i:i + 1].contiguous(), None if draft is None else draft[i:i + 1].contiguous())

    redone = _redo_requests(ranks[0].ver, redo, rows_of, tokens, verify_len, temperature, conf,
                            seed, step, request_offset, final)
    return outs, final, dict(redone=redone, refined=refined), votes


class LmHeadVerifier:
    """The LM head with verification fused into its epilogue
    (spec_lmhead_*): takes the two models' last hidden states and the shared
    output head instead of logits.  Uses (and must not outlive) ``ver``."""

    def __init__(self, ver: SpecVerifier, max_hidden=4096, cta_pairs=2):
        self.ver = ver
        self.device = ver.device
        self.max_hidden = max_hidden
        h = _vp()
        _check(lib().spec_lmhead_init(ctypes.byref(h), ver._h, int(max_hidden)), "spec_lmhead_init")
        self._h = h
        self.set_cta_pairs(cta_pairs)

    def set_cta_pairs(self, pairs):
        """GEMM tiles: 0 one CTA per tile, 1 CTA pairs (cta_group::2) for both
        GEMMs, 2 (default) CTA pairs for the row-writing GEMM only."""
        _check(lib().spec_lmhead_set_cta_pairs(self._h, int(pairs)), "spec_lmhead_set_cta_pairs")
        self.cta_pairs = int(pairs)

    def close(self):
        if getattr(self, "_h", None):
            lib().spec_lmhead_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def errors(self):
        out = _u32(0)
        _check(lib().spec_lmhead_errors(self._h, ctypes.byref(out)), "spec_lmhead_errors")
        return int(out.value)

    def logits(self, hidden, head, stream=None, out=None):
        """fp32 logits [..., V] = hidden [..., H] (bf16) x head [V, H] (bf16)^T."""
        H = hidden.shape[-1]
        V = head.shape[0]
        rows = hidden.numel() // H
        if tuple(head.shape) != (V, H):
            raise ValueError("head must be [V, H] with H = %d" % H)
        if out is None:
            out = torch.empty(tuple(hidden.shape[:-1]) + (V,), dtype=torch.float32, device=self.device)
        st = lib().spec_lmhead_logits(self._h, _dev_ptr(hidden, torch.bfloat16, self.device, "hidden"),
                                      rows, _dev_ptr(head, torch.bfloat16, self.device, "head"), H, V,
                                      _dev_ptr(out, torch.float32, self.device, "out"),
                                      _stream_handle(stream, self.device))
        _check(st, "spec_lmhead_logits")
        return out

    def verify(self, hidden_target, hidden_draft, head, tokens, verify_len=None, temperature=None,
               conf=None, seed=0, step=0, request_offset=0, stream=None, out=None, redo_whole=True):
        """spec_lmhead_verify; with ``redo_whole`` the (rare) requests it
        flags are verified again on their full rows (spec_lmhead_logits, then
        the single-context path).  Returns the outputs of spec_verify_run,
        plus "redo" [B] int32."""
        B, kp1, H = hidden_target.shape
        k = kp1 - 1
        V = head.shape[0]
        if hidden_draft is not None and tuple(hidden_draft.shape) != (B, k, H):
            raise ValueError("hidden_draft must be [B, k, H] = %s" % ((B, k, H),))
        if tuple(tokens.shape) != (B, k):
            raise ValueError("draft tokens must be [B, k] = %s" % ((B, k),))
        o = self.ver._outputs(B, k, True, out)
        redo = o.get("redo")
        if redo is None:
            redo = o["redo"] = torch.empty(B, dtype=torch.int32, device=self.device)
        cref, _keep = self.ver._conf(conf)
        st = lib().spec_lmhead_verify(
            self._h, _dev_ptr(hidden_target, torch.bfloat16, self.device, "hidden_target"),
            _dev_ptr(hidden_draft, torch.bfloat16, self.device, "hidden_draft"),
            _dev_ptr(head, torch.bfloat16, self.device, "head"), H,
            _dev_ptr(tokens, torch.int32, self.device, "tokens"),
            _dev_ptr(verify_len, torch.int32, self.device, "verify_len"),
            _dev_ptr(temperature, torch.float32, self.device, "temperature"), cref, B, k, V,
            int(seed), int(step), int(request_offset),
            _dev_ptr(o["accepted"], torch.int32), _dev_ptr(o["tokens"], torch.int32),
            _dev_ptr(o.get("p")), _dev_ptr(o.get("q")), _dev_ptr(o["status"]),
            _dev_ptr(redo, torch.int32), _stream_handle(stream, self.device))
        _check(st, "spec_lmhead_verify")
        if redo_whole:
            def rows_of(i):
                t = self.logits(hidden_target[i:i + 1], head, stream)
                d = None if hidden_draft is None else self.logits(hidden_draft[i:i + 1], head, stream)
                return t, d

            keys = {key: o[key] for key in o if key != "redo"}
            _redo_requests(self.ver, redo, rows_of, tokens, verify_len, temperature, conf, seed,
                           step, request_offset, keys)
        return o
