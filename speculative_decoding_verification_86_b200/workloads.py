"""Seeded synthetic inputs for batched speculative-decoding verification.

This module only draws inputs.  It holds none of the verification arithmetic;
both the CUDA path and the CPU oracle are fed from here.

The recipes restate the benchmark configurations (shapes, value
distributions, seeds).  Logits are drawn in fp32 from a seeded
``torch.Generator`` on the requested device and rounded to the storage dtype
(round-to-nearest-even).  Drafted tokens come from the drafter's own
distribution through the Gumbel-max trick, ``argmax(d / T + G)`` with
``G = -log(-log(U))``: a sampling recipe for the *inputs*, independent of the
verification rule.  At temperature 0 the drafter proposes its own argmax.

Every generator returns a dict of tensors on ``device``:
  target  [B, k+1, V]  bf16 or fp32   (row k is the bonus row)
  draft   [B, k, V]    same dtype
  tokens  [B, k]       int32
  verify_len [B] int32 or None,  temperature [B] fp32 or None
  conf    dict(hidden [B, kb, H] bf16, w [H] bf16, bias, threshold) or None
  seed    the Philox seed the verifier is called with (same as the recipe seed)
"""
from __future__ import annotations

import math

import torch

VOCAB_QWEN = 151936
VOCAB_GEMMA = 262144


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def _gumbel_argmax(logits_f32, T, g, device):
    """Index of max(logits / T + Gumbel noise) along the last axis."""
    u = torch.rand(logits_f32.shape, generator=g, device=device, dtype=torch.float32)
    u = u.clamp_(min=1e-20, max=1.0 - 1e-7)
    noise = -torch.log(-torch.log(u))
    return torch.argmax(logits_f32 / T + noise, dim=-1).to(torch.int32)


def _draft_tokens(draft, temperature, g, device, group=16):
    """Drafted tokens from the drafter's logits, ``group`` requests at a time."""
    B, k, V = draft.shape
    out = torch.empty((B, k), dtype=torch.int32, device=device)
    for lo in range(0, B, group):
        hi = min(B, lo + group)
        d = draft[lo:hi].float()
        if temperature is None:
            out[lo:hi] = _gumbel_argmax(d, 1.0, g, device)
            continue
        t = temperature[lo:hi].float().view(-1, 1, 1)
        greedy = torch.argmax(d, dim=-1).to(torch.int32)
        sampled = _gumbel_argmax(d, torch.where(t > 0, t, torch.ones_like(t)), g, device)
        out[lo:hi] = torch.where(temperature[lo:hi].view(-1, 1) > 0, sampled, greedy)
    return out


def _correlated_logits(B, k, V, g, device, dtype, group=16):
    """target ~ N(0, 3^2); draft = 0.8 * target + 0.6 * N(0, 3^2)  (per element)."""
    target = torch.empty((B, k + 1, V), dtype=dtype, device=device)
    draft = torch.empty((B, k, V), dtype=dtype, device=device)
    for lo in range(0, B, group):
        hi = min(B, lo + group)
        t = _normal((hi - lo, k + 1, V), 3.0, g, device)
        n = _normal((hi - lo, k, V), 3.0, g, device)
        target[lo:hi] = t.to(dtype)
        draft[lo:hi] = (0.8 * t[:, :k] + 0.6 * n).to(dtype)
    return target, draft


def tiny(device="cpu", seed=0):
    """B=4, k=5, V=1000 fp32: target ~ N(0, 2^2); draft = target + N(0, 1);
    tokens drafted at T=1; full block verified."""
    B, k, V = 4, 5, 1000
    g = _gen(device, seed)
    t = _normal((B, k + 1, V), 2.0, g, device)
    d = t[:, :k] + _normal((B, k, V), 1.0, g, device)
    tokens = _draft_tokens(d, None, g, device)
    return dict(target=t.contiguous(), draft=d.contiguous(), tokens=tokens, verify_len=None,
                temperature=None, conf=None, seed=seed, name="tiny stochastic B=4 k=5 V=1000 fp32")


def stochastic(device="cpu", seed=1, B=64, k=5, V=VOCAB_QWEN, fixed_len=None,
               dtype=torch.bfloat16):
    """B=64, k=5, V=151936 bf16, correlated logits, T=1, L_i ~ U{2..6}
    (clamped to k by the verifier).  ``fixed_len`` replaces the random lengths."""
    g = _gen(device, seed)
    target, draft = _correlated_logits(B, k, V, g, device, dtype)
    tokens = _draft_tokens(draft, None, g, device)
    if fixed_len is None:
        vlen = torch.randint(2, 7, (B,), generator=g, device=device, dtype=torch.int32)
    else:
        vlen = torch.full((B,), int(fixed_len), dtype=torch.int32, device=device)
    return dict(target=target, draft=draft, tokens=tokens, verify_len=vlen, temperature=None,
                conf=None, seed=seed, name="stochastic B=%d k=%d V=%d" % (B, k, V))


def headline(device="cpu", seed=1, B=256):
    """Stochastic verify at B=256, k=5, V=151936 bf16, every request verifying
    its full block (L_i = 5), T=1; logits as in ``stochastic``."""
    w = stochastic(device, seed=seed, B=B, k=5, V=VOCAB_QWEN, fixed_len=5)
    w["name"] = "stochastic verify B=%d k=5 V=151936 bf16 L=5 T=1" % B
    return w


def greedy(device="cpu", seed=2, B=256, k=5, V=VOCAB_QWEN, agree=0.7):
    """Temperature 0: target ~ N(0, 3^2) bf16; each drafted token equals the
    target row's first maximal index with probability 0.7, else uniform."""
    g = _gen(device, seed)
    target = torch.empty((B, k + 1, V), dtype=torch.bfloat16, device=device)
    for lo in range(0, B, 32):
        hi = min(B, lo + 32)
        target[lo:hi] = _normal((hi - lo, k + 1, V), 3.0, g, device).to(torch.bfloat16)
    first_max = torch.argmax(target[:, :k].float(), dim=-1).to(torch.int32)
    coin = torch.rand((B, k), generator=g, device=device) < agree
    rand_tok = torch.randint(0, V, (B, k), generator=g, device=device, dtype=torch.int32)
    tokens = torch.where(coin, first_max, rand_tok).to(torch.int32)
    temp = torch.zeros(B, dtype=torch.float32, device=device)
    return dict(target=target, draft=None, tokens=tokens, verify_len=None, temperature=temp,
                conf=None, seed=seed, name="greedy B=%d k=%d V=%d" % (B, k, V))


def confidence(device="cpu", seed=3, B=128, k=8, V=VOCAB_GEMMA, H=2560):
    """Verify + confidence head: logits as in ``stochastic`` with k=8,
    V=262144; hidden ~ N(0,1) [B,8,2560] bf16; w ~ N(0, 1/2560) bf16;
    bias 0.5; threshold 0.3."""
    g = _gen(device, seed)
    target, draft = _correlated_logits(B, k, V, g, device, torch.bfloat16, group=8)
    tokens = _draft_tokens(draft, None, g, device, group=8)
    hidden = _normal((B, k, H), 1.0, g, device).to(torch.bfloat16)
    w = _normal((H,), 1.0 / math.sqrt(H), g, device).to(torch.bfloat16)
    conf = dict(hidden=hidden, w=w, bias=0.5, threshold=0.3)
    return dict(target=target, draft=draft, tokens=tokens, verify_len=None, temperature=None,
                conf=conf, seed=seed, name="verify + confidence head B=%d k=%d V=%d" % (B, k, V))


def confidence_batch_budget(device="cpu", seed=3, B=128, k=8, V=VOCAB_GEMMA, H=2560,
                            threshold=0.05, total=None):
    """The confidence workload under a batch-wide verify budget: the same
    logits and head, a low per-request threshold (0.05) and a budget of
    ``total`` positions for the whole batch (default 2 per request)."""
    w = confidence(device, seed, B, k, V, H)
    w["conf"] = dict(w["conf"], threshold=threshold, total=2 * B if total is None else int(total))
    w["name"] = "verify + confidence head, batch budget %d, B=%d k=%d V=%d" % (
        w["conf"]["total"], B, k, V)
    return w


def sweep(device="cpu", seed=4, B=128, k=5, V=VOCAB_QWEN):
    """Load sweep point: correlated bf16 logits, T_i drawn from {0, 0.7, 1.0},
    L_i ~ U{1..5}."""
    g = _gen(device, seed)
    target, draft = _correlated_logits(B, k, V, g, device, torch.bfloat16)
    choice = torch.randint(0, 3, (B,), generator=g, device=device)
    temps = torch.tensor([0.0, 0.7, 1.0], dtype=torch.float32, device=device)[choice]
    vlen = torch.randint(1, 6, (B,), generator=g, device=device, dtype=torch.int32)
    tokens = _draft_tokens(draft, temps, g, device)
    return dict(target=target, draft=draft, tokens=tokens, verify_len=vlen, temperature=temps,
                conf=None, seed=seed, name="load sweep B=%d k=%d V=%d" % (B, k, V))


SWEEP_BATCHES = (1, 8, 32, 128, 512, 1024)

HIDDEN_QWEN3_4B = 2560


def lmhead(device="cpu", seed=5, B=256, k=5, V=VOCAB_QWEN, H=HIDDEN_QWEN3_4B, grid=False,
           temperature=None, verify_len=None, w_levels=1):
    """Inputs of verification fused into the shared LM head: the two models'
    last hidden states and the output head W [V, H] (the drafter shares the
    target's head), all bf16.

    Real-valued recipe: target hidden h_t ~ N(0, 1); drafter hidden
    h_d = 0.8 h_t + 0.6 N(0, 1); W ~ N(0, (3 / sqrt(H))^2), so logits have a
    standard deviation near 3 and the two models' rows are correlated, as in
    the logit recipes.  ``grid=True`` draws instead small integers times powers
    of two (h_t in {-3..3}/4, h_d = clamp(round(0.8 h_t + N(0, 0.6^2)))/4,
    W in {-w_levels..w_levels}/8): every product and every partial sum of h W^T
    is then exact in fp32, so the logits do not depend on summation order.
    Drafted tokens are sampled from the drafter's own logits (fp32 matmul of
    the bf16 inputs) at each request's temperature."""
    g = _gen(device, seed)
    if grid:
        ht = torch.randint(-3, 4, (B, k + 1, H), generator=g, device=device).float()
        hd = torch.clamp(torch.round(0.8 * ht[:, :k] + 0.6 * _normal((B, k, H), 1.0, g, device)), -3, 3)
        W = torch.randint(-w_levels, w_levels + 1, (V, H), generator=g, device=device).float()
        ht, hd, W = ht * 0.25, hd * 0.25, W * 0.125
    else:
        ht = _normal((B, k + 1, H), 1.0, g, device)
        hd = 0.8 * ht[:, :k] + 0.6 * _normal((B, k, H), 1.0, g, device)
        W = _normal((V, H), 3.0 / math.sqrt(H), g, device)
    ht, hd, W = ht.to(torch.bfloat16), hd.to(torch.bfloat16), W.to(torch.bfloat16)
    tokens = torch.empty((B, k), dtype=torch.int32, device=device)
    Wt = W.float().T
    for lo in range(0, B, 16):
        hi = min(B, lo + 16)
        d = hd[lo:hi].float() @ Wt
        t = None if temperature is None else temperature[lo:hi]
        tokens[lo:hi] = _draft_tokens(d, t, g, device)
    return dict(hidden_target=ht.contiguous(), hidden_draft=hd.contiguous(), head=W.contiguous(),
                tokens=tokens, verify_len=verify_len, temperature=temperature, conf=None,
                seed=seed, name="LM-head fused B=%d k=%d V=%d H=%d%s" % (B, k, V, H,
                                                                        " (exact grid)" if grid else ""))


def to_numpy_inputs(w):
    """Host copies in the oracle's formats (bf16 as raw uint16 bits)."""
    import numpy as np

    def logits(t):
        if t is None:
            return None
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()

    def opt(t):
        return None if t is None else t.detach().cpu().contiguous().numpy()

    conf = None
    if w.get("conf") is not None:
        c = w["conf"]
        conf = dict(hidden=c["hidden"].detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16),
                    w=c["w"].detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16),
                    bias=float(c["bias"]), threshold=float(c["threshold"]),
                    total=int(c.get("total", 0)))
    return dict(target=logits(w["target"]), draft=logits(w.get("draft")),
                tokens=opt(w["tokens"]), verify_len=opt(w.get("verify_len")),
                temperature=opt(w.get("temperature")), conf=conf,
                dtype=1 if w["target"].dtype == torch.bfloat16 else 0, seed=int(w["seed"]))
