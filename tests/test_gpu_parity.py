"""CUDA path vs the fp64 CPU oracle, element by element, through the C ABI.

Bar (from the verification rule's tolerances): p_j(x_j) and q_j(x_j) within
1e-5 absolute + 1e-4 relative; accepted lengths and emitted tokens bit-exact,
except for requests holding an accept draw within 1e-6 of p/q (counted; they
must stay below 1e-5 of all decisions); greedy results and confidence budgets
bit-exact.  Inputs are the seeded synthetic workloads, generated on the GPU and
copied to the host for the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_helpers import THREADS, compare, run_oracle  # noqa: F401
from speculative_decoding_verification_86_b200 import binding, build, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["prefix", "dense", "auto"])
def ver(cuda_device, request):
    build.build()
    v = binding.SpecVerifier(cuda_device, max_batch=1024, max_k=16, max_vocab=262144,
                             mode=request.param)
    yield v
    v.close()


def run_gpu(ver, w, uniforms=None, **kw):
    o = ver.run(w["target"], w.get("draft"), w["tokens"], verify_len=w.get("verify_len"),
                temperature=w.get("temperature"), conf=w.get("conf"), seed=w["seed"],
                uniforms=uniforms, **kw)
    torch.cuda.synchronize()
    assert ver.last_counters()["engine_error"] == 0
    return {k: v.cpu().numpy() for k, v in o.items()}


# ------------------------------------------------------------ the configs ----

def test_tiny_fp32(ver):
    w = workloads.tiny("cuda", seed=0)
    compare(run_gpu(ver, w), run_oracle(w))


def test_stochastic_b64(ver):
    w = workloads.stochastic("cuda", seed=1)
    g, o = run_gpu(ver, w), run_oracle(w)
    compare(g, o)
    c = ver.last_counters()
    assert c["sample_fp32"] + c["sample_fp64"] == 64


def test_headline_b256_full_block(ver):
    w = workloads.headline("cuda", seed=1)
    compare(run_gpu(ver, w), run_oracle(w))


def test_greedy_b256(ver):
    w = workloads.greedy("cuda", seed=2)
    o = run_oracle(w)
    g = ver.greedy(w["target"], w["tokens"])
    torch.cuda.synchronize()
    g = {k: v.cpu().numpy() for k, v in g.items()}
    np.testing.assert_array_equal(g["accepted"], o["accepted"])
    np.testing.assert_array_equal(g["tokens"], o["tokens"])
    np.testing.assert_array_equal(g["status"], 0)
    # the same requests through the mixed entry point with T = 0
    g2 = run_gpu(ver, dict(w, draft=None))
    compare(g2, o)
    assert (o["accepted"] < 5).any() and (o["accepted"] == 5).any()


def test_confidence_head_b128(ver):
    w = workloads.confidence("cuda", seed=3)
    o = run_oracle(w)
    compare(run_gpu(ver, w), o)
    c = w["conf"]
    L, surv = ver.conf_budget(c["hidden"], c["w"], c["bias"], c["threshold"])
    torch.cuda.synchronize()
    h = workloads.to_numpy_inputs(w)["conf"]
    oL, osurv, opref = oracle.conf_budget(h["hidden"], h["w"], h["bias"], h["threshold"])
    np.testing.assert_array_equal(L.cpu().numpy(), oL)
    np.testing.assert_array_equal(o["verify_len_used"], oL)
    np.testing.assert_allclose(surv.cpu().numpy(), osurv, rtol=1e-6, atol=1e-7)
    # no prefix product sits within rounding of the threshold
    assert np.min(np.abs(opref - h["threshold"])) > 1e-12


@pytest.mark.parametrize("B", workloads.SWEEP_BATCHES)
def test_load_sweep(ver, B):
    w = workloads.sweep("cuda", seed=4, B=B)
    compare(run_gpu(ver, w), run_oracle(w))


# --------------------------------------------------------- special cases ----

def test_draft_equal_target_accepts_everything(ver):
    w = workloads.stochastic("cuda", seed=5, B=48, k=5, V=20000)
    w["draft"] = w["target"][:, :5].contiguous()
    w["temperature"] = torch.tensor([0.7, 1.0, 1.3] * 16, device="cuda")
    g, o = run_gpu(ver, w), run_oracle(w)
    compare(g, o)
    assert np.array_equal(g["accepted"], np.clip(w["verify_len"].cpu().numpy(), 0, 5))


def test_zero_length_and_zero_block(ver):
    w = workloads.stochastic("cuda", seed=6, B=16, k=4, V=8192 + 8)
    w["verify_len"] = torch.zeros(16, dtype=torch.int32, device="cuda")
    compare(run_gpu(ver, w), run_oracle(w))
    w0 = dict(w, target=w["target"][:, :1].contiguous(), draft=w["draft"][:, :0].contiguous(),
              tokens=w["tokens"][:, :0].contiguous(), verify_len=None)
    g, o = run_gpu(ver, w0), run_oracle(w0)
    compare(g, o)
    assert np.all(g["accepted"] == 0)


@pytest.mark.parametrize("dtype,V", [(torch.bfloat16, 8), (torch.float32, 4), (torch.float32, 4100),
                                     (torch.bfloat16, 262144)])
def test_small_and_ragged_vocabularies(ver, dtype, V):
    B = 8 if V > 100000 else 64
    w = workloads.stochastic("cuda", seed=7, B=B, k=3, V=V, dtype=dtype)
    w["temperature"] = torch.tensor([0.0, 0.5, 1.0, 2.0] * (B // 4), device="cuda")
    compare(run_gpu(ver, w), run_oracle(w))


def test_single_request_max_block(ver):
    w = workloads.stochastic("cuda", seed=8, B=1, k=16, V=151936, fixed_len=16)
    w["draft"] = (0.3 * w["draft"].float() + 0.7 * w["target"][:, :16].float()).to(torch.bfloat16)
    compare(run_gpu(ver, w), run_oracle(w))


def test_errors_reported_per_request(ver):
    w = workloads.stochastic("cuda", seed=9, B=8, k=3, V=4096, fixed_len=3)
    t, d = w["target"], w["draft"]
    t[0, 0, 17] = float("nan")                 # NaN in the first row read
    t[1, 0, 5] = float("inf")                  # +inf
    t[2, 0, :] = float("-inf")                 # whole row masked
    t[3, 0, 9] = float("-inf")                 # one masked token: fine
    d[3, 0, 11] = float("-inf")
    w["tokens"][4, 0] = 4096                   # out of range
    w["tokens"][5, 0] = -3
    temps = torch.ones(8, device="cuda")
    temps[6] = -1.0
    temps[7] = float("nan")
    w["temperature"] = temps
    g, o = run_gpu(ver, w), run_oracle(w)
    compare(g, o)
    assert list(g["status"][:3]) == [2, 2, 2] and g["status"][3] == 0
    assert list(g["status"][4:]) == [1, 1, 4, 4]
    assert np.all(g["accepted"][[0, 1, 2, 4, 5, 6, 7]] == -1)


def test_sampled_request_without_draft_logits_fails(ver):
    w = workloads.greedy("cuda", seed=10, B=4, k=2, V=1024)
    w["temperature"] = torch.tensor([0.0, 1.0, 0.0, 0.5], device="cuda")
    g = run_gpu(ver, w)
    assert list(g["status"]) == [0, 4, 0, 4]


# --------------------------------------- draws on the decision boundaries ----

def _residual_cdf(trow, drow, T, resid):
    z = trow / T
    p = np.exp(z - z.max())
    p /= p.sum()
    if not resid:
        return np.cumsum(p) / p.sum()
    zq = drow / T
    q = np.exp(zq - zq.max())
    q /= q.sum()
    r = np.maximum(0.0, p - q)
    return np.cumsum(r) / r.sum()


def test_draws_on_decision_boundaries_take_the_fp64_paths(ver):
    w = workloads.stochastic("cuda", seed=11, B=64, k=4, V=16384, fixed_len=4)
    B, k = 64, 4
    base = run_oracle(w)
    rho = np.where(base["q_x"] > 0, base["p_x"] / np.maximum(base["q_x"], 1e-300), 2.0)
    rng = np.random.default_rng(0)
    u = rng.random((B, k + 1, 2))
    # accept draws a relative 1e-9 either side of p/q (inside every fp32 bound)
    for i in range(B):
        for j in range(k):
            if base["p_x"][i, j] >= 0 and rho[i, j] < 1:
                u[i, j, 0] = rho[i, j] * (1 + (1e-9 if (i + j) % 2 else -1e-9))
    first = oracle.verify(*[workloads.to_numpy_inputs(w)[x] for x in ("target", "draft", "tokens")],
                          dtype=oracle.DTYPE_BF16, verify_len=w["verify_len"].cpu().numpy(), u_override=u)
    # sample draws a relative 1e-12 from a cell edge of the row each chain stops at
    h = workloads.to_numpy_inputs(w)
    tv = torch.from_numpy(h["target"].view(np.int16)).view(torch.bfloat16).double().numpy()
    dv = torch.from_numpy(h["draft"].view(np.int16)).view(torch.bfloat16).double().numpy()
    for i in range(B):
        n = first["accepted"][i]
        cdf = _residual_cdf(tv[i, n], dv[i, n] if n < k else None, 1.0, n < k)
        t = int(np.argmax(np.diff(np.concatenate([[0.0], cdf]))))  # widest cell
        u[i, n, 1] = min(cdf[t] * (1 + (1e-12 if i % 2 else -1e-12)), 1 - 2 ** -53)
    o = run_oracle(w, u_override=u)
    g = run_gpu(ver, w, uniforms=torch.from_numpy(u).cuda())
    compare(g, o, strict=True)
    c = ver.last_counters()
    assert c["accept_fp64"] > 0 and c["sample_fp64"] > 0


@pytest.mark.parametrize("u_floor,tok_floor", [(0.6, 38), (0.01, 0)])
def test_residual_floor_and_fallback_through_refinement(ver, u_floor, tok_floor):
    V = 64
    t = torch.zeros((2, 2, V), dtype=torch.float32)
    d = torch.zeros((2, 1, V), dtype=torch.float32)
    d[0, 0, 0] = 1e-13         # p and q differ by ~1e-14: residual under the floor
    t[1, 0, 40:] = float("-inf")  # request 1: x = 50 is masked in the target -> rejected
    w = dict(target=t.cuda(), draft=d.cuda(), tokens=torch.tensor([[0], [50]], dtype=torch.int32).cuda(),
             verify_len=None, temperature=None, conf=None, seed=0)
    u = np.array([[[1 - 2.0 ** -50, u_floor], [0.5, 0.5]],
                  [[0.5, 1.0], [0.5, 0.5]]])            # u' = 1: past every cell
    o = run_oracle(w, u_override=u)
    g = run_gpu(ver, w, uniforms=torch.from_numpy(u).cuda())
    compare(g, o, strict=True)
    # floor: drawn from p (uniform over 64).  At u' = 0.01 the residual, which
    # has no weight on token 0 (q_0 > p_0), would give token 1 instead.
    assert o["tokens"][0, 0] == tok_floor
    assert o["tokens"][1, 0] == 39       # fallback: last index with positive residual


# ------------------------------------------------------ API-level checks ----

def test_deterministic_and_request_offset(ver):
    w = workloads.stochastic("cuda", seed=12, B=32, k=5, V=32768)
    a = run_gpu(ver, w)
    b = run_gpu(ver, w)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])
    half = {key: (v[16:].contiguous() if isinstance(v, torch.Tensor) and v.dim() and v.shape[0] == 32 else v)
            for key, v in w.items()}
    h = ver.run(half["target"], half["draft"], half["tokens"], verify_len=half["verify_len"],
                seed=w["seed"], request_offset=16)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(h["tokens"].cpu().numpy(), a["tokens"][16:])
    np.testing.assert_array_equal(h["accepted"].cpu().numpy(), a["accepted"][16:])


def test_host_buffer_entry_point(ver):
    w = workloads.stochastic("cuda", seed=13, B=16, k=5, V=151936)
    a = run_gpu(ver, w)
    hw = {k: (v.cpu().pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    o = ver.run_host(hw["target"], hw["draft"], hw["tokens"], verify_len=hw["verify_len"], seed=w["seed"])
    np.testing.assert_array_equal(o["tokens"].numpy(), a["tokens"])
    np.testing.assert_array_equal(o["accepted"].numpy(), a["accepted"])
    np.testing.assert_array_equal(o["p"].numpy(), a["p"])


def test_empty_batch(ver):
    t = torch.zeros((0, 3, 64), dtype=torch.bfloat16, device="cuda")
    o = ver.run(t, torch.zeros((0, 2, 64), dtype=torch.bfloat16, device="cuda"),
                torch.zeros((0, 2), dtype=torch.int32, device="cuda"))
    assert o["accepted"].numel() == 0


def test_unsupported_layouts_are_refused(ver):
    t = torch.zeros((1, 2, 12), dtype=torch.bfloat16, device="cuda")    # 24-byte rows
    with pytest.raises(binding.SpecVerifyError) as e:
        ver.run(t, t[:, :1].contiguous(), torch.zeros((1, 1), dtype=torch.int32, device="cuda"))
    assert e.value.status == binding.SPEC_ERR_UNSUPPORTED


def test_ex2_error_bound_holds_on_this_device(cuda_device):
    build.build()
    measured, bound = binding.selfcheck_ex2(cuda_device.index, -126.0, 0.0)
    assert 0 < measured <= bound, (measured, bound)


# ------------------------------------------------------ batch-wide budget ----

def _conf_case(B, kb, H, seed, bias=0.5, same_rows=False):
    g = torch.Generator(device="cuda").manual_seed(seed)
    hidden = torch.randn(B, kb, H, generator=g, device="cuda").to(torch.bfloat16)
    if same_rows:
        hidden[:] = hidden[0]
    w = (torch.randn(H, generator=g, device="cuda") * (2.0 / H ** 0.5)).to(torch.bfloat16)
    return hidden, w


def _oracle_lengths(hidden, w, bias, tau, vlen, k, total):
    hb = hidden.cpu().view(torch.int16).numpy().view(np.uint16)
    wb = w.cpu().view(torch.int16).numpy().view(np.uint16)
    static, _, pref = oracle.conf_budget(hb, wb, bias, tau)
    lim = np.full(len(static), k) if vlen is None else np.clip(vlen.cpu().numpy(), 0, k)
    cap = np.minimum(lim, static).astype(np.int32)
    if total <= 0:
        return cap, pref, cap
    return oracle.budget_topn(pref, cap, total), pref, cap


def _assert_decidable(L, pref, cap):
    """Kept and dropped survivals are apart by more than rounding (so the
    fp64 values of the two sides cannot order them differently)."""
    kept = [pref[i, j] for i in range(len(L)) for j in range(L[i])]
    drop = [pref[i, j] for i in range(len(L)) for j in range(L[i], cap[i])]
    if kept and drop:
        assert min(kept) - max(drop) > 1e-12 * max(drop)


@pytest.mark.parametrize("B,kb,H,with_vlen", [(128, 8, 2560, False), (77, 5, 300, True),
                                              (1000, 16, 64, True)])
def test_batch_budget_lengths(ver, B, kb, H, with_vlen):
    hidden, w = _conf_case(B, kb, H, seed=B)
    k = kb
    g = torch.Generator(device="cuda").manual_seed(B + 1)
    vlen = torch.randint(-1, k + 2, (B,), generator=g, device="cuda", dtype=torch.int32) if with_vlen else None
    bias, tau = 0.5, 0.02
    _, pref0, cap0 = _oracle_lengths(hidden, w, bias, tau, vlen, k, 0)
    M = int(cap0.sum())
    assert M > 2
    for total in (0, 1, 2, M // 3, M - 1, M, M + 5, 10 ** 9):
        conf = dict(hidden=hidden, w=w, bias=bias, threshold=tau, total=total)
        L, surv = ver.lengths(conf, k, verify_len=vlen, with_survival=True)
        torch.cuda.synchronize()
        oL, pref, cap = _oracle_lengths(hidden, w, bias, tau, vlen, k, total)
        np.testing.assert_array_equal(L.cpu().numpy(), oL, err_msg="total=%d" % total)
        assert int(oL.sum()) == (M if total <= 0 else min(total, M))
        _assert_decidable(oL, pref, cap)


def test_batch_budget_ties_go_to_lower_request_then_position(ver):
    B, kb, H = 40, 6, 128
    # identical requests: equal survivals across requests
    hidden, w = _conf_case(B, kb, H, seed=5, same_rows=True)
    for total in (1, 7, 59, 100, 239):
        conf = dict(hidden=hidden, w=w, bias=0.5, threshold=0.0, total=total)
        L, _ = ver.lengths(conf, kb)
        torch.cuda.synchronize()
        oL, _, _ = _oracle_lengths(hidden, w, 0.5, 0.0, None, kb, total)
        np.testing.assert_array_equal(L.cpu().numpy(), oL, err_msg="total=%d" % total)
    # survival exactly 1 everywhere: every position ties; requests fill in order
    for total in (1, 13, 100):
        conf = dict(hidden=hidden, w=w, bias=100.0, threshold=0.5, total=total)
        L, _ = ver.lengths(conf, kb)
        torch.cuda.synchronize()
        expect = np.clip(total - kb * np.arange(B), 0, kb)
        np.testing.assert_array_equal(L.cpu().numpy(), expect)


def test_batch_budget_through_verification(ver):
    w = workloads.confidence_batch_budget("cuda", seed=3)
    o = run_oracle(w)
    g = run_gpu(ver, w)
    compare(g, o)
    total = w["conf"]["total"]
    assert int(o["verify_len_used"].sum()) == total
    L, _ = ver.lengths(w["conf"], w["tokens"].shape[1])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(L.cpu().numpy(), o["verify_len_used"])
    # the host-buffer entry point carries the budget too
    h = {key: (v.cpu() if isinstance(v, torch.Tensor) else v) for key, v in w.items()}
    hc = dict(w["conf"], hidden=w["conf"]["hidden"].cpu(), w=w["conf"]["w"].cpu())
    gh = ver.run_host(h["target"], h["draft"], h["tokens"], conf=hc, seed=w["seed"])
    np.testing.assert_array_equal(gh["accepted"].numpy(), g["accepted"])
    np.testing.assert_array_equal(gh["tokens"].numpy(), g["tokens"])


# ------------------------------------------------------ hand-worked cases ----

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_hand_worked_golden_cases(ver, dtype):
    """The hand-derived cases (several with a draw exactly on a decision edge)
    through the C ABI, in both logit formats."""
    import golden_cases
    for c in golden_cases.load():
        dev = ver.device
        w = dict(target=torch.from_numpy(c["target"]).to(dev, dtype),
                 draft=torch.from_numpy(c["draft"]).to(dev, dtype),
                 tokens=torch.from_numpy(c["tokens"]).to(dev),
                 verify_len=torch.from_numpy(c["verify_len"]).to(dev),
                 temperature=torch.from_numpy(c["temperature"]).to(dev), seed=0)
        g = run_gpu(ver, w, uniforms=torch.from_numpy(c["u"]).to(dev))
        assert g["status"][0] == 0, c["name"]
        assert g["accepted"][0] == c["n"], c["name"]
        assert g["tokens"][0].tolist() == c["out_tokens"].tolist(), c["name"]


# --------------------------------------------------------- maximum sizes ----

@pytest.mark.parametrize("dtype,V", [(torch.bfloat16, 2097152), (torch.float32, 1048576)])
def test_maximum_block_and_vocabulary(cuda_device, dtype, V):
    """k = 16 (the largest block) and the largest vocabulary a context takes
    (2^21 logits; fp32 at half that to bound memory), B = 2, against the oracle."""
    build.build()
    g = torch.Generator(device="cuda").manual_seed(17)
    B, k = 2, 16
    target = (torch.randn(B, k + 1, V, generator=g, device="cuda") * 2.5).to(dtype)
    draft = (0.9 * target[:, :k].float() + 0.5 * torch.randn(B, k, V, generator=g, device="cuda")).to(dtype)
    # drafted tokens: the target's arg-max (accepted often, so the chain runs long)
    tokens = target[:, :k].float().argmax(dim=2).to(torch.int32)
    w = dict(target=target, draft=draft, tokens=tokens, verify_len=None, temperature=None, conf=None,
             seed=21)
    v = binding.SpecVerifier(cuda_device, max_batch=B, max_k=k, max_vocab=2097152)
    try:
        for mode in ("prefix", "dense"):
            v.set_mode(mode)
            compare(run_gpu(v, w), run_oracle(w))
    finally:
        v.close()


def test_masked_logits_at_scale(ver):
    """About 1 % of the logits of every row masked (-inf) in target and draft
    rows: the statistics and sample passes meet masked arguments in most
    segments (their unclamped fast paths must fall back to the clamped ones)."""
    w = workloads.stochastic("cuda", seed=12, B=32)
    g = torch.Generator(device="cuda").manual_seed(12)
    for key in ("target", "draft"):
        t = w[key]
        mask = torch.rand(t.shape, generator=g, device="cuda") < 0.01
        t.masked_fill_(mask, float("-inf"))
    compare(run_gpu(ver, w), run_oracle(w))


def test_extreme_temperatures(ver):
    """Temperatures from 1e-3 (nearly greedy: c = log2(e)/T ~ 1443, every
    argument but the top few huge) to 100 (nearly uniform) on full-size rows."""
    w = workloads.stochastic("cuda", seed=13, B=24)
    temps = torch.tensor([1e-3, 5e-3, 0.02, 0.1, 3.0, 10.0, 30.0, 100.0] * 3, device="cuda")
    w["temperature"] = temps.contiguous()
    compare(run_gpu(ver, w), run_oracle(w))


def test_fp32_full_vocabulary_mixed_temperatures(ver):
    """fp32 logits over the full 151936-token vocabulary with greedy and sampled
    requests mixed in one batch."""
    w = workloads.stochastic("cuda", seed=14, B=48, V=151936, dtype=torch.float32)
    w["temperature"] = torch.tensor([0.0, 0.6, 1.0, 1.7] * 12, device="cuda")
    compare(run_gpu(ver, w), run_oracle(w))
