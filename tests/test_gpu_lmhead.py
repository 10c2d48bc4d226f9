"""The LM head with verification fused into its epilogue (tcgen05 GEMM, one
CTA per tile and CTA pairs), through the C ABI, against the fp64 oracle.

Logits: on integer grids (every product and partial sum exact in fp32) the
GEMM's fp32 logits must equal the oracle's fp64 ones bit for bit; on
real-valued inputs they must stay within the fp32 dot-product bound.
Verification: on grid inputs the fused path must meet the verification bar
against the oracle's verification of the exact logits (tokens and lengths
bit-exact apart from accept draws within 1e-6 of p/q, p and q within
1e-5 + 1e-4 relative); on real-valued inputs it must give the decisions of
the unfused path (the same GEMM writing logits, then the verifier).
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_86_b200 import binding, build, workloads

from test_gpu_parity import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=[0, 1, 2], ids=["cta", "cta_pairs", "default"])
def lm(cuda_device, request):
    build.build()
    v = binding.SpecVerifier(cuda_device, max_batch=256, max_k=8, max_vocab=151936, mode="dense")
    h = binding.LmHeadVerifier(v, max_hidden=2560, cta_pairs=request.param)
    yield v, h
    assert h.errors() == 0
    h.close()
    v.close()


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _np(t):
    return None if t is None else t.detach().cpu().contiguous().numpy()


def _grid(shape, lo, hi, scale, g):
    return (torch.randint(lo, hi + 1, shape, generator=g, device="cuda").float() * scale).to(torch.bfloat16)


@pytest.mark.parametrize("rows,H,V", [(16, 256, 2000), (300, 200, 20000), (129, 64, 4100), (5, 8, 4100)])
def test_logits_exact_grid(lm, rows, H, V):
    _, h = lm
    g = torch.Generator(device="cuda").manual_seed(rows + H)
    x = _grid((rows, H), -3, 3, 0.25, g)
    w = _grid((V, H), -3, 3, 0.125, g)
    got = h.logits(x, w)
    torch.cuda.synchronize()
    want = oracle.lmhead_logits(_bits(x), _bits(w))
    np.testing.assert_array_equal(got.cpu().numpy().astype(np.float64), want)


def test_logits_exact_grid_full_head_sampled_rows(lm):
    """B(2k+1) = 2816 rows x the full 151936-token head, H = 2560: rows sampled
    across the M tiles (every column of each)."""
    _, h = lm
    g = torch.Generator(device="cuda").manual_seed(7)
    x = _grid((2816, 2560), -3, 3, 0.25, g)
    w = _grid((151936, 2560), -1, 1, 0.125, g)
    got = h.logits(x, w)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 1000, 2047, 2815]
    want = oracle.lmhead_logits(_bits(x[rows]), _bits(w))
    np.testing.assert_array_equal(got[rows].cpu().numpy().astype(np.float64), want)


def test_logits_real_valued_within_fp32_bound(lm):
    _, h = lm
    g = torch.Generator(device="cuda").manual_seed(11)
    rows, H, V = 200, 2560, 20000
    x = torch.randn((rows, H), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((V, H), generator=g, device="cuda") / 16).to(torch.bfloat16)
    got = h.logits(x, w)
    torch.cuda.synchronize()
    xb, wb = _bits(x), _bits(w)
    want = oracle.lmhead_logits(xb, wb)
    mag = np.abs(oracle.bf16_to_f64(xb)) @ np.abs(oracle.bf16_to_f64(wb)).T
    err = np.abs(got.cpu().numpy().astype(np.float64) - want)
    # fp32 accumulation of H products: within (H + 2) units of 2^-23 of sum |h w|
    assert np.all(err <= (H + 2) * 2.0 ** -23 * mag)
    assert err.max() > 0  # the bound is exercised, not vacuous


def _run_fused(h, w, **kw):
    o = h.verify(w["hidden_target"], w["hidden_draft"], w["head"], w["tokens"],
                 verify_len=w.get("verify_len"), temperature=w.get("temperature"), seed=w["seed"], **kw)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in o.items()}


def _run_oracle(w, rows=None, request_offset=0):
    sl = slice(None) if rows is None else rows
    return oracle.verify_lmhead(_bits(w["hidden_target"][sl]), _bits(w["hidden_draft"][sl]),
                                _bits(w["head"]), _np(w["tokens"][sl]),
                                verify_len=_np(None if w.get("verify_len") is None else w["verify_len"][sl]),
                                temperature=_np(None if w.get("temperature") is None else w["temperature"][sl]),
                                seed=w["seed"], request_offset=request_offset, threads=16)


def _temps(B, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    choice = torch.randint(0, 3, (B,), generator=g, device="cuda")
    return torch.tensor([0.0, 0.7, 1.0], device="cuda")[choice].contiguous()


@pytest.mark.parametrize("B,k,V,H,mixed", [
    (4, 3, 2000, 256, False),      # one M tile, one part, ragged N tile
    (40, 3, 20000, 200, True),     # two M tiles per model, 5 parts over 2 segments, ragged K
    (24, 5, 151936, 256, True),    # the full head's vocabulary
    (8, 0, 4096, 128, False),      # k = 0: the bonus row only
    (6, 2, 4100, 64, True),        # V % 16 = 4: a partial 16-column batch at every row's end
    (1, 3, 2000, 8, False),        # B = 1, H = 8: one k-block, mostly zero-filled
])
def test_fused_verify_grid_vs_oracle(lm, B, k, V, H, mixed):
    _, h = lm
    temps = _temps(B, B + V) if mixed else None
    vlen = None
    if mixed:
        g = torch.Generator(device="cuda").manual_seed(3)
        vlen = torch.randint(0, k + 1, (B,), generator=g, device="cuda", dtype=torch.int32)
    w = workloads.lmhead("cuda", seed=B + k, B=B, k=k, V=V, H=H, grid=True, temperature=temps,
                         verify_len=vlen, w_levels=3)
    g_out = _run_fused(h, w)
    o = _run_oracle(w)
    compare(g_out, o)
    assert (g_out["redo"] == 0).all() or (g_out["redo"] == 1).sum() <= 1


def test_fused_every_request_continues_past_position_0(lm):
    """The drafter's hidden states are the target's: p = q at every position,
    so every sampled request accepts its whole block, and greedy requests
    whose drafted tokens are the target's lowest arg-max accept too: the second
    statistics pass gets every remaining row (its largest row count)."""
    _, h = lm
    B, k, V, H = 24, 4, 20000, 128
    temps = _temps(B, 11)
    w = workloads.lmhead("cuda", seed=12, B=B, k=k, V=V, H=H, grid=True, temperature=temps)
    w["hidden_draft"] = w["hidden_target"][:, :k].contiguous()
    t = w["hidden_target"][:, :k].float() @ w["head"].float().T  # exact on the grid
    greedy = temps == 0
    w["tokens"] = torch.where(greedy[:, None], t.argmax(dim=2).to(torch.int32), w["tokens"]).contiguous()
    g_out = _run_fused(h, w)
    o = _run_oracle(w)
    compare(g_out, o)
    assert (g_out["accepted"] == k).all()


def test_fused_every_request_stops_at_position_0(lm):
    """Greedy requests whose drafted tokens are never the target's arg-max:
    every request stops at position 0, and the second statistics pass runs
    with no rows."""
    _, h = lm
    B, k, V, H = 16, 3, 4100, 64
    w = workloads.lmhead("cuda", seed=13, B=B, k=k, V=V, H=H, grid=True,
                         temperature=torch.zeros(B, device="cuda"))
    t = w["hidden_target"][:, :k].float() @ w["head"].float().T  # exact on the grid
    top = t.argmax(dim=2)
    w["tokens"] = ((top + 1) % V).to(torch.int32).contiguous()
    g_out = _run_fused(h, w)
    o = _run_oracle(w)
    compare(g_out, o)
    assert (g_out["accepted"] == 0).all()


def test_fused_matches_unfused_real_valued(lm):
    """Real-valued inputs: the fused path decides as the verifier does on the
    same GEMM's logits (decisions are certified, so summation order inside the
    statistics cannot change them)."""
    v, h = lm
    B, k = 64, 5
    w = workloads.lmhead("cuda", seed=21, B=B, k=k, temperature=_temps(B, 5))
    fused = _run_fused(h, w)
    t = h.logits(w["hidden_target"], w["head"])
    d = h.logits(w["hidden_draft"], w["head"])
    o = v.run(t, d, w["tokens"], temperature=w["temperature"], seed=w["seed"])
    torch.cuda.synchronize()
    o = {key: val.cpu().numpy() for key, val in o.items()}
    for key in ("accepted", "tokens", "status"):
        np.testing.assert_array_equal(fused[key], o[key])
    for key in ("p", "q"):
        np.testing.assert_allclose(fused[key], o[key], rtol=2e-6, atol=1e-9)


def test_fused_full_size_grid(lm):
    """The bench's shape (B=256, k=5, V=151936, H=2560) on the exact grid:
    every request against the unfused path, sampled requests against the
    oracle (with their global request index, so the draws match)."""
    v, h = lm
    B, k = 256, 5
    w = workloads.lmhead("cuda", seed=5, B=B, k=k, grid=True)
    fused = _run_fused(h, w)
    t = h.logits(w["hidden_target"], w["head"])
    d = h.logits(w["hidden_draft"], w["head"])
    o = v.run(t, d, w["tokens"], seed=w["seed"])
    torch.cuda.synchronize()
    o = {key: val.cpu().numpy() for key, val in o.items()}
    for key in ("accepted", "tokens", "status"):
        np.testing.assert_array_equal(fused[key], o[key])
    for i in (0, 129, 255):
        oi = _run_oracle(w, rows=slice(i, i + 1), request_offset=i)
        gi = {key: val[i:i + 1] for key, val in fused.items()}
        compare(gi, oi)
    assert 0 < fused["accepted"].mean() < k


def test_redo_recomputes_the_same_outputs(lm):
    """The whole-request redo (the rare exit of the fused path) gives the
    outputs the fused pass gave, for requests forced through it."""
    v, h = lm
    B, k = 16, 4
    w = workloads.lmhead("cuda", seed=9, B=B, k=k, V=20000, H=512, grid=True, w_levels=3,
                         temperature=_temps(B, 9))
    o = h.verify(w["hidden_target"], w["hidden_draft"], w["head"], w["tokens"],
                 temperature=w["temperature"], seed=w["seed"], redo_whole=False)
    torch.cuda.synchronize()
    first = {key: val.clone() for key, val in o.items()}
    redo = torch.zeros(B, dtype=torch.int32)
    redo[[0, 5, 11]] = 1

    def rows_of(i):
        return (h.logits(w["hidden_target"][i:i + 1], w["head"]),
                h.logits(w["hidden_draft"][i:i + 1], w["head"]))

    keys = {key: o[key] for key in o if key != "redo"}
    for key in keys:
        keys[key][[0, 5, 11]] = -7  # overwritten by the redo
    binding._redo_requests(v, redo, rows_of, w["tokens"], None, w["temperature"], None, w["seed"],
                           0, 0, keys)
    torch.cuda.synchronize()
    for key in keys:
        torch.testing.assert_close(keys[key], first[key], rtol=2e-6, atol=1e-9)


def test_fused_greedy_without_drafter_hidden_states(lm):
    """Temperature 0 everywhere: the drafter's hidden states are not needed
    (None), the chain compares arg-maxes of the head's fp32 logits."""
    _, h = lm
    B, k = 12, 4
    temps = torch.zeros(B, device="cuda")
    w = workloads.lmhead("cuda", seed=31, B=B, k=k, V=20000, H=256, grid=True, w_levels=3,
                         temperature=temps)
    w = dict(w, hidden_draft=None)
    o = h.verify(w["hidden_target"], None, w["head"], w["tokens"], temperature=temps, seed=w["seed"])
    torch.cuda.synchronize()
    g = {key: val.cpu().numpy() for key, val in o.items()}
    want = oracle.verify_lmhead(_bits(w["hidden_target"]), None, _bits(w["head"]), _np(w["tokens"]),
                                temperature=_np(temps), seed=w["seed"])
    np.testing.assert_array_equal(g["accepted"], want["accepted"])
    np.testing.assert_array_equal(g["tokens"], want["tokens"])
    np.testing.assert_array_equal(g["status"], 0)


def test_fused_with_confidence_head(lm):
    """The confidence head truncates the verified lengths before the chain,
    as in spec_verify_run."""
    _, h = lm
    B, k, Hc = 16, 5, 512
    w = workloads.lmhead("cuda", seed=41, B=B, k=k, V=20000, H=256, grid=True, w_levels=3)
    g = torch.Generator(device="cuda").manual_seed(41)
    conf = dict(hidden=torch.randn((B, k, Hc), generator=g, device="cuda").to(torch.bfloat16),
                w=(torch.randn(Hc, generator=g, device="cuda") / Hc ** 0.5).to(torch.bfloat16),
                bias=0.5, threshold=0.3)
    o = h.verify(w["hidden_target"], w["hidden_draft"], w["head"], w["tokens"], conf=conf,
                 seed=w["seed"])
    torch.cuda.synchronize()
    gout = {key: val.cpu().numpy() for key, val in o.items()}
    oc = dict(hidden=_bits(conf["hidden"]), w=_bits(conf["w"]), bias=0.5, threshold=0.3)
    want = oracle.verify_lmhead(_bits(w["hidden_target"]), _bits(w["hidden_draft"]), _bits(w["head"]),
                                _np(w["tokens"]), conf=oc, seed=w["seed"])
    compare(gout, want)
    assert (want["verify_len_used"] < k).any()  # the head cut some blocks


def test_fused_other_model_shapes(cuda_device):
    """Another model family's shapes: V=262144 (a Gemma-size vocabulary),
    H=3840, k=8 drafted positions, mixed temperatures and lengths, on the
    exact grid: fused against the unfused path for every request and against
    the oracle for sampled requests."""
    build.build()
    B, k, V, H = 32, 8, 262144, 3840
    v = binding.SpecVerifier(cuda_device, max_batch=B, max_k=k, max_vocab=V, mode="dense")
    h = binding.LmHeadVerifier(v, max_hidden=H)
    try:
        g = torch.Generator(device="cuda").manual_seed(8)
        vlen = torch.randint(0, k + 1, (B,), generator=g, device="cuda", dtype=torch.int32)
        temps = _temps(B, 8)
        w = workloads.lmhead("cuda", seed=8, B=B, k=k, V=V, H=H, grid=True, temperature=temps,
                             verify_len=vlen)
        fused = _run_fused(h, w)
        t = h.logits(w["hidden_target"], w["head"])
        d = h.logits(w["hidden_draft"], w["head"])
        o = v.run(t, d, w["tokens"], verify_len=vlen, temperature=temps, seed=w["seed"])
        torch.cuda.synchronize()
        o = {key: val.cpu().numpy() for key, val in o.items()}
        for key in ("accepted", "tokens", "status"):
            np.testing.assert_array_equal(fused[key], o[key])
        for i in (0, 17, 31):
            oi = _run_oracle(w, rows=slice(i, i + 1), request_offset=i)
            compare({key: val[i:i + 1] for key, val in fused.items()}, oi)
        assert h.errors() == 0
    finally:
        h.close()
        v.close()


@pytest.mark.parametrize("B,k,V,H,status", [
    (2, 2, 2000, 12, "SPEC_ERR_UNSUPPORTED"),   # H % 8 != 0: a row is not a whole number of 16-byte units
    (2, 2, 2002, 64, "SPEC_ERR_UNSUPPORTED"),   # V % 4 != 0
    (2, 2, 2000, 2568, "SPEC_ERR_INVALID_ARG"),  # H above the context's max_hidden
    (257, 1, 2000, 64, "SPEC_ERR_INVALID_ARG"),  # B above the verifier's max_batch
    (2, 9, 2000, 64, "SPEC_ERR_INVALID_ARG"),    # k above the verifier's max_k
])
def test_unsupported_shapes_are_refused(lm, B, k, V, H, status):
    """Refused before any launch, and the context stays usable afterwards."""
    _, h = lm
    w = workloads.lmhead("cuda", seed=1, B=B, k=k, V=V, H=H, grid=True)
    with pytest.raises(binding.SpecVerifyError) as e:
        _run_fused(h, w)
    assert e.value.status == getattr(binding, status)
    ok = workloads.lmhead("cuda", seed=2, B=4, k=3, V=2000, H=256, grid=True)
    compare(_run_fused(h, ok), _run_oracle(ok))
