"""The seeded input generators produce the recipes the design notes state:
shapes, dtypes, value distributions, length mixes and determinism per seed.
Small vocabularies keep the draws cheap; every recipe is per element or per
request, so its statistics do not depend on V or B."""
import math

import numpy as np
import pytest
import torch

from speculative_decoding_verification_86_b200 import workloads as W


def _f(t):
    return t.float().numpy().astype(np.float64)


def test_correlated_logits_recipe():
    w = W.stochastic("cpu", seed=1, B=32, k=5, V=4096)
    t, d = w["target"], w["draft"]
    assert t.dtype == torch.bfloat16 and tuple(t.shape) == (32, 6, 4096)
    assert d.dtype == torch.bfloat16 and tuple(d.shape) == (32, 5, 4096)
    tf, df = _f(t), _f(d)
    # target ~ N(0, 3^2); draft = 0.8 target + 0.6 N(0, 3^2): also std 3, correlation 0.8
    assert abs(tf.std() - 3.0) < 0.03 and abs(tf.mean()) < 0.03
    assert abs(df.std() - 3.0) < 0.03
    corr = np.corrcoef(tf[:, :5].ravel(), df.ravel())[0, 1]
    assert abs(corr - 0.8) < 0.01
    vl = w["verify_len"].numpy()
    assert vl.min() >= 2 and vl.max() <= 6 and set(vl.tolist()) == {2, 3, 4, 5, 6}
    tok = w["tokens"].numpy()
    assert tok.dtype == np.int32 and tok.min() >= 0 and tok.max() < 4096
    assert w["temperature"] is None


def test_drafted_tokens_follow_the_drafters_softmax():
    """Gumbel-max at T = 1: the drafted token is distributed as softmax(draft row)."""
    V, n = 8, 20000
    w = W.stochastic("cpu", seed=7, B=n, k=1, V=V)
    d = _f(w["draft"][:, 0])
    p = np.exp(d - d.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    expected = p.sum(axis=0)            # expected count per token id
    counts = np.bincount(w["tokens"][:, 0].numpy(), minlength=V)
    chi2 = float(((counts - expected) ** 2 / expected).sum())
    assert chi2 < 30.0                  # 7 degrees of freedom: p ~ 1e-4


def test_headline_verifies_every_position():
    w = W.headline("cpu", seed=1, B=4)
    assert tuple(w["target"].shape) == (4, 6, W.VOCAB_QWEN)
    assert (w["verify_len"] == 5).all() and w["temperature"] is None
    assert "B=4 k=5 V=151936" in w["name"]


def test_greedy_recipe():
    B, k, V = 2000, 5, 512
    w = W.greedy("cpu", seed=2, B=B, k=k, V=V)
    assert w["draft"] is None and (w["temperature"] == 0).all()
    first_max = torch.argmax(w["target"][:, :k].float(), dim=-1)
    agree = (w["tokens"] == first_max).double().mean().item()
    want = 0.7 + 0.3 / V
    assert abs(agree - want) < 4 * math.sqrt(want * (1 - want) / (B * k))


def test_confidence_recipe_length_statistics():
    """hidden ~ N(0, 1), w ~ N(0, 1/H), bias 0.5, threshold 0.3: over many
    requests the verified length has mean about 1.83 and is 0 for about 9 %."""
    w = W.confidence("cpu", seed=3, B=4096, k=8, V=16)
    c = w["conf"]
    assert tuple(c["hidden"].shape) == (4096, 8, 2560) and c["hidden"].dtype == torch.bfloat16
    assert c["bias"] == 0.5 and c["threshold"] == 0.3
    assert abs(_f(c["w"]).std() * math.sqrt(2560) - 1.0) < 0.05
    z = c["hidden"].double() @ c["w"].double() + c["bias"]
    P = torch.cumprod(torch.sigmoid(z), dim=1)
    L = torch.cumprod((P >= c["threshold"]).int(), dim=1).sum(dim=1).double()
    assert 1.75 < L.mean().item() < 1.91
    assert 0.07 < (L == 0).double().mean().item() < 0.11


def test_batch_budget_recipe():
    w = W.confidence_batch_budget("cpu", seed=3, B=8, k=8, V=16)
    assert w["conf"]["threshold"] == 0.05 and w["conf"]["total"] == 16
    assert W.confidence_batch_budget("cpu", seed=3, B=8, k=8, V=16, total=5)["conf"]["total"] == 5


def test_sweep_recipe():
    w = W.sweep("cpu", seed=4, B=3000, k=5, V=16)
    T = w["temperature"].numpy()
    assert set(np.unique(T).tolist()) == {0.0, float(np.float32(0.7)), 1.0}
    for v in (0.0, 0.7, 1.0):
        assert abs(np.isclose(T, v).mean() - 1 / 3) < 0.04
    vl = w["verify_len"].numpy()
    assert set(vl.tolist()) == {1, 2, 3, 4, 5}
    # greedy requests draft the drafter's own arg-max
    g = T == 0
    am = torch.argmax(w["draft"].float(), dim=-1).numpy()
    assert (w["tokens"].numpy()[g] == am[g]).all()


def test_lmhead_grid_values_are_on_the_grid():
    w = W.lmhead("cpu", seed=5, B=4, k=3, V=64, H=32, grid=True, w_levels=3)
    ht, hd, head = _f(w["hidden_target"]), _f(w["hidden_draft"]), _f(w["head"])
    assert np.all(np.abs(ht * 4 - np.round(ht * 4)) == 0) and np.abs(ht).max() <= 0.75
    assert np.all(np.abs(hd * 4 - np.round(hd * 4)) == 0) and np.abs(hd).max() <= 0.75
    assert np.all(np.abs(head * 8 - np.round(head * 8)) == 0) and np.abs(head).max() <= 3 / 8
    assert set(np.unique(np.round(head * 8)).tolist()) <= set(range(-3, 4))


def test_lmhead_real_valued_logit_scale():
    """W ~ N(0, (3/sqrt(H))^2) and h ~ N(0, 1): logits have std close to 3."""
    w = W.lmhead("cpu", seed=5, B=8, k=2, V=2048, H=256)
    lt = w["hidden_target"].float() @ w["head"].float().T
    assert abs(lt.std().item() - 3.0) < 0.15


@pytest.mark.parametrize("make", [
    lambda s: W.stochastic("cpu", seed=s, B=4, k=3, V=256),
    lambda s: W.greedy("cpu", seed=s, B=4, k=3, V=256),
    lambda s: W.sweep("cpu", seed=s, B=4, k=3, V=256),
    lambda s: W.lmhead("cpu", seed=s, B=2, k=2, V=64, H=16),
])
def test_seeded_and_deterministic(make):
    a, b, c = make(11), make(11), make(12)
    for key, v in a.items():
        if isinstance(v, torch.Tensor):
            assert torch.equal(v, b[key]), key
    assert any(isinstance(v, torch.Tensor) and not torch.equal(v, c[key])
               for key, v in a.items() if key != "temperature")
