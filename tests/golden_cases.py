"""Loader of the hand-worked cases in golden/uniform_support_cases.txt (shared by
the oracle pins and the GPU parity tests; it holds no verification arithmetic)."""
import os

import numpy as np

PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "uniform_support_cases.txt")


def _row(spec, V):
    kind, _, body = spec.strip().partition(":")
    if kind == "S":
        row = np.full(V, -np.inf, dtype=np.float32)
        row[[int(t) for t in body.split(",")]] = 0.0
        return row
    if kind == "L":
        vals = [float(v) for v in body.split(",")]
        assert len(vals) == V
        return np.array(vals, dtype=np.float32)
    raise ValueError("bad row spec %r" % spec)


def load():
    cases, cur = [], None
    for line in open(PATH):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest}
            cases.append(cur)
        else:
            cur[key] = rest
    out = []
    for c in cases:
        V, k = int(c["V"]), int(c["k"])
        target = np.stack([_row(s, V) for s in c["target"].split("|")])[None]
        draft = np.stack([_row(s, V) for s in c["draft"].split("|")])[None]
        u = np.array([[float(v) for v in pair.split()] for pair in c["u"].split("|")])[None]
        assert target.shape == (1, k + 1, V) and draft.shape == (1, k, V) and u.shape == (1, k + 1, 2)
        out.append(dict(
            name=c["name"], V=V, k=k, target=target, draft=draft,
            tokens=np.array([[int(t) for t in c["tokens"].split()]], dtype=np.int32),
            verify_len=np.array([int(c["L"])], dtype=np.int32),
            temperature=np.array([float(c["T"])], dtype=np.float32),
            u=np.ascontiguousarray(u, dtype=np.float64),
            n=int(c["expect_n"]),
            out_tokens=np.array([int(t) for t in c["expect_tokens"].split()], dtype=np.int32)))
    return out
