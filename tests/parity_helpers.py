"""Element-by-element comparison of the CUDA path with the fp64 CPU oracle,
shared by the GPU test files.

Bar (from the verification rule's tolerances): p_j(x_j) and q_j(x_j) within
1e-5 absolute + 1e-4 relative; accepted lengths and emitted tokens bit-exact,
except for requests holding an accept draw within 1e-6 of p/q (counted; they
must stay below 1e-5 of all decisions); greedy results bit-exact.
"""
import os

import numpy as np

import oracle
from speculative_decoding_verification_86_b200 import workloads

THREADS = max(1, min(32, os.cpu_count() or 1))


def run_oracle(w, u_override=None, request_offset=0):
    h = workloads.to_numpy_inputs(w)
    return oracle.verify(h["target"], h["draft"], h["tokens"], dtype=h["dtype"],
                         verify_len=h["verify_len"], temperature=h["temperature"], conf=h["conf"],
                         seed=h["seed"], u_override=u_override, request_offset=request_offset,
                         threads=THREADS)


def compare(g, o, strict=False):
    """Assert parity; returns (decisions, exempt decisions).  ``strict``: no
    exemption at all (draws placed a known distance from the decision edges)."""
    am = o["accept_margin"]
    evaluated = am >= 0
    exempt = evaluated & (am < (0.0 if strict else 1e-6))
    n_dec = int(evaluated.sum()) + int((o["sample_margin"] >= 0).sum())
    n_ex = int(exempt.sum())
    assert n_ex <= 1e-5 * max(n_dec, 1), (n_ex, n_dec)
    ok = ~exempt.any(axis=1) if am.shape[1] else np.ones(len(o["accepted"]), bool)
    np.testing.assert_array_equal(g["status"][ok].astype(np.uint32), o["status"][ok])
    np.testing.assert_array_equal(g["accepted"][ok], o["accepted"][ok])
    np.testing.assert_array_equal(g["tokens"][ok], o["tokens"][ok])
    if "p" in g:
        for gv, ov in ((g["p"], o["p_x"]), (g["q"], o["q_x"])):
            gv, ov = gv[ok], ov[ok]
            ev = ov >= 0
            assert np.all(gv[~ev] == -1.0)
            err = np.abs(gv[ev].astype(np.float64) - ov[ev])
            assert np.all(err <= 1e-5 + 1e-4 * np.abs(ov[ev])), err.max()
    return n_dec, n_ex


def host(o):
    """Device outputs as numpy arrays."""
    return {k: v.cpu().numpy() for k, v in o.items()}
