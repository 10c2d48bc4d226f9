"""The oracle's pins are sensitive: for each plausible mistake planted in a
copy of ``oracle.c`` (a comparison made non-strict, an operand swapped, a
term dropped, a wrong row, draw or constant), the pin suite run against that
copy fails.  The copy is compiled with the oracle's own flags into a
temporary directory and loaded through ``ORACLE_LIB_OVERRIDE``; the oracle
itself is never modified (CPU only)."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["tests/test_oracle.py", "tests/test_oracle_budget.py"]

# name -> (exact text in oracle.c, its mutated form).  Only mistakes that change
# a result belong here: for example, counting every position with P_j >= tau
# instead of the leading run would change nothing, since P never grows; and a
# NaN or +inf that the sampled rows' scan missed would still fail the request
# through the checks on the maximum and the normaliser.
MUTANTS = {
    # accept / reject rule
    "accept comparison not strict": ("if (u * q < p) {", "if (u * q <= p) {"),
    "accept ratio inverted": ("if (u * q < p) {", "if (u * p < q) {"),
    "accept draw reused for the sample": ("double u2 = draw_uniform(in, i, j, 1);",
                                          "double u2 = draw_uniform(in, i, j, 0);"),
    # residual distribution
    "residual sign flipped": ("double r = p - q;", "double r = q - p;"),
    "residual not clamped at zero": ("return r > 0.0 ? r : 0.0;", "return fabs(r);"),
    "residual floor skipped": ("if (residual_total(&rc, V) >= ORC_RESIDUAL_FLOOR) {", "if (1) {"),
    # inverse CDF
    "inverse CDF comparison not strict": ("if (running > target) {", "if (running >= target) {"),
    "fallback takes the first positive weight": (
        "if (w > 0.0) last_positive = t;", "if (w > 0.0 && last_positive < 0) last_positive = t;"),
    # bonus token
    "bonus from the previous row": ("const void* trow = (const char*)trows + L * row_bytes;",
                                    "const void* trow = (const char*)trows + (L > 0 ? L - 1 : 0) * row_bytes;"),
    "bonus with the accept draw": ("draw_uniform(in, i, L, 1)", "draw_uniform(in, i, L, 0)"),
    # softmax
    "temperature multiplies in the normaliser": (
        "for (int64_t t = 0; t < V; ++t) Z += exp(load_logit(row, dtype, t) / T - m);",
        "for (int64_t t = 0; t < V; ++t) Z += exp(load_logit(row, dtype, t) * T - m);"),
    "bf16 widened from the wrong half": ("uint32_t w = (uint32_t)bits << 16;",
                                         "uint32_t w = (uint32_t)bits << 15;"),
    # greedy
    "greedy takes the last maximal index": ("if (best_t < 0 || v > best) {",
                                            "if (best_t < 0 || v >= best) {"),
    "greedy emits the drafted token on disagreement": ("tok[j] = a;", "tok[j] = x[j];"),
    # random draws
    "Philox with nine rounds": ("for (int round = 0; round < 10; ++round) {",
                                "for (int round = 0; round < 9; ++round) {"),
    "Philox Weyl increment off by one": ("k1 += 0xBB67AE85u;", "k1 += 0xBB67AE86u;"),
    "uniform from 27 + 27 bits": ("double lo = (double)(w[1] >> 6);", "double lo = (double)(w[1] >> 5);"),
    "counter words swapped": ("uint32_t ctr[4] = {2u * position + draw, request, step, 0u};",
                              "uint32_t ctr[4] = {2u * position + draw, request, 0u, step};"),
    "request offset ignored": ("return oracle_uniform(in->seed, in->request_offset + (uint32_t)i,",
                               "return oracle_uniform(in->seed, (uint32_t)i,"),
    # lengths, confidence head and batch budget
    "verify_len clamped one short": ("if (L > k) L = k;", "if (L > k) L = k - 1;"),
    "survival not a running product": ("prefix *= s;", "prefix = s;"),
    "confidence bias dropped": ("z += (double)bias;", "z += 0.0;"),
    "confidence threshold strict": ("prefix >= (double)threshold", "prefix > (double)threshold"),
    "budget keeps the smallest survivals": ("if (x->P != y->P) return x->P > y->P ? -1 : 1;",
                                            "if (x->P != y->P) return x->P < y->P ? -1 : 1;"),
    "budget ties to the higher request": ("if (x->i != y->i) return x->i < y->i ? -1 : 1;",
                                          "if (x->i != y->i) return x->i > y->i ? -1 : 1;"),
    "negative verify_len not clamped": ("if (L < 0) L = 0;", "if (L < 0) L = -L;"),
    # the accept test's probabilities
    "q of the drafted token read from the target row": (
        "double q = exp(load_logit(drow, in->dtype, x[j]) / T - mq) / Zq;",
        "double q = exp(load_logit(trow, in->dtype, x[j]) / T - mq) / Zq;"),
    "p normalised by the drafter's sum": (
        "double p = exp(load_logit(trow, in->dtype, x[j]) / T - mp) / Zp;",
        "double p = exp(load_logit(trow, in->dtype, x[j]) / T - mp) / Zq;"),
    "residual q normalised by the target's sum": (
        "double q = exp(load_logit(c->drow, c->dtype, t) / c->T - c->mq) / c->Zq;",
        "double q = exp(load_logit(c->drow, c->dtype, t) / c->T - c->mq) / c->Zp;"),
    # the uniform's 53 bits
    "uniform scaled by 2^53 - 1": ("/ 9007199254740992.0;", "/ 9007199254740991.0;"),
    "uniform high word shifted one bit less": ("double hi = (double)(w[0] >> 5);",
                                               "double hi = (double)(w[0] >> 4);"),
    # error semantics
    "+inf in a greedy row not detected": (
        "        if (isnan(v) || v == INFINITY) return ORC_ERR_NONFINITE;\n        if (best_t < 0",
        "        if (isnan(v)) return ORC_ERR_NONFINITE;\n        if (best_t < 0"),
    "drafted token V accepted as in range": (
        "if (x[j] < 0 || (int64_t)x[j] >= V) { err = ORC_ERR_BAD_TOKEN; break; }\n            const void* trow",
        "if (x[j] < 0 || (int64_t)x[j] > V) { err = ORC_ERR_BAD_TOKEN; break; }\n            const void* trow"),
    "negative temperature accepted": ("if (!(T >= 0.0f) || isinf(T)) return 0;", "if (isinf(T)) return 0;"),
    # chain bookkeeping
    "stochastic rejection counts the rejected position": ("            n = j;\n            break;\n        }\n        if (!err && n == L) {\n            /* 4.",
                                                          "            n = j + 1;\n            break;\n        }\n        if (!err && n == L) {\n            /* 4."),
}


def _run_pins_on(index, name, old, new, tmp_path):
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    assert src.count(old) == 1, "mutation site not unique: %s" % name
    d = tmp_path / ("mutant%02d" % index)
    d.mkdir()
    c_path = d / "oracle.c"
    c_path.write_text(src.replace(old, new))
    lib = oracle.compile_source(str(c_path), str(d / "liboracle_mutant.so"))
    env = dict(os.environ, ORACLE_LIB_OVERRIDE=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"] + PIN_FILES,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    failed = [s.split(" ")[1] for s in r.stdout.splitlines() if s.startswith("FAILED ")]
    return r.returncode, failed


def test_every_planted_mistake_fails_a_pin(tmp_path):
    oracle.build()
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        futs = {n: ex.submit(_run_pins_on, q, n, o, m, tmp_path)
                for q, (n, (o, m)) in enumerate(MUTANTS.items())}
        results = {n: f.result() for n, f in futs.items()}
    survivors = sorted(n for n, (rc, _) in results.items() if rc == 0)
    broken = sorted(n for n, (rc, _) in results.items() if rc not in (0, 1))
    assert not survivors, "mistakes no pin catches: %s" % survivors
    assert not broken, "mutants that did not run the pins: %s" % broken
    for n, (_, failed) in results.items():
        assert failed, n
