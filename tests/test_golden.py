"""The oracle's alpha-entmax, routing and prior-induced stage 2 against
hand-derived worked cases (tests/golden/entmax_worked_cases.txt: closed forms
with their derivations, independent of the oracle's sort-based threshold
search).

A wrong scale (gamma, or x = z instead of (alpha - 1) z), a sum instead of
the GQA mean, a support error, a prior on the wrong block or the wrong
diagonal prior changes these values far beyond the 1e-12 tolerance.
"""

import math
import os

import numpy as np
import pytest

from oracle.dash_oracle import block_summaries, entmax, forward_row, route_row

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "entmax_worked_cases.txt")


def _value(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"sqrt": math.sqrt, "log": math.log, "exp": math.exp}))


def load_cases() -> dict:
    cases, cur = {}, None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = cases.setdefault(rest.strip(), {})
            continue
        cur[key] = [_value(v) for v in rest.split(";")]
    return cases


CASES = load_cases()


def test_fixture_has_the_cases():
    assert {"sparsemax_three", "entmax15_two_of_three", "entmax15_full_support", "route_gqa_two_heads",
            "stage2_one_token_blocks"} <= set(CASES)


@pytest.mark.parametrize("name", sorted(n for n in CASES if "tau" in CASES[n]))
def test_entmax_worked_case(name):
    c = CASES[name]
    p, tau = entmax(np.array(c["z"]), c["alpha"][0])
    np.testing.assert_allclose(p, c["p"], rtol=0, atol=1e-12)
    assert abs(tau - c["tau"][0]) <= 1e-12
    assert abs(p.sum() - 1.0) <= 1e-12


def test_route_gqa_worked_case():
    c = CASES["route_gqa_two_heads"]
    d = int(c["d"][0])
    summ = np.array(c["summaries"]).reshape(-1, d)
    q = np.array([c["q0"], c["q1"]])
    r = route_row(q, summ, c["alpha"][0])
    np.testing.assert_allclose(r["pbar"], c["pbar"], rtol=0, atol=1e-12)
    assert r["idx"].tolist() == [int(i) for i in c["idx"]]
    np.testing.assert_allclose(r["logp"], np.log(c["pbar"]), rtol=0, atol=1e-12)
    # the two heads' distributions are the single-vector cases
    np.testing.assert_allclose(r["p"][0], CASES["entmax15_two_of_three"]["p"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["p"][1], CASES["entmax15_full_support"]["p"], rtol=0, atol=1e-12)


def test_stage2_worked_case():
    c = CASES["stage2_one_token_blocks"]
    blk = int(c["block"][0])
    k = np.array(c["k"])[:, None]
    v = np.array(c["v"])[:, None]
    q = np.array([c["q"]])
    w = np.array([c["w_s"]])
    n = len(k)
    summ = block_summaries(k, w, blk, n)
    np.testing.assert_allclose(summ[:, 0], c["k"], rtol=0, atol=1e-15)
    alpha = c["alpha"][0]
    for sigma, key in ((1.0, "out_causal_pos2_sigma1"), (2.0, "out_causal_pos2_sigma2")):
        r = forward_row(q, k, v, summ, 2, n, blk, alpha, True, sigma=sigma)
        assert r["blocks"].tolist() == [0, 1]
        np.testing.assert_allclose(r["pbar"], c["pbar"], rtol=0, atol=1e-12)
        assert abs(r["out"][0, 0] - c[key][0]) <= 1e-12, key
    r = forward_row(q, k, v, summ, 0, n, blk, alpha, False)
    assert r["blocks"].tolist() == [1, 2]
    assert abs(r["out"][0, 0] - c["out_noncausal_pos0"][0]) <= 1e-12
