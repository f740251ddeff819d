"""The oracle against the hand-derived worked cases in tests/golden/.

Each fixture states its derivation and the passages it follows; values are
exact (rationals and logarithms) and are compared to 1e-14.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")
TOL = 1e-14
MODES = {"train": oracle.TRAIN, "sparse": oracle.SPARSE, "threshold": oracle.THRESHOLD}


def val(x):
    """An exact fixture value: a number, "a/b" or "ln(a/b)"."""
    if isinstance(x, (int, float)):
        return float(x)
    x = x.strip()
    if x.startswith("ln(") and x.endswith(")"):
        return math.log(float(Fraction(x[3:-1])))
    return float(Fraction(x))


def arr(xs):
    return np.array([[val(v) for v in row] for row in xs] if isinstance(xs[0], list)
                    else [val(v) for v in xs])


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        case = json.load(f)
    assert case["cite"] and case["derivation"]
    N = len(case["Q"])
    t = {k: arr(case[k]).reshape(1, 1, N, 1) for k in ("Q", "K", "V", "dO")}
    t["S"] = arr(case["S"]).reshape(1, 1, N, N)
    return case, t


def close(x, ref):
    return np.max(np.abs(np.asarray(x, dtype=np.float64) - ref)) < TOL


def test_three_tokens_block1():
    case, t = load("three_tokens_block1.json")
    e = case["expected"]
    O, LSE = oracle.gated_attention_forward(t["Q"], t["K"], t["V"], t["S"], case["block"])
    assert close(O[0, 0, :, 0], arr(e["O"])) and close(LSE[0, 0], arr(e["LSE"]))
    dQ, dK, dV, dS, G = oracle.gated_attention_backward(t["Q"], t["K"], t["V"], t["S"], t["dO"],
                                                        case["block"])
    g = e["G_row"]
    assert close(G[0, 0, g["row"], g["cols"]], arr(g["values"]))
    assert close(dS[0, 0], arr(e["dS"])) and close(dV[0, 0, :, 0], arr(e["dV"]))


@pytest.mark.parametrize("mode", ["train", "sparse", "threshold"])
def test_four_tokens_block1(mode):
    case, t = load("four_tokens_modes_block1.json")
    e = case["modes"][mode]
    kw = dict(mode=MODES[mode], topk=e["topk"], tau=e["tau"])
    bs = case["block"]
    O, LSE = oracle.gated_attention_forward(t["Q"], t["K"], t["V"], t["S"], bs, **kw)
    assert close(O[0, 0, :, 0], arr(e["O"])) and close(LSE[0, 0], arr(e["LSE"]))
    dQ, dK, dV, dS, _ = oracle.gated_attention_backward(t["Q"], t["K"], t["V"], t["S"], t["dO"], bs, **kw)
    assert close(dS[0, 0, 3], arr(e["dS_row3"])) and close(dS[0, 0, :3], 0.0)
    assert close(dQ[0, 0, :, 0], arr(e["dQ"])) and close(dK, 0.0)
    assert close(dV[0, 0, :, 0], arr(e["dV"]))
    for dec in e.get("decode", []):
        L = dec["L"]
        o, lse = oracle.gated_decode(t["Q"][:, :, L - 1], t["K"][:, :, :L], t["V"][:, :, :L],
                                     t["S"][:, :, dec["score_row"], :L], L, bs, e["topk"], mode=MODES[mode],
                                     tau=e["tau"])
        assert close(o[0, 0, 0], val(dec["O"])) and close(lse[0, 0], val(dec["LSE"])), L


def test_golden_catches_unnormalised_gate():
    """Row 3's Top-2 output ignores a shift of its scores, and gates normalised
    over the whole history instead of the kept set (the oracle's
    renormalise=False option, a plausible misreading) miss the golden value."""
    case, t = load("four_tokens_modes_block1.json")
    S = t["S"].copy()
    S[0, 0, 3, :3] += 1.0  # a shift the normalised gates ignore ...
    O, _ = oracle.gated_attention_forward(t["Q"], t["K"], t["V"], S, 1, mode=oracle.SPARSE, topk=2)
    assert close(O[0, 0, 3, 0], val(case["modes"]["sparse"]["O"][3]))
    raw = oracle.gated_attention_forward(t["Q"], t["K"], t["V"], S, 1, mode=oracle.SPARSE, topk=2,
                                         renormalise=False)[0]
    assert not close(raw[0, 0, 3, 0], val(case["modes"]["sparse"]["O"][3]))  # ... and a wrong one does not
