"""Hand-worked examples of the gated delta-rule update (tests/golden/*.json).

The pages print no worked numbers, so each fixture is evaluated by hand from
the update's definition and carries its derivation and citation.
"""
import json
import os

import numpy as np

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_two_token_worked_example():
    d = _load("two_token_2x2.json")
    q = np.array(d["q"])[None, :, None, :]
    k = np.array(d["k"])[None, :, None, :]
    v = np.array(d["v"])[None, :, None, :]
    beta = np.array(d["beta"])[None, :, None]
    g = np.array(d["g"])[None, :, None]
    S0 = np.array(d["S0"], dtype=float)[None, None]
    o, ST = oracle.recurrent_fwd(q, k, v, beta, g, S0)
    np.testing.assert_allclose(o[0, :, 0], np.array(d["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(ST[0, 0], np.array(d["ST"]), rtol=0, atol=1e-12)


def test_one_token_hand_gradients():
    d = _load("one_token_scalar_grad.json")
    arr = lambda x: np.array([[[[x]]]], dtype=float)
    q, k, v = arr(d["q"]), arr(d["k"]), arr(d["v"])
    beta = np.array([[[d["beta"]]]])
    g = np.array([[[d["g"]]]])
    S0 = arr(d["S0"])
    o, ST = oracle.recurrent_fwd(q, k, v, beta, g, S0)
    assert abs(o.item() - d["o"]) < 1e-12 and abs(ST.item() - d["ST"]) < 1e-12
    gr = oracle.recurrent_bwd(q, k, v, beta, g, S0, arr(d["dO"]))
    for name in ("dq", "dk", "dv", "dbeta", "dg", "dS0"):
        assert abs(gr[name].item() - d[name]) < 1e-12, name


def test_sfda_two_token_rotation_example():
    d = _load("sfda_two_token_rotation.json")
    q = np.array(d["q"])[None, :, None, :]
    k = np.array(d["k"])[None, :, None, :]
    v = np.array(d["v"])[None, :, None, :]
    beta = np.array(d["beta"])[None, :, None]
    g = np.array(d["g"])[None, :, None, :]
    S0 = np.array(d["S0"], dtype=float)[None, None]
    o, ST = oracle.recurrent_fwd(q, k, v, beta, g, S0, gate=oracle.GATE_PHASE)
    np.testing.assert_allclose(o[0, :, 0], np.array(d["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(ST[0, 0], np.array(d["ST"]), rtol=0, atol=1e-12)
