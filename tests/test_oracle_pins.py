"""The fp64 oracle against pins that do not go through its own loop.

Closed forms, explicit products, library routines, split invariance and a
hand-derived worked example; then a mutation test that plants one plausible
mistake at a time into the oracle (compiled with SSM_ORACLE_MUTANT) and shows
that at least one pin fails for every mistake.
"""
import json
import os

import numpy as np
import pytest

import oracle
import oracle_pins as P

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check(0)


def test_hand_example_scan():
    g = _golden()["scan_mamba1_two_steps"]
    i = g["inputs"]
    y, hf, _ = oracle.scan_fwd(oracle.MAMBA1, np.array(i["x"]).reshape(1, 2, 1), np.array(i["dt"]).reshape(1, 2, 1),
                               np.array([[i["A"]]]), np.array(i["B"]).reshape(1, 2, 1), np.array(i["C"]).reshape(1, 2, 1),
                               D=np.array([i["D"]]), dt_bias=np.array([i["dt_bias"]]),
                               h0=np.array([i["h0"]]).reshape(1, 1, 1), delta_softplus=i["delta_softplus"])
    np.testing.assert_allclose(y.ravel(), g["expected"]["y"], rtol=1e-15)
    np.testing.assert_allclose(hf.ravel(), [g["expected"]["h_final"]], rtol=1e-15)


def test_hand_example_conv():
    g = _golden()["conv_with_state"]
    i = g["inputs"]
    out, so = oracle.conv1d_fwd(np.array(i["x"]).reshape(1, 2, 1), np.array(i["w"]).reshape(1, 4),
                                b=np.array([i["bias"]]), state_in=np.array(i["state_in"]).reshape(1, 1, 3),
                                activation=False)
    np.testing.assert_array_equal(out.ravel(), g["expected"]["pre_activation"])
    np.testing.assert_array_equal(so.ravel(), g["expected"]["state_out"])


MUTANTS = {
    1: "h0 ignored (the (h0, 0) seed)",
    2: "D skip term dropped",
    3: "decay sign flipped",
    4: "conv taps reversed",
    5: "strided group map h % G",
    6: "read-out before the state update",
    7: "dt_bias dropped",
    8: "gate on x instead of z",
    9: "B and C swapped",
    10: "conv state ignored",
    11: "softplus switch inverted",
    12: "skip term on the pre-conv x",
    13: "intermediate state recorded one token early",
    14: "backward: dh not carried back through exp(delta A)",
    15: "decode: conv state rolled the wrong way",
    16: "decode: conv window read one position too old (width-K state)",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: f"m{m}")
def test_pins_catch_planted_mistake(mutant):
    assert oracle.mutant_id(mutant) == mutant
    failed = []
    for check in P.ALL_CHECKS:
        try:
            check(mutant)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {mutant}: {MUTANTS[mutant]}"
