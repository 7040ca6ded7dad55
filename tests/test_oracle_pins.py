"""The CPU oracle checked against facts other than itself (see tests/_pins.py), and
mutation tests: every deliberately broken build of the oracle fails at least one pin."""
import math
import tempfile
from pathlib import Path

import numpy as np
import pytest

import oracle
import synth
from tests import _pins

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", _pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_closed_form_two_keys(orc):
    """q=(1,0), keys (1,0),(0,1), values (1,0),(0,1), scale 1: logits (1, 0), so
    O = (e, 1)/(e+1) and LSE = ln(e+1).  (Two bf16-exact unit vectors, d padded to 16.)"""
    d = 16
    one = synth.f32_to_bf16_bits(np.array([1.0], dtype=np.float32))[0]
    q = np.zeros((1, 1, 1, d), np.uint16); q[0, 0, 0, 0] = one
    k = np.zeros((1, 2, 1, d), np.uint16); k[0, 0, 0, 0] = one; k[0, 1, 0, 1] = one
    v = k.copy()
    O, L = orc.forward(q, k, v, 1.0, False)
    e = math.e
    assert abs(O[0, 0, 0, 0] - e / (e + 1)) < 1e-15
    assert abs(O[0, 0, 0, 1] - 1 / (e + 1)) < 1e-15
    assert abs(L[0, 0, 0] - math.log(e + 1)) < 1e-15
    # causal with Nq = 1, Nk = 2: bottom-right alignment lets the single query see both keys
    Oc, Lc = orc.forward(q, k, v, 1.0, True)
    assert np.array_equal(Oc, O) and np.array_equal(Lc, L)


def test_no_visible_key_rows(orc):
    """Causal with Nq > Nk: the first Nq - Nk rows see no key -> O = 0, LSE = -inf;
    Nk = 0 -> every row is empty."""
    x = _pins.tiny_inputs(1, 2, 1, 6, 2, 32, seed=30)
    O, L = orc.forward(x["q"], x["k"], x["v"], 0.3, True)
    assert (O[0, :4] == 0).all() and np.isneginf(L[0, :, :4]).all()
    assert np.isfinite(L[0, :, 4:]).all()
    k0 = np.zeros((1, 0, 1, 32), np.uint16)
    O0, L0 = orc.forward(x["q"], k0, k0, 0.3, False)
    assert (O0 == 0).all() and np.isneginf(L0).all()


def test_threads_do_not_change_result(orc):
    x = _pins.tiny_inputs(1, 3, 1, 50, 40, 32, seed=31)
    O1, L1 = orc.forward(x["q"], x["k"], x["v"], 0.3, True, threads=1)
    O4, L4 = orc.forward(x["q"], x["k"], x["v"], 0.3, True, threads=4)
    assert np.array_equal(O1, O4) and np.array_equal(L1, L4)


def test_invalid_sizes_rejected(orc):
    x = _pins.tiny_inputs(1, 3, 1, 4, 4, 32, seed=32)
    k2 = np.zeros((1, 4, 2, 32), np.uint16)   # Hq=3 not a multiple of Hkv=2
    with pytest.raises(RuntimeError):
        orc.forward(x["q"], k2, k2, 0.3, False)


MUTANTS = ["ORACLE_PLANT_NO_SCALE", "ORACLE_PLANT_GQA_MODULO", "ORACLE_PLANT_CAUSAL_STRICT",
           "ORACLE_PLANT_TRANSPOSE_V", "ORACLE_PLANT_LSE_NO_MAX", "ORACLE_PLANT_NO_NORMALIZE",
           "ORACLE_PLANT_WINDOW_OFF_BY_ONE", "ORACLE_PLANT_F16_BIAS", "ORACLE_PLANT_BWD_NO_D",
           "ORACLE_PLANT_BWD_DQ_NO_SCALE", "ORACLE_PLANT_BWD_DV_NO_P", "ORACLE_PLANT_E4M3_BIAS"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_pins_catch_planted_mistake(mutant):
    """Each planted mistake (dropped scale, modulo GQA mapping, diagonal masked,
    transposed V index, LSE without the max, missing normalisation, window one key too
    wide, fp16 exponent bias off by one, backward without the D term, dQ without the
    scale, dV without the P weights, E4M3 exponent bias off by one) fails a pin."""
    with tempfile.TemporaryDirectory() as td:
        lib = oracle.build(Path(td) / f"lib_{mutant}.so", defines=(mutant,))
        bad = oracle.Oracle(lib)
        failed = []
        for pin in _pins.ALL_PINS:
            try:
                pin(bad)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"no pin caught {mutant}"
