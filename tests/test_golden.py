"""The oracle still reproduces its frozen regression fixture, and the fixture
itself agrees with the brute-force operator products (CPU only)."""
import json
import os

import numpy as np

import oracle
from tests.oracle_helpers import brute_force

HERE = os.path.dirname(os.path.abspath(__file__))


def load():
    with open(os.path.join(HERE, "golden", "oracle_small.json")) as f:
        d = json.load(f)
    inp = {k: np.array(v, dtype=np.float64) for k, v in d["inputs"].items()}
    return inp, np.array(d["o"]), np.array(d["hT"])


def test_oracle_matches_fixture():
    inp, o_ref, hT_ref = load()
    o, hT = oracle.kda_fwd(**inp)
    np.testing.assert_allclose(o, o_ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(hT, hT_ref, rtol=1e-13, atol=1e-15)


def test_fixture_matches_brute_force():
    inp, o_ref, hT_ref = load()
    for h in range(inp["q"].shape[2]):
        o_bf, S_bf = brute_force(inp["q"][0, :, h], inp["k"][0, :, h], inp["v"][0, :, h],
                                 inp["g"][0, :, h], inp["beta"][0, :, h], inp["h0"][0, h])
        np.testing.assert_allclose(o_ref[0, :, h], o_bf, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(hT_ref[0, h], S_bf, rtol=1e-12, atol=1e-13)
