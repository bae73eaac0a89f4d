"""Write the oracle regression fixture ``oracle_small.json``.

Calls only ``oracle/``.  The fixture freezes the oracle's output on one small
seeded case so that a later change to the oracle's arithmetic shows up as a
diff; the pins in ``tests/test_oracle_pins.py`` are what tie that output to the
recurrence of the "Kimi K3" open-weights field notes
(ailearn.mscapital.top/kimi-k3.html), panel "KDA 单头递归".

Usage: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def case():
    rng = np.random.default_rng(42)
    B, T, H, dk, dv = 1, 7, 2, 3, 2
    q = rng.standard_normal((B, T, H, dk)).round(3)
    k = rng.standard_normal((B, T, H, dk)).round(3) * 0.5
    v = rng.standard_normal((B, T, H, dv)).round(3)
    g = -rng.uniform(0, 5, (B, T, H, dk)).round(3)
    beta = rng.uniform(0, 1, (B, T, H)).round(3)
    h0 = rng.standard_normal((B, H, dk, dv)).round(3)
    return dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)


def main():
    inp = case()
    o, hT = oracle.kda_fwd(**inp)
    out = {"what": "fp64 oracle output on a small seeded case (regression fixture)",
           "source": "recurrence of the 'Kimi K3' open-weights field notes, panel 'KDA 单头递归'",
           "inputs": {n: a.tolist() for n, a in inp.items()},
           "o": o.tolist(), "hT": hT.tolist()}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
