"""Writes oracle_tiny.json: a regression fixture of the fp64 oracle.

Calls only ``oracle/``.  The inputs are small exact binary fractions so the
file is readable; the pages print no worked example of their own, so this
fixture guards the oracle against accidental change rather than citing one.
Run:  python tests/golden/make_golden.py
"""
import json
import sys
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parents[2]
sys.path.insert(0, str(ROOT))
import oracle  # noqa: E402


def case():
    T, H, dk, dv = 5, 1, 3, 2
    r = np.random.default_rng(7)
    q = np.round(r.standard_normal((1, T, H, dk)) * 8) / 8
    k = np.round(r.standard_normal((1, T, H, dk)) * 8) / 8
    v = np.round(r.standard_normal((1, T, H, dv)) * 8) / 8
    la = -np.round(np.abs(r.standard_normal((1, T, H, dk))) * 4) / 8
    beta = np.round(r.uniform(0, 1, (1, T, H)) * 8) / 8
    S0 = np.round(r.standard_normal((1, H, dk, dv)) * 8) / 8
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0)


def main():
    x = case()
    o, S = oracle.forward(**x)
    out = {k: v.tolist() for k, v in x.items()}
    out["o"] = o.tolist()
    out["S_T"] = S.tolist()
    (Path(__file__).parent / "oracle_tiny.json").write_text(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
