"""Writes the oracle regression fixtures in this folder.

Calls only ``oracle/`` (and ``synth/`` for the seeded inputs).  The fixtures
pin the oracle against unintended change; its correctness pins are the closed
forms and invariants in ``tests/test_oracle_*.py``.

    python tests/golden/make_golden.py
"""

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import MuonHParams, muon_step, AdamWHParams, adamw_step  # noqa: E402
from synth.workloads import custom_workload  # noqa: E402
from synth.gen import matrix_inputs, tail_inputs  # noqa: E402


def main():
    wl = custom_workload([(6, 10)], dtype="f32", tail=16, seed=77)
    mi = matrix_inputs(wl, wl.matrices[0], step=0, buf_init="random")
    hp = MuonHParams()
    Wn, O, bn = muon_step(mi.W, mi.G, mi.buf, hp)
    out = {
        "what": "oracle muon_step on a seeded 6x10 fp32 case (custom_workload seed 77, random buf)",
        "W": mi.W.astype(float).tolist(), "G": mi.G.astype(float).tolist(),
        "buf": mi.buf.astype(float).tolist(),
        "O": O.tolist(), "W_new": Wn.tolist(), "buf_new": bn.tolist(),
    }
    with open(os.path.join(HERE, "oracle_tiny_step.json"), "w") as f:
        json.dump(out, f, indent=1)
    ti = tail_inputs(wl, step=0, state="random")
    ah = AdamWHParams()
    p, m, v = adamw_step(ti.p, ti.g, ti.m, ti.v, 3, ah)
    out = {
        "what": "oracle adamw_step at t=3 on a seeded 16-element tail (custom_workload seed 77, random state)",
        "p": ti.p.astype(float).tolist(), "g": ti.g.astype(float).tolist(),
        "m": ti.m.astype(float).tolist(), "v": ti.v.astype(float).tolist(), "t": 3,
        "p_new": p.tolist(), "m_new": m.tolist(), "v_new": v.tolist(),
    }
    with open(os.path.join(HERE, "oracle_tiny_adamw.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
