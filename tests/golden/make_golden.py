"""Writes the stored traces under tests/golden/ from the seeded workloads and
the oracle only (python tests/golden/make_golden.py from the repo root).

tiny_tau_trace.json: the tiny workload's per-step update counts M and the
threshold decisions of the FlashBlock rule (technical summary, §2 "Adaptive
reuse strategies": reuse when M < tau, else recompute; step 0 has no cache).
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle.controllers import ThresholdController  # noqa: E402
from workloads import make_workload  # noqa: E402


def tiny_trace():
    wl = make_workload("tiny")
    tau = wl.spec.tau
    ctl = ThresholdController(wl.prefix, "f32", tau=tau)
    ms, dec = [], []
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        ms.append(int(st.m_updated[0]))
        dec.append(bool(out["recompute"][0]))
    return {"_about": "tiny workload (seed 1000): update count M per step and the "
                      "threshold decision (True = recompute the block-external partial); "
                      "rule: step 0 computes, later steps compute iff M >= tau.",
            "tau": tau, "m_updated": ms, "recompute": dec}


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_tau_trace.json"), "w") as f:
        json.dump(tiny_trace(), f, indent=1)
        f.write("\n")
