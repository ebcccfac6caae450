"""Writes tests/golden/oracle_small_cases.json by calling only the oracle package.

The stored expected values come from the fp64 oracle (after its pins pass) on small seeded
workloads from gated_linear_recurrence_conv1d_b200.inputs; they freeze the oracle's output so
that a later change to its arithmetic shows up as a failing regression test.
Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from gated_linear_recurrence_conv1d_b200 import inputs  # noqa: E402

CASES = [
    dict(name="f32_T8", base="tiny_f32", batch=1, seq_len=8, heads=2, head_dim=16, seed=123),
    dict(name="bf16_T8_resets", base="packed_bf16", batch=2, seq_len=8, heads=2, head_dim=16,
         seed=321, doc_len=(2, 5)),
]


def make_case(c):
    kw = dict(batch=c["batch"], seq_len=c["seq_len"], heads=c["heads"], head_dim=c["head_dim"])
    if "doc_len" in c:
        kw["doc_len"] = tuple(c["doc_len"])
    wl = inputs.WORKLOADS[c["base"]].scaled(**kw)
    prob = inputs.make_problem(wl, seed=c["seed"])
    out, h, tail = oracle.prefill(prob.params, prob.x, prob.y, wl.heads, reset=prob.reset)
    return wl, prob, out, h, tail


def main():
    cases = []
    for c in CASES:
        wl, prob, out, h, tail = make_case(c)
        cases.append(dict(c, out=[float(v) for v in out.ravel()], h=[float(v) for v in h.ravel()]))
    with open(os.path.join(HERE, "oracle_small_cases.json"), "w") as f:
        json.dump(dict(_note="fp64 oracle outputs; written by tests/golden/make_golden.py",
                       cases=cases), f, indent=0)


if __name__ == "__main__":
    main()
