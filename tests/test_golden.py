"""The oracle still produces its committed regression records (no GPU).

The records are written by tests/golden/make_golden.py from the oracle alone;
the pages print no worked example for this op, so these are change detectors,
not pins (the pins are in test_oracle_pins.py)."""
import json
import os

import numpy as np

import oracle
import workloads as W
from tests.golden.make_golden import CASES, QGRAD_CASES, digest, record_qgrad

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_regression_records():
    rec = json.load(open(os.path.join(HERE, "oracle_records.json")))
    assert len(rec["cases"]) == len(CASES)
    for w, r in zip(CASES, rec["cases"]):
        assert r["workload"] == w.describe()
        x, gy = W.make_inputs(w)
        assert digest(x) == r["inputs_sha256"]["x"], "input generator changed"
        assert digest(gy) == r["inputs_sha256"]["grad_y"], "input generator changed"
        giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy, w.group_size)
        for name, a in (("grad_input_q", giq), ("grad_input_s", gis), ("y_q_t", yqt), ("y_s_t", yst)):
            assert digest(a) == r["outputs_sha256"][name], name
        for m, c, v in r["samples"]["grad_input_q"]:
            assert int(giq[m, c]) == v
        for k, t, v in r["samples"]["y_q_t"]:
            assert int(yqt[k, t]) == v
        for m, j, v in r["samples"]["grad_input_s"]:
            assert float(gis[m, j]) == v
        for k, i, v in r["samples"]["y_s_t"]:
            assert float(yst[k, i]) == v


def test_quantized_grad_y_oracle_matches_regression_records():
    rec = json.load(open(os.path.join(HERE, "oracle_records.json")))
    assert len(rec["qgrad_cases"]) == len(QGRAD_CASES)
    for w, r in zip(QGRAD_CASES, rec["qgrad_cases"]):
        assert record_qgrad(w) == r, w.name
