"""Write the oracle's regression records into tests/golden/.

The pages ("kernelgen-challenge-9-task3-silu-quant") print no worked example
for this op, so no stored value here comes from them.  These records come
from the CPU oracle alone (this script imports only ``oracle`` and
``workloads``); they do not pin the oracle -- the pins live in
tests/test_oracle_pins.py -- they only make any later change to the oracle's
arithmetic visible: if a record stops matching, the commit that changes the
oracle regenerates it and names the passage, or the reading of it, that
justifies the change.

    python tests/golden/make_golden.py
"""
from __future__ import annotations

import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads as W  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))
CASES = [W.WORKLOADS[0], W.small_workload(200, 384, seed=3),
         W.small_workload(129, 256, seed=9, outlier_frac=0.01, zero_group_every=16)]


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def record(w: W.Workload) -> dict:
    x, gy = W.make_inputs(w)
    giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy, w.group_size)
    rng = np.random.default_rng(0)
    idx_gi = [(int(rng.integers(w.M)), int(rng.integers(2 * w.K))) for _ in range(8)]
    idx_y = [(int(rng.integers(w.K)), int(rng.integers(w.M))) for _ in range(8)]
    return {
        "workload": w.describe(),
        "inputs_sha256": {"x": digest(x), "grad_y": digest(gy)},
        "outputs_sha256": {"grad_input_q": digest(giq), "grad_input_s": digest(gis),
                           "y_q_t": digest(yqt), "y_s_t": digest(yst)},
        "samples": {
            "grad_input_q": [[m, c, int(giq[m, c])] for m, c in idx_gi],
            "grad_input_s": [[m, c // w.group_size, float(gis[m, c // w.group_size])] for m, c in idx_gi],
            "y_q_t": [[k, t, int(yqt[k, t])] for k, t in idx_y],
            "y_s_t": [[k, t // w.group_size, float(yst[k, t // w.group_size])] for k, t in idx_y],
        },
    }


# grad_y handed over as INT8 codes + fp32 scales (workloads.quantized_grad_y)
QGRAD_CASES = [W.small_workload(200, 384, seed=5, zero_group_every=7),
               W.small_workload(129, 256, seed=11, zero_group_every=3)]


def record_qgrad(w: W.Workload) -> dict:
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w)
    outs = oracle.silu_dot_fwd_bwd_quant_fuse_qgrad(x, q, s, w.group_size)
    y = oracle.swiglu_bwd_bf16_dy(x, oracle.dequant_grad_y(q, s))[0]
    names = ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")
    return {
        "workload": w.describe(),
        "inputs_sha256": {"x": digest(x), "grad_y_q": digest(q), "grad_y_s": digest(s)},
        "outputs_sha256": dict({n: digest(a) for n, a in zip(names, outs)}, y=digest(y)),
    }


def main() -> None:
    out = {"source": "CPU oracle (oracle/sdq_oracle.cpp) on workloads.make_inputs; "
                     "regression record only, not a pin",
           "cases": [record(w) for w in CASES],
           "qgrad_cases": [record_qgrad(w) for w in QGRAD_CASES]}
    with open(os.path.join(HERE, "oracle_records.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
