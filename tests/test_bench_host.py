"""Host-side pieces of bench.py (no GPU): the kernel-source digest that keys
the recorded ncu traffic, and the algorithmic byte counts."""
from __future__ import annotations

import bench
import workloads as W


def test_digest_ignores_comments_but_not_code(tmp_path, monkeypatch):
    src = "// header\nint f(int a) {  /* why */\n  return a + 1;  // note\n}\n"
    (tmp_path / "k.cuh").write_text(src)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_sha(["k.cuh"])
    (tmp_path / "k.cuh").write_text("// another header\n\n" + src.replace("why", "because"))
    assert bench.kernel_sha(["k.cuh"]) == base
    (tmp_path / "k.cuh").write_text(src.replace("a + 1", "a + 2"))
    assert bench.kernel_sha(["k.cuh"]) != base


def test_recorded_traffic_matches_the_current_sources():
    """The committed ncu traffic record names the digest of the sources as
    they stand, for every bench workload of both kernels."""
    for w in W.WORKLOADS[1:3] + W.WORKLOADS[4:]:
        assert bench.recorded_traffic(w.name) is not None, w.name
        assert bench.recorded_traffic(w.name + "_swiglu_q8_1", bench.FWD_SOURCES) is not None, w.name


def test_algorithmic_bytes():
    w = W.BY_NAME["swiglu_bwd_int8_M4096_K1408"]
    assert w.algorithmic_bytes() == 52445184
    assert bench.int8_grad_y_bytes(w) == 52445184 - 4096 * 1408 + 4 * 4096 * 11
