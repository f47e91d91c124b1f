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


def test_recorded_traffic_is_keyed_by_the_current_sources(tmp_path, monkeypatch):
    """A traffic record counts only while the kernel sources it was taken on
    stand unchanged: a line under another digest reads as no record."""
    (tmp_path / "k.cuh").write_text("int f() { return 1; }\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_sha(["k.cuh"])
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# workload sha read write write_back\n"
        f"wl_a {sha} 100 20 30\n"
        f"wl_b 0123456789abcdef 100 20 30\n"
        f"wl_c {sha} 100 20\n")
    assert bench.recorded_traffic("wl_a", ["k.cuh"]) == 150
    assert bench.recorded_traffic("wl_b", ["k.cuh"]) is None
    assert bench.recorded_traffic("wl_c", ["k.cuh"]) == 120
    assert bench.recorded_traffic("wl_d", ["k.cuh"]) is None


def test_algorithmic_bytes():
    w = W.BY_NAME["swiglu_bwd_int8_M4096_K1408"]
    assert w.algorithmic_bytes() == 52445184
    assert bench.int8_grad_y_bytes(w) == 52445184 - 4096 * 1408 + 4 * 4096 * 11


def test_buffer_sets_rotate_at_least_three_and_exceed_three_l2():
    """Consecutive timed calls never share buffers, and the sets together
    exceed 3x L2 (no more sets than that needs, beyond the minimum of 3)."""
    l2 = 126 * 2**20
    assert bench.buffer_sets(1_067_974_656, l2) == 3   # one call larger than L2
    for w in W.WORKLOADS:
        per_call = w.algorithmic_bytes()
        n = bench.buffer_sets(per_call, l2)
        assert n >= 3
        assert n * per_call >= 3 * l2
        if n > 3:
            assert (n - 1) * per_call < 3 * l2
