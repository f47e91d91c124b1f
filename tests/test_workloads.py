"""The seeded input generator: deterministic, chunk-independent, and with the
distributions and structure each workload states (no GPU)."""
import numpy as np

import workloads as W


def test_counter_based_draws_are_chunk_independent():
    key = W.stream_key(5, W.STREAM_X)
    whole = W.normals(key, 0, 1001)
    parts = np.concatenate([W.normals(key, 0, 333), W.normals(key, 333, 1), W.normals(key, 334, 667)])
    assert np.array_equal(whole, parts)


def test_splitmix64_published_vector():
    # splitmix64 seeded with 0: first outputs of the reference generator
    # (x += 0x9E3779B97F4A7C15; mix) -- counter draw n of key 0.
    d = W.draws(0, 0, 3)
    assert [int(v) for v in d] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_distributions_and_determinism():
    w = W.small_workload(512, 1024, seed=1, sigma_x=1.5, sigma_grad_y=1e-3)
    x, gy = W.make_inputs(w)
    x2, gy2 = W.make_inputs(w)
    assert np.array_equal(x, x2) and np.array_equal(gy, gy2)
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    gf = W.bf16_bits_to_f32(gy).astype(np.float64)
    assert abs(xf.std() - 1.5) < 0.01 and abs(xf.mean()) < 0.01
    assert abs(gf.std() - 1e-3) < 1e-5
    # streams are distinct
    assert not np.array_equal(x[:, :1024].ravel()[:1000], gy.ravel()[:1000])


def test_outliers_and_zero_groups():
    w = W.Workload("t", 640, 512, 1.0, 0.02, 3, outlier_frac=1e-2, zero_group_every=64)
    x, gy = W.make_inputs(w)
    xf = W.bf16_bits_to_f32(x)
    frac = (np.abs(xf) > 6).mean()
    assert 0.005 < frac < 0.012   # ~1% times P(|50 z| > 6)
    for r, j in W.zero_group_positions(w):
        assert not x[r, j * 128:(j + 1) * 128].any()
        assert not x[r, 512 + j * 128:512 + (j + 1) * 128].any()
    assert len(W.zero_group_positions(w)) == 10


def test_algorithmic_bytes():
    w = W.WORKLOADS[4]
    assert w.algorithmic_bytes() == 1_067_974_656
    assert W.WORKLOADS[0].algorithmic_bytes() == 595_968
