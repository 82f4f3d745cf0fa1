import numpy as np

from matrix_orthogonalising_optimizer_03_b200 import workloads as wl


def test_shape_sets():
    assert wl.WORKLOADS["gpt160m"].n_matrices == 72
    assert wl.WORKLOADS["gpt400m"].n_matrices == 144
    assert wl.WORKLOADS["moe_1b"].n_matrices == 6368
    assert wl.WORKLOADS["dense_1p5b"].n_matrices == 168
    assert wl.WORKLOADS["gpt160m"].n_params == 84_934_656
    # algorithmic Newton-Schulz flops of one step (symmetric Gram / polynomial counted once)
    assert abs(wl.workload_ns_flops(wl.WORKLOADS["gpt160m"]) / 1.142e12 - 1) < 2e-3
    assert abs(wl.workload_ns_flops(wl.WORKLOADS["dense_1p5b"]) / 4.511e13 - 1) < 2e-3


def test_generator_is_deterministic_and_bf16_exact():
    w = wl.WORKLOADS["gpt160m"]
    spec = w.matrices()[60]
    g1, g2 = wl.grad(w, spec, 3), wl.grad(w, spec, 3)
    assert np.array_equal(g1, g2)
    assert not np.array_equal(g1, wl.grad(w, spec, 4))
    assert np.array_equal(wl.bf16_round(g1), g1)
    assert g1.shape == (spec.rows, spec.cols)
    assert abs(g1.std() / 1e-3 - 1) < 0.01
    W = wl.weight(w, spec)
    assert abs(W.std() / 0.02 - 1) < 0.01


def test_bf16_round_ties_to_even():
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-3], dtype=np.float32)
    r = wl.bf16_round(x)
    assert r[0] == 1.0 and r[1] == 1.0 + 2 ** -6 and r[2] == -2.5
    assert abs(r[3] - 1e-3) <= 1e-3 * 2 ** -8
    assert np.array_equal(wl.bf16_bits(np.float32([1.0])), np.uint16([0x3F80]))
