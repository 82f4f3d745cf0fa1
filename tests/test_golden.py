"""Values the pages print, stored under tests/golden/ with their citations, against the
oracle's defaults and arithmetic, the C ABI's muon_hparams_default and the binding's
defaults. CPU only: the library is loaded, no kernel runs."""
import ctypes
import inspect
import json
import os

import numpy as np
import pytest

from oracle import muon_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def host_lib():
    """libmuon.so loaded on the host (its host functions need no GPU)."""
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    from matrix_orthogonalising_optimizer_03_b200 import build as build_mod
    build_mod.build()
    return B.load()


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        d = json.load(f)
    assert d["source"]
    return d


def test_muon_defaults_match_the_printed_listing():
    g = _load("muon_defaults.json")
    hp = orc.HParams()
    assert tuple(hp.ns_coeffs) == tuple(g["ns_coeffs"])
    assert orc.QUINTIC == tuple(g["ns_coeffs"])
    assert hp.ns_steps == g["ns_steps"]
    assert hp.eps == g["eps"]
    assert hp.lr == g["lr"] and hp.momentum == g["momentum"]
    assert hp.nesterov is g["nesterov"] and hp.weight_decay == g["weight_decay"]


def test_c_abi_and_binding_defaults_match_the_printed_listing(host_lib):
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    g = _load("muon_defaults.json")
    hp = B.MuonHParams()
    assert host_lib.muon_hparams_default(ctypes.byref(hp)) == 0
    f32 = lambda x: float(np.float32(x))
    assert [hp.ns_coeffs[i] for i in range(3)] == [f32(v) for v in g["ns_coeffs"]]
    assert hp.ns_steps == g["ns_steps"]
    assert hp.eps == f32(g["eps"]) and hp.lr == f32(g["lr"]) and hp.momentum == f32(g["momentum"])
    assert hp.weight_decay == f32(g["weight_decay"])
    assert bool(hp.flags & B.MUON_NESTEROV) is g["nesterov"]
    sig = inspect.signature(B.hparams).parameters
    assert tuple(sig["ns_coeffs"].default) == tuple(g["ns_coeffs"])
    for key in ("ns_steps", "eps", "lr", "momentum", "weight_decay", "nesterov"):
        assert sig[key].default == g[key], key


def test_moonlight_update_rms():
    """An orthogonalised full-rank [A, B] update has RMS sqrt(1/max(A, B)); the scale
    0.2 sqrt(max(A, B)) brings it to 0.2."""
    g = _load("moonlight_scale.json")
    assert orc.HParams().scale_k == g["scale_k"]
    rng = np.random.default_rng(5)
    for case in g["cases"]:
        rows, cols = case["shape"]
        O = orc.polar_factor(rng.standard_normal((rows, cols)))
        rms = np.sqrt(np.mean(O * O))
        assert rms == pytest.approx(case["raw_rms"], rel=1e-10)
        s = orc.update_scale(rows, cols, "moonlight", g["scale_k"])
        assert s * rms == pytest.approx(case["scaled_rms"], rel=1e-10)


def test_qk_clip_threshold_and_powers(host_lib):
    from matrix_orthogonalising_optimizer_03_b200 import binding as B
    g = _load("qk_clip.json")
    assert inspect.signature(orc.qk_clip).parameters["tau"].default == g["tau"]
    assert inspect.signature(B.qk_clip).parameters["tau"].default == g["tau"]
    powers = g["power"]
    for case in g["cases"]:
        W = np.ones((4, 3))
        slices = [(0, 0, 1, 0, powers["query_nonrotary"]), (0, 1, 1, 0, powers["key_nonrotary"]),
                  (0, 2, 1, 0, powers["query_rotary"]), (0, 3, 1, 0, powers["key_rotary_shared"])]
        out = orc.qk_clip([W], slices, [case["s_max"]], g["tau"])[0]
        gam = case["gamma"]
        assert np.allclose(out[0], gam ** 0.5) and np.allclose(out[1], gam ** 0.5)
        assert np.allclose(out[2], gam) and np.allclose(out[3], 1.0)
