"""C-ABI library: loads without a GPU, exports every declared symbol, matches the
header's struct layouts, and rejects bad arguments on the host (no CUDA call)."""
import ctypes
import os
import re
import subprocess

import pytest

from matrix_orthogonalising_optimizer_03_b200 import binding as B
from matrix_orthogonalising_optimizer_03_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MUON_API\s+[\w\s\*]+?\b(muon_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    for name in names:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (muon_\w+)", out))
    assert exported == set(names)


def test_struct_layouts_match_c_compiler(tmp_path):
    src = tmp_path / "sizes.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "muon.h"\n'
                   'int main(void){printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(muon_matrix_t),'
                   ' sizeof(muon_hparams_t), sizeof(muon_stats_t), sizeof(muon_ns_matrix_t),'
                   ' offsetof(muon_hparams_t, flags), offsetof(muon_matrix_t, w_dtype));return 0;}\n')
    exe = tmp_path / "sizes"
    subprocess.run(["gcc", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()))
    assert got == [ctypes.sizeof(B.MuonMatrix), ctypes.sizeof(B.MuonHParams),
                   ctypes.sizeof(B.MuonStats), ctypes.sizeof(B.MuonNSMatrix),
                   B.MuonHParams.flags.offset, B.MuonMatrix.w_dtype.offset]


def test_status_strings_and_defaults(lib):
    for code, name in B.STATUS_NAMES.items():
        assert lib.muon_status_string(code).decode() == name
    hp = B.MuonHParams()
    assert lib.muon_hparams_default(ctypes.byref(hp)) == 0
    assert (hp.lr, hp.ns_steps, hp.mode, hp.scale, hp.flags) == (pytest.approx(0.02), 5, 0, 0, 1)
    assert list(hp.ns_coeffs) == pytest.approx([3.4445, -4.7750, 2.0315])
    assert hp.momentum == pytest.approx(0.95) and hp.scale_k == pytest.approx(0.2)


def _mat(w, g, m, rows, cols, ldw=None, ldg=None, ldm=None, wd=0, gd=1):
    return B.MuonMatrix(w, g, m, rows, cols, ldw or cols, ldg or cols, ldm or cols, wd, gd)


def _arr(*ms):
    a = (B.MuonMatrix * len(ms))()
    for i, m in enumerate(ms):
        a[i] = m
    return a


FAKE = 1 << 40  # host-side validation never dereferences device pointers


def test_host_validation_error_codes(lib):
    hp = B.MuonHParams()
    lib.muon_hparams_default(ctypes.byref(hp))
    ok = _mat(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), 64, 128)
    assert lib.muon_validate(_arr(ok), 1, ctypes.byref(hp)) == 0
    assert lib.muon_validate(_arr(ok), 0, ctypes.byref(hp)) == 0
    assert lib.muon_validate(_arr(ok), -1, ctypes.byref(hp)) == 1
    assert lib.muon_validate(_arr(_mat(0, FAKE, FAKE + (1 << 30), 4, 4)), 1, ctypes.byref(hp)) == 1
    assert lib.muon_validate(_arr(_mat(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), 0, 4)), 1,
                             ctypes.byref(hp)) == 2          # "non-2-D" / empty matrix
    assert lib.muon_validate(_arr(_mat(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), 4, 8, ldw=4)), 1,
                             ctypes.byref(hp)) == 2          # ld < cols
    assert lib.muon_validate(_arr(_mat(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), 4, 8, wd=1)), 1,
                             ctypes.byref(hp)) == 3          # W must be fp32
    assert lib.muon_validate(_arr(_mat(FAKE, FAKE + 64, FAKE + (2 << 30), 4, 8)), 1,
                             ctypes.byref(hp)) == 4          # grad overlaps W
    a = _mat(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), 4, 8)
    b = _mat(FAKE + 96, FAKE + (3 << 30), FAKE + (4 << 30), 4, 8)
    assert lib.muon_validate(_arr(a, b), 2, ctypes.byref(hp)) == 4   # W of two matrices overlap
    shared_g = _mat(FAKE + (5 << 30), FAKE + (1 << 30), FAKE + (6 << 30), 4, 8)
    assert lib.muon_validate(_arr(a, shared_g), 2, ctypes.byref(hp)) == 0  # read-only overlap is fine
    bad = B.MuonHParams()
    lib.muon_hparams_default(ctypes.byref(bad))
    bad.ns_steps = -1
    assert lib.muon_validate(_arr(ok), 1, ctypes.byref(bad)) == 1
    bad.ns_steps, bad.mode = 5, 7
    assert lib.muon_validate(_arr(ok), 1, ctypes.byref(bad)) == 1


def test_workspace_size_and_plan_are_host_only(lib):
    hp = B.MuonHParams()
    lib.muon_hparams_default(ctypes.byref(hp))
    mats = [_mat(FAKE + (3 * i) * (1 << 30), FAKE + (3 * i + 1) * (1 << 30),
                 FAKE + (3 * i + 2) * (1 << 30), r, c) for i, (r, c) in
            enumerate([(768, 768), (3072, 768), (768, 3072), (17, 33)])]
    arr = _arr(*mats)
    ws = lib.muon_workspace_size(arr, 4, ctypes.byref(hp))
    # X (two slabs) + S + P in bf16 for each oriented class, plus tables
    slab = 2 * (768 * 768 + 2 * 768 * 3072 + 17 * 64) * 2 + 2 * (768 * 768 * 3 + 17 * 64) * 2
    assert slab <= ws <= slab + (1 << 20)
    plan = ctypes.c_void_p()
    assert lib.muon_plan_create(arr, 4, ctypes.byref(hp), ctypes.byref(plan)) == 0
    assert lib.muon_plan_workspace_size(plan) == ws
    hp2 = B.MuonHParams.from_buffer_copy(hp)
    hp2.lr = 0.01
    assert lib.muon_plan_set_hparams(plan, ctypes.byref(hp2)) == 0
    hp2.flags |= B.MUON_NS_FP32
    assert lib.muon_plan_set_hparams(plan, ctypes.byref(hp2)) == 1   # layout flag change
    assert lib.muon_plan_step(plan, None, 0, None, None) == 5        # no workspace
    lib.muon_plan_destroy(plan)
    hp.flags |= B.MUON_NS_FP32
    assert lib.muon_workspace_size(arr, 4, ctypes.byref(hp)) > ws    # fp32 slabs
    assert lib.muon_workspace_size(arr, 4, None) == 0


def _ns(x, o, rows, cols, ldx=None, ldo=None, dtype=1):
    return B.MuonNSMatrix(x, o, rows, cols, ldx or cols, ldo or cols, dtype, 0)


def _ns_arr(m):
    a = (B.MuonNSMatrix * 1)()
    a[0] = m
    return a


def test_both_newton_schulz_entry_points_give_the_same_status(lib):
    """The workspace entry point and the no-alloc entry point validate through one host
    routine: every bad argument gets the same status from both, before any CUDA call."""
    def hp_with(**kw):
        hp = B.MuonHParams()
        lib.muon_hparams_default(ctypes.byref(hp))
        for k, v in kw.items():
            setattr(hp, k, v)
        return hp

    ok = _ns(FAKE, FAKE + (1 << 30), 64, 96)
    cases = [
        (ok, hp_with(eps=float("inf")), 1), (ok, hp_with(eps=float("nan")), 1),
        (ok, hp_with(eps=-1.0), 1), (ok, hp_with(mode=9), 1), (ok, hp_with(scale=7), 1),
        (ok, hp_with(flags=0x100), 1), (ok, hp_with(ns_steps=-1), 1), (ok, hp_with(ns_steps=65), 1),
        (_ns(0, FAKE, 4, 4), hp_with(), 1), (_ns(FAKE, FAKE + (1 << 30), 0, 4), hp_with(), 2),
        (_ns(FAKE, FAKE + (1 << 30), 4, 8, ldx=4), hp_with(), 2),
        (_ns(FAKE, FAKE + (1 << 30), 4, 8, dtype=5), hp_with(), 3),
        (_ns(FAKE, FAKE + 8, 4, 8), hp_with(), 4),                    # O overlaps X
        (_ns(FAKE + 1, FAKE + (1 << 30), 4, 8), hp_with(), 1),         # misaligned bf16 X
    ]
    for m, hp, want in cases:
        batched = lib.muon_newton_schulz_batched(_ns_arr(m), 1, ctypes.byref(hp), None, 0, None)
        noalloc = lib.muon_newton_schulz_noalloc(ctypes.byref(m), ctypes.byref(hp), None, None)
        assert batched == noalloc == want, (want, batched, noalloc)
    assert lib.muon_newton_schulz_noalloc(None, ctypes.byref(hp_with()), None, None) == 1
    assert lib.muon_newton_schulz_noalloc(ctypes.byref(ok), None, None, None) == 1


class _FakeCudaTensor:
    """Stands in for a CUDA tensor where only attributes are inspected."""

    def __init__(self, dtype, numel, device="cuda:0"):
        import torch
        self.dtype, self._numel, self.is_cuda = dtype, numel, True
        self.device = torch.device(device)

    def numel(self):
        return self._numel

    def data_ptr(self):
        raise AssertionError("a rejected status tensor must never be dereferenced")


def test_noalloc_binding_rejects_bad_status_before_any_launch(lib):
    """A status word that is not a one-element int32/uint32 CUDA tensor raises MuonError
    before the library is called (the kernels would otherwise store through it)."""
    import torch
    hp = B.hparams()
    x = torch.zeros(8, 8, dtype=torch.bfloat16)
    o = torch.zeros(8, 8, dtype=torch.bfloat16)
    bad = [torch.zeros(1, dtype=torch.int32),               # host memory
           _FakeCudaTensor(torch.int64, 1),                  # wrong dtype
           _FakeCudaTensor(torch.float32, 1),
           _FakeCudaTensor(torch.int32, 0)]                  # empty
    for status in bad:
        with pytest.raises(B.MuonError) as e:
            B.newton_schulz_noalloc(x, o, hp, status=status)
        assert e.value.status == 1 and "status" in str(e.value)


def test_qk_clip_plan_rejects_bad_inputs_before_any_launch(lib):
    """QkClipPlan checks its slices and S_max on the host: host-memory weights, weights of
    another dtype or layout, and a host S_max raise MuonError before the library is
    called."""
    import torch
    s_dev = _FakeCudaTensor(torch.float32, 4)
    bad = [[(torch.zeros(8, 8), 0, 4, 0, 0.5)],                       # host weights
           [(torch.zeros(2, 8, 8), 0, 4, 0, 0.5)],                    # not 2-D
           [(torch.zeros(8, 8).t()[:, :4], 0, 4, 0, 0.5)]]            # column-major view
    for slices in bad:
        with pytest.raises(B.MuonError):
            B.QkClipPlan(slices, s_dev)
