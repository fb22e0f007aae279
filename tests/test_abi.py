"""The C-ABI library without a GPU: it builds, loads, exports every symbol
include/muon.h declares, and its host-side logic (defaults, argument checks,
workspace planning) behaves.  No compute call is made."""

import ctypes
import os
import re

import pytest

import pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mx():
    from matrix_aware_optimizer_step_b200 import build
    build.build()
    import matrix_aware_optimizer_step_b200 as m
    return m


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "muon.h")).read()
    return sorted(set(re.findall(r"MUON_API\s+[\w\s\*]+?\b(muon_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for must in ("muon_init", "muon_step", "muon_adamw_step", "muon_newton_refresh",
                 "muon_orthogonalize", "muon_destroy", "muon_last_error"):
        assert must in names


PAGE_TITLES = ("Muon: An optimizer for the hidden layers of neural networks",
               "Muon: when the LLM optimizer treats weight matrices as",
               "The Newton-Muon Optimizer")


def declaration_comments():
    """(name, comment text) of every MUON_API declaration: the comment block
    that ends right above it (or above the declaration before it, for a
    pair declared back to back)."""
    src = open(os.path.join(ROOT, "include", "muon.h")).read()
    out = []
    for m in re.finditer(r"MUON_API\s+[\w\s\*]+?\b(muon_\w+)\s*\(", src):
        head = src[:m.start()]
        end = head.rstrip().rfind("*/")
        start = head.rfind("/*", 0, end)
        between = head[end + 2:]
        assert end >= 0 and start >= 0 and between.count(";") == 0, m.group(1)
        out.append((m.group(1), " ".join(head[start:end].split())))
    return out


def test_every_declaration_cites_its_source():
    """Each entry point's comment names the page and section that define the
    operation, or says that the pages have no counterpart."""
    found = declaration_comments()
    assert {n for n, _ in found} == set(declared_symbols())
    for name, text in found:
        cited = any(t in text for t in PAGE_TITLES)
        assert cited or "No counterpart on the pages" in text, name
    must_cite = {"muon_init", "muon_step", "muon_adamw_step", "muon_newton_refresh",
                 "muon_newton_precondition", "muon_orthogonalize", "muon_default_hparams"}
    for name, text in found:
        if name in must_cite:
            assert any(t in text for t in PAGE_TITLES), name


def test_library_exports_every_declared_symbol(mx):
    lib = mx.load_library()
    names = declared_symbols()
    assert set(names) == set(mx.binding.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def test_defaults_match_the_pages(mx):
    g = pins.read_golden("defaults.txt")
    q = pins.read_golden("quintic_coefficients.txt")
    hp = mx.default_hparams()
    assert abs(hp.lr - g["muon.lr"]) < 1e-9 and abs(hp.weight_decay - g["muon.weight_decay"]) < 1e-9
    assert abs(hp.momentum - g["muon.momentum"]) < 1e-7 and hp.nesterov == 1
    assert hp.ns_steps == int(q["ns_steps"])
    for name, key in (("ns_a", "a"), ("ns_b", "b"), ("ns_c", "c")):
        assert abs(getattr(hp, name) - q[key]) < 1e-6
    a = mx.default_adamw_hparams()
    assert abs(a.lr - g["adamw.lr"]) < 1e-10 and abs(a.beta1 - g["adamw.beta1"]) < 1e-7
    assert abs(a.beta2 - g["adamw.beta2"]) < 1e-7 and abs(a.weight_decay - g["adamw.weight_decay"]) < 1e-9


def test_status_strings(mx):
    lib = mx.load_library()
    for code, name in [(0, "MUON_OK"), (1, "MUON_ERR_INVALID_ARG"), (3, "MUON_ERR_WORKSPACE"),
                       (5, "MUON_ERR_NONFINITE"), (6, "MUON_ERR_TIMEOUT")]:
        assert lib.muon_status_string(code).decode() == name
    assert lib.muon_last_error(None).decode() == "NULL context"


def _group(mx, rows, cols, count, dtype=1, keep=None):
    g = mx.binding.Group()
    g.rows, g.cols, g.count, g.grad_dtype = rows, cols, count, dtype
    arr = (ctypes.c_void_p * count)(*([256] * count))   # non-null dummies, never dereferenced
    keep.append(arr)
    g.weights = g.grads = g.momentum = ctypes.cast(arr, ctypes.c_void_p)
    return g


def test_query_workspace_plans_wide_layout(mx):
    """Workspace = per shape run: two wide bf16 X buffers (m x ld_n) and the
    symmetric A, B (m x ld_m); plus one fp32 norm per matrix and one fp32
    partial per 64x64 tile; 256-byte aligned regions.  Tall
    matrices share the run of their transpose."""
    lib = mx.load_library()
    keep = []
    arr = (mx.binding.Group * 3)()
    arr[0] = _group(mx, 768, 3072, 12, keep=keep)
    arr[1] = _group(mx, 3072, 768, 12, keep=keep)
    arr[2] = _group(mx, 768, 768, 48, keep=keep)
    n = ctypes.c_size_t()
    assert lib.muon_query_workspace(arr, 3, ctypes.byref(n)) == 0

    def r256(x):
        return (x + 255) // 256 * 256
    tiles = 24 * 576 + 48 * 144           # 64x64 tiles: one fp32 partial norm each
    want = r256(72 * 4) + r256(tiles * 4)
    want += 2 * r256(24 * 768 * 3072 * 2) + 2 * r256(24 * 768 * 768 * 2)
    want += 2 * r256(48 * 768 * 768 * 2) + 2 * r256(48 * 768 * 768 * 2)
    assert n.value == want
    # ragged: leading dimensions padded to a multiple of 8 elements
    arr1 = (mx.binding.Group * 1)()
    arr1[0] = _group(mx, 5, 3, 1, keep=keep)
    assert lib.muon_query_workspace(arr1, 1, ctypes.byref(n)) == 0
    assert n.value == r256(4) + r256(4) + 2 * r256(3 * 8 * 2) + 2 * r256(3 * 8 * 2)


def test_query_workspace_rejects_bad_groups(mx):
    lib = mx.load_library()
    keep = []
    n = ctypes.c_size_t()
    arr = (mx.binding.Group * 1)()
    arr[0] = _group(mx, 0, 5, 1, keep=keep)
    assert lib.muon_query_workspace(arr, 1, ctypes.byref(n)) == 1
    arr[0] = _group(mx, 4, 5, 1, dtype=7, keep=keep)
    assert lib.muon_query_workspace(arr, 1, ctypes.byref(n)) == 1
    arr[0] = _group(mx, 4, 5, 1, keep=keep)
    arr[0].grads = None
    assert lib.muon_query_workspace(arr, 1, ctypes.byref(n)) == 1
    arr[0] = _group(mx, 4, 6, 1, keep=keep)
    p = (ctypes.c_void_p * 1)(256)
    keep.append(p)
    arr[0].precond = ctypes.cast(p, ctypes.c_void_p)
    arr[0].precond_blocks = 4          # 4 does not divide 6
    assert lib.muon_query_workspace(arr, 1, ctypes.byref(n)) == 1
    assert lib.muon_query_workspace(arr, -1, ctypes.byref(n)) == 1


def test_init_without_device_fails_cleanly(mx):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    lib = mx.load_library()
    ctx = ctypes.c_void_p()
    assert lib.muon_init(ctypes.byref(ctx), 0, 0) != 0
    assert not ctx.value


def test_product_path_does_not_touch_the_oracle():
    """The library package never imports the oracle (no CPU fallback)."""
    pkg = os.path.join(ROOT, "matrix_aware_optimizer_step_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.lower(), f


def test_binding_structs_match_the_header(tmp_path):
    """Every ctypes struct of the binding has the size and field offsets the
    C compiler gives the matching struct of include/muon.h (a host program
    built with gcc prints them; no GPU involved)."""
    import ctypes
    import shutil
    import subprocess
    from matrix_aware_optimizer_step_b200 import binding as b
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    pairs = {"muon_hparams": b.Hparams, "muon_group": b.Group, "muon_ns_group": b.NsGroup,
             "muon_adamw_tensor": b.AdamwTensor, "muon_adamw_hparams": b.AdamwHparams,
             "muon_act_desc": b.ActDesc, "muon_kernel_times": b.KernelTimes}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "muon.h"', "int main(void) {"]
    for cname, cls in pairs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    inc = os.path.join(ROOT, "include")
    subprocess.run(["gcc", "-std=c99", "-I", inc, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {}
    for ln in out:
        if ln:
            parts = ln.split()
            got[(parts[0], parts[1])] = int(parts[2])
    for cname, cls in pairs.items():
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for fname, _ in cls._fields_:
            assert got[(cname, fname)] == getattr(cls, fname).offset, (cname, fname)
