"""The benchmark's work accounting against independent definitions (CPU).

The NS TFLOP/s metric counts 4 m^2 n + 2 m^3 FLOPs per iteration with
m = min(rows, cols) and n = max ("Muon: when the LLM optimizer treats weight
matrices as matrices", section 3: two m x m x n products and one m^3
product per iteration); the oracle's ns_nominal_flops states the same count,
and it is pinned separately against the three products.  The byte counts
follow from the dtypes of what each pass reads and writes.
"""

import importlib.util
import os

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", ["single-256", "gpt2-small", "llama3-8b", "sweep-1024", "newton-gpt2-small"])
def test_ns_flops_match_the_metric_definition(bench, name):
    w, aux = bench.workload_def(name)
    work, elems, aux_el = bench.step_work(w, aux)
    ns = work["gram"][1] + work["poly"][1] + work["update"][1] + work["ns_small"][1]
    assert ns == sum(oracle.ns_nominal_flops(m.rows, m.cols, 5) for m in w.mats)
    assert elems == sum(m.rows * m.cols for m in w.mats)
    assert aux_el == sum(n for _, n in aux)


def test_gpt2_small_counts(bench):
    """72 matrices, 84.93 M hidden parameters, 39.5 M aux; 1.63 TFLOP of
    nominal NS work per step; 12 B per element for the momentum pass with
    bf16 gradients and 26 B per aux element for AdamW."""
    w, aux = bench.workload_def("gpt2-small")
    work, elems, aux_el = bench.step_work(w, aux)
    assert len(w.mats) == 72
    assert elems == 12 * (4 * 768 * 768 + 2 * 3072 * 768)
    assert aux_el == 39505152
    ns = work["gram"][1] + work["poly"][1] + work["update"][1]
    assert abs(ns / 1e12 - 1.63) < 0.01
    assert work["momentum"] == ("byte", elems * 12)
    assert work["adamw"] == ("byte", aux_el * 26)
    # the fused last update: one iteration's 2 m^2 n, and its compulsory
    # bytes: bf16 B' (m = 768 for all 72 matrices) and X read once, fp32 W
    # read and written once (2 m^2 + 2 m n + 8 m n)
    per_iter = sum(2 * min(m.rows, m.cols) ** 2 * max(m.rows, m.cols) for m in w.mats)
    assert work["update_apply"] == ("mixed", (per_iter, 2 * 72 * 768 * 768 + 10 * elems))
    assert 2 * 72 * 768 * 768 + 10 * elems == 934281216


def test_newton_refresh_counts(bench):
    """Per refresh and d-wide block: 2 N d^2 on the tensor cores for
    S = X^T X / N, and d^3/3 FLOPs each for Cholesky, L^-1 and L^-T L^-1;
    amortised over the refresh period."""
    w, aux = bench.workload_def("newton-gpt2-small")
    work, _, _ = bench.step_work(w, aux)
    tc = alu = 0
    for _, tokens, width in w.acts:
        nb = 4 if width > 768 else 1
        d = width // nb
        tc += nb * 2 * tokens * d * d
        alu += nb * d ** 3
    kind, (t_tc, t_alu) = work["newton_refresh"]
    assert kind == "seq"
    assert t_tc == pytest.approx(tc / w.refresh_every)
    assert t_alu == pytest.approx(alu / w.refresh_every, rel=1e-6)


def test_executed_flops_follow_the_tile_enumeration(bench):
    """Executed tensor-core work: whole 256 x 256 pair tiles, the symmetric
    products only on and above the diagonal.  For m a multiple of 256 with
    T = m / 256 tiles per side, executed / nominal is (T + 1) / (2 T) for
    the Gram and polynomial products and 1 for the update."""
    w, aux = bench.workload_def("llama3-8b")
    work, _, _ = bench.step_work(w, aux)
    exe = bench.executed_flops(w)
    assert exe["update"] == work["update"][1]
    # per shape class the ratio is (T+1)/(2T); over the set it is the
    # nominal-weighted mix of those ratios
    want_g = sum(2 * min(m.rows, m.cols) ** 2 * max(m.rows, m.cols) * 5
                 * (min(m.rows, m.cols) // 256 + 1) / (2 * (min(m.rows, m.cols) // 256)) for m in w.mats)
    want_p = sum(2 * min(m.rows, m.cols) ** 3 * 5
                 * (min(m.rows, m.cols) // 256 + 1) / (2 * (min(m.rows, m.cols) // 256)) for m in w.mats)
    assert exe["gram"] == pytest.approx(want_g, rel=1e-12)
    assert exe["poly"] == pytest.approx(want_p, rel=1e-12)


def test_executed_flops_round_ragged_shapes_up_to_tiles(bench):
    """A 300 x 200 matrix (m = 200, n = 300): one 256-tile per side of the
    Gram over K = 320 (300 rounded up to 64), one poly tile over K = 256,
    and two update tiles over K = 256; five iterations."""
    import workloads as wl
    w = wl.Workload("t", [wl.Mat("a", 300, 200)], "f32", 1.0, 0.02, 1)
    exe = bench.executed_flops(w)
    t = 2 * 256 * 256
    assert exe == {"gram": t * 320 * 5, "poly": t * 256 * 5, "update": 2 * t * 256 * 5, "ns_small": 0}


def test_shape_classes_merge_a_shape_with_its_transpose(bench):
    """The oracle orthogonalises a tall matrix through its transpose, so the
    CPU baseline samples one matrix per wide shape: three for Llama-3-8B
    (4096^2 x64, 1024x4096 x64, 4096x14336 x96), two for GPT-2-small."""
    w, _ = bench.workload_def("llama3-8b")
    cls = {k: c for k, _, c in bench.shape_classes(w)}
    assert cls == {(4096, 4096): 64, (1024, 4096): 64, (4096, 14336): 96}
    w, _ = bench.workload_def("gpt2-small")
    cls = {k: c for k, _, c in bench.shape_classes(w)}
    assert cls == {(768, 768): 48, (768, 3072): 24}


def test_small_matrices_form_their_own_class(bench):
    """A 256 x 256 matrix runs every iteration in one launch: its nominal
    FLOPs (6 m^3 per iteration) and its executed work (three 256-tile
    products over K = 256) go to the small-matrix class."""
    w, aux = bench.workload_def("single-256")
    work, _, _ = bench.step_work(w, aux)
    assert work["gram"][1] == work["poly"][1] == work["update"][1] == 0
    assert work["ns_small"][1] == 6 * 256 ** 3 * 5
    assert bench.executed_flops(w)["ns_small"] == 3 * 2 * 256 ** 3 * 5


def test_newton_momentum_counted_with_the_preconditioning(bench):
    """Every GPT-2-small matrix is preconditioned on the tensor cores (block
    width 768), and that product applies the momentum in its epilogue: its
    class carries the algorithmic 2 rows cols d FLOPs and 12 B per element
    (bf16 G read, fp32 buffer read and written, bf16 U written); no
    momentum-kernel bytes remain."""
    w, aux = bench.workload_def("newton-gpt2-small")
    work, elems, _ = bench.step_work(w, aux)
    flops = 0
    for m in w.mats:
        nb = w.precond[m.name][1]
        flops += 2 * m.rows * m.cols * (m.cols // nb)
    assert work["precondition"] == ("mixed", (flops, 12 * elems))
    assert "momentum" not in work
