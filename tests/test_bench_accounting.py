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
    ns = work["gram"][1] + work["poly"][1] + work["update"][1]
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
    # the fused last update: one iteration's 2 m^2 n and 8 B of fp32 weight per element
    per_iter = sum(2 * min(m.rows, m.cols) ** 2 * max(m.rows, m.cols) for m in w.mats)
    assert work["update_apply"] == ("mixed", (per_iter, elems * 8))


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
