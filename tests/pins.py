"""Pins of the fp64 oracle to facts fixed outside it.

Each ``pin_*`` takes an oracle module and raises AssertionError when the
oracle disagrees with a fact it cannot have produced itself: numbers printed
on the pages (golden fixtures), closed forms, invariants of the mathematics,
brute force on tiny inputs, or a black-box library routine run on the CPU.
They are plain functions so the mutation tests can run them against oracles
with a planted mistake.
"""

from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = [float(x) for x in v] if len(v) > 1 else float(v[0])
    return vals


def _p_scalar(s, a, b, c):
    # Scalar quintic written out with Python floats, independent of NumPy.
    return a * s + b * s * s * s + c * s * s * s * s * s


def _p_iter(s, steps, a, b, c):
    for _ in range(steps):
        s = _p_scalar(s, a, b, c)
    return s


# ---------------------------------------------------------------------------
# Newton-Schulz
# ---------------------------------------------------------------------------

def pin_coefficients(o):
    """The printed coefficients and the default step count."""
    g = read_golden("quintic_coefficients.txt")
    assert (o.NS_A, o.NS_B, o.NS_C) == (g["a"], g["b"], g["c"]), "coefficients"
    assert abs(o.quintic_scalar(1.0) - g["p_at_1"]) < 1e-12, "p(1)"
    assert o.muon_defaults()["ns_steps"] == int(g["ns_steps"])


def pin_defaults(o):
    g = read_golden("defaults.txt")
    m, a = o.muon_defaults(), o.adamw_defaults()
    assert m["lr"] == g["muon.lr"] and m["weight_decay"] == g["muon.weight_decay"]
    assert m["momentum"] == g["muon.momentum"] and bool(m["nesterov"]) == bool(g["muon.nesterov"])
    assert a["lr"] == g["adamw.lr"] and a["weight_decay"] == g["adamw.weight_decay"]
    assert (a["beta1"], a["beta2"]) == (g["adamw.beta1"], g["adamw.beta2"])


def pin_diagonal(o):
    """A diagonal input is mapped entrywise by the iterated scalar quintic of
    its normalised diagonal (square and both rectangular orientations)."""
    rng = np.random.default_rng(11)
    for shape in [(6, 6), (4, 7), (7, 4), (1, 1), (1, 5)]:
        k = min(shape)
        d = rng.uniform(0.05, 2.0, size=k) * rng.choice([-1.0, 1.0], size=k)
        g = np.zeros(shape)
        g[np.arange(k), np.arange(k)] = d
        out = o.newton_schulz(g, 5)
        nrm = math.sqrt(sum(float(x) * float(x) for x in d)) + 1e-7
        want = np.zeros(shape)
        for i in range(k):
            want[i, i] = _p_iter(float(d[i]) / nrm, 5, 3.4445, -4.7750, 2.0315)
        err = np.abs(out - want).max()
        assert err < 1e-12, f"diagonal {shape}: {err}"
    # Steps other than five follow the same scalar map.
    d = np.array([0.3, 1.0, 0.01])
    for steps in (0, 1, 2, 7):
        out = o.newton_schulz(np.diag(d), steps)
        nrm = math.sqrt(float(d @ d)) + 1e-7
        want = [_p_iter(x / nrm, steps, 3.4445, -4.7750, 2.0315) for x in d]
        assert np.abs(np.diag(out) - want).max() < 1e-12, f"steps {steps}"


def pin_svd(o):
    """p(X) = U p(S) V^T: brute-force SVD of tiny random matrices."""
    rng = np.random.default_rng(12)
    for shape in [(4, 4), (5, 8), (8, 5), (16, 16), (3, 9)]:
        g = rng.standard_normal(shape)
        u, s, vt = np.linalg.svd(g, full_matrices=False)
        nrm = np.linalg.norm(g) + 1e-7
        f = np.array([_p_iter(x / nrm, 5, 3.4445, -4.7750, 2.0315) for x in s])
        want = (u * f) @ vt
        out = o.newton_schulz(g, 5)
        err = np.linalg.norm(out - want) / np.linalg.norm(want)
        assert err < 1e-12, f"svd {shape}: {err}"


def pin_band(o):
    """Singular values whose normalised size is at least 1e-2 land in the
    quintic's band (about 0.68 to 1.13), and the blog's worked example
    diag(20, 3, 0.2) comes out with equalised magnitudes and its singular
    vectors kept."""
    rng = np.random.default_rng(13)
    for shape in [(32, 32), (24, 40)]:
        g = rng.standard_normal(shape)
        s_in = np.linalg.svd(g, compute_uv=False) / (np.linalg.norm(g) + 1e-7)
        s_out = np.linalg.svd(o.newton_schulz(g, 5), compute_uv=False)
        # both sorted descending, and p^5 is monotone on the relevant range
        # only piecewise, so compare as sets restricted to s_in >= 1e-2
        sel = s_in >= 1e-2
        u, _, vt = np.linalg.svd(g, full_matrices=False)
        out = o.newton_schulz(g, 5)
        proj = np.diag(u.T @ out @ vt.T)
        assert np.all((proj[sel] > 0.68) & (proj[sel] < 1.135)), proj[sel]
        assert s_out.max() < 1.21
    sig = read_golden("worked_example_singular_values.txt")["sigma"]
    q1, _ = np.linalg.qr(rng.standard_normal((3, 3)))
    q2, _ = np.linalg.qr(rng.standard_normal((3, 3)))
    g = q1 @ np.diag(sig) @ q2.T
    out = o.newton_schulz(g, 5)
    proj = q1.T @ out @ q2
    off = proj - np.diag(np.diag(proj))
    assert np.abs(off).max() < 1e-12, "singular vectors kept"
    assert np.all((np.diag(proj) > 0.68) & (np.diag(proj) < 1.135)), np.diag(proj)


def pin_transpose_and_scale(o):
    rng = np.random.default_rng(14)
    for shape in [(6, 10), (10, 6), (9, 9)]:
        g = rng.standard_normal(shape)
        a = o.newton_schulz(g, 5)
        b = o.newton_schulz(g.T, 5)
        assert np.abs(a - b.T).max() < 1e-12, "transpose symmetry"
        c = o.newton_schulz(37.5 * g, 5)
        assert np.abs(a - c).max() < 1e-6, "scale invariance"
        assert a.shape == shape


def pin_zero_grad(o):
    """A zero update leaves only the decay: NS(0) = 0 thanks to eps."""
    w = np.ones((4, 6))
    w1, buf, out = o.muon_step(w, np.zeros((4, 6)), np.zeros((4, 6)))
    assert np.all(out == 0) and np.all(buf == 0)
    assert np.allclose(w1, 1.0 - 0.02 * 0.01)


# ---------------------------------------------------------------------------
# Momentum, scale, apply
# ---------------------------------------------------------------------------

def pin_momentum_closed_form(o):
    """Constant gradient from a zero buffer: buf_k = (1 - beta^k) g and the
    Nesterov look-ahead u_k = (1-beta) g + beta buf_k."""
    g = np.array([[1.5, -2.0], [0.25, 4.0]])
    beta = 0.95
    buf = np.zeros_like(g)
    for k in range(1, 6):
        buf, u = o.nesterov_momentum(g, buf, beta, True)
        assert np.allclose(buf, (1 - beta ** k) * g, rtol=1e-14, atol=0)
        assert np.allclose(u, (1 - beta) * g + beta * (1 - beta ** k) * g, rtol=1e-14, atol=0)
    buf2, u2 = o.nesterov_momentum(g, np.zeros_like(g), beta, False)
    assert np.array_equal(buf2, u2)


def pin_apply_closed_form(o):
    w = np.array([[2.0, -1.0]])
    out = np.array([[0.5, 0.25]])
    got = o.apply_update(w, out, lr=0.1, weight_decay=0.5, scale=3.0)
    # hand arithmetic: w*(1-0.05) - 0.3*o
    assert np.allclose(got, [[2.0 * 0.95 - 0.15, -0.95 - 0.075]], rtol=1e-15)


def pin_shape_scale(o):
    assert o.shape_scale(3072, 768, "original") == 2.0
    assert o.shape_scale(768, 3072, "original") == 1.0
    assert o.shape_scale(256, 256, "original") == 1.0
    assert abs(o.shape_scale(768, 3072, "match_rms_adamw") - 0.2 * math.sqrt(3072)) < 1e-12
    assert abs(o.shape_scale(4096, 1024, "match_rms_adamw") - 12.8) < 1e-12
    assert o.shape_scale(5, 3, "none") == 1.0


def pin_torch_muon(o):
    """Black-box cross-check against torch.optim.Muon run on the CPU in
    float64.  Its momentum buffer must agree to rounding; its update agrees
    to its own bf16 Newton-Schulz error (about 1e-2)."""
    import torch
    torch.manual_seed(3)
    for rows, cols, mode in [(48, 48, None), (72, 36, "original"), (36, 72, "match_rms_adamw")]:
        w0 = torch.randn(rows, cols, dtype=torch.float64) * 0.02
        p = torch.nn.Parameter(w0.clone())
        opt = torch.optim.Muon([p], lr=0.02, weight_decay=0.01, adjust_lr_fn=mode)
        buf = np.zeros((rows, cols))
        w = w0.numpy().copy()
        hp = dict(scale=mode or "original")
        for step in range(3):
            g = torch.randn(rows, cols, dtype=torch.float64)
            p.grad = g.clone()
            opt.step()
            w_prev = w
            w, buf, _ = o.muon_step(w, g.numpy(), buf, hp)
            tb = opt.state[p]["momentum_buffer"].numpy()
            assert np.abs(tb - buf).max() < 1e-14, "momentum buffer"
            d_t = p.detach().numpy() - w_prev * (1 - 0.02 * 0.01)
            d_o = w - w_prev * (1 - 0.02 * 0.01)
            rel = np.linalg.norm(d_t - d_o) / np.linalg.norm(d_o)
            assert rel < 3e-2, f"update {rows}x{cols} {mode}: {rel}"
            p.data.copy_(torch.from_numpy(w))   # keep both on the oracle's weights


# ---------------------------------------------------------------------------
# AdamW
# ---------------------------------------------------------------------------

def pin_adamw(o):
    """Closed form of the first step, then black-box torch.optim.AdamW
    (float64, CPU) over several steps."""
    import torch
    g = np.array([0.5, -2.0, 1e-3, 0.0])
    w0 = np.array([1.0, 2.0, -3.0, 4.0])
    w1, m, v = o.adamw_step(w0, g, np.zeros(4), np.zeros(4), 1)
    want = w0 * (1 - 3e-4 * 0.01) - 3e-4 * g / (np.abs(g) + 1e-8)
    assert np.allclose(w1, want, rtol=1e-14, atol=1e-18)
    torch.manual_seed(4)
    p = torch.nn.Parameter(torch.randn(64, dtype=torch.float64))
    opt = torch.optim.AdamW([p], lr=3e-4, betas=(0.9, 0.95), weight_decay=0.01, eps=1e-8)
    w, m, v = p.detach().numpy().copy(), np.zeros(64), np.zeros(64)
    for step in range(1, 6):
        gr = torch.randn(64, dtype=torch.float64)
        p.grad = gr.clone()
        opt.step()
        w, m, v = o.adamw_step(w, gr.numpy(), m, v, step)
        assert np.abs(p.detach().numpy() - w).max() < 1e-14, f"adamw step {step}"
        assert np.abs(opt.state[p]["exp_avg"].numpy() - m).max() < 1e-15
        assert np.abs(opt.state[p]["exp_avg_sq"].numpy() - v).max() < 1e-15


# ---------------------------------------------------------------------------
# Newton-Muon
# ---------------------------------------------------------------------------

def pin_second_moment(o):
    """S = X^T X / N against explicit triple loops on a tiny input."""
    rng = np.random.default_rng(15)
    x = rng.standard_normal((7, 3))
    got = o.second_moment(x)
    for i in range(3):
        for j in range(3):
            acc = 0.0
            for t in range(7):
                acc += float(x[t, i]) * float(x[t, j])
            assert abs(got[i, j] - acc / 7) < 1e-14


def pin_newton(o):
    rng = np.random.default_rng(16)
    x = rng.standard_normal((64, 6))
    s = o.second_moment(x)
    si = o.spd_inverse(s)
    assert np.abs(s @ si - np.eye(6)).max() < 1e-12, "S S^-1 = I"
    assert np.abs(o.spd_inverse(np.eye(4), damping=1.0) - 0.5 * np.eye(4)).max() < 1e-15
    g = rng.standard_normal((5, 6))
    # S = I reduces Newton-Muon to Muon
    w = rng.standard_normal((5, 6))
    buf = rng.standard_normal((5, 6))
    a = o.newton_muon_step(w, g, buf, [np.eye(6)])
    b = o.muon_step(w, g, buf)
    for x1, x2 in zip(a, b):
        assert np.abs(x1 - x2).max() < 1e-15
    # diagonal S^-1 scales columns
    dg = np.array([1.0, 2.0, 0.5, 4.0, 3.0, 0.25])
    pg = o.right_precondition(g, [np.diag(dg)])
    assert np.abs(pg - g * dg[None, :]).max() < 1e-15
    # block diagonal: four blocks equal the full block-diagonal matrix
    d = 3
    blocks = [o.spd_inverse(o.second_moment(rng.standard_normal((40, d)))) for _ in range(4)]
    g4 = rng.standard_normal((5, 4 * d))
    full = np.zeros((4 * d, 4 * d))
    for k, bk in enumerate(blocks):
        full[k * d:(k + 1) * d, k * d:(k + 1) * d] = bk
    assert np.abs(o.right_precondition(g4, blocks) - g4 @ full).max() < 1e-13
    # precondition happens on the raw gradient, before momentum
    s_inv = [np.diag(dg)]
    w1, b1, _ = o.newton_muon_step(w, g, buf, s_inv)
    assert np.abs(b1 - (0.95 * buf + 0.05 * (g * dg[None, :]))).max() < 1e-15


def pin_flops(o):
    """4 m^2 n + 2 m^3 per iteration: X X^T is 2 m^2 n, A A is 2 m^3 and
    B X is 2 m^2 n multiply-adds-as-two-flops."""
    assert o.ns_nominal_flops(256, 256, 5) == 5 * 6 * 256 ** 3
    assert o.ns_nominal_flops(3072, 768, 1) == 4 * 768 * 768 * 3072 + 2 * 768 ** 3
    assert o.ns_nominal_flops(768, 3072, 1) == o.ns_nominal_flops(3072, 768, 1)


ALL_PINS = [pin_coefficients, pin_defaults, pin_diagonal, pin_svd, pin_band,
            pin_transpose_and_scale, pin_zero_grad, pin_momentum_closed_form,
            pin_apply_closed_form, pin_shape_scale, pin_torch_muon, pin_adamw,
            pin_second_moment, pin_newton, pin_flops]
