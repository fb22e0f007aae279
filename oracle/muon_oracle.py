"""Plain fp64 CPU oracle of the Muon optimizer step, its aux AdamW step and the
Newton-Muon right-preconditioner.

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously correct
definition that the CUDA path is checked against.  Only the test-suite, the
smoke check and the CPU-baseline leg of the benchmark may import it; the
library itself never does, and there is no CPU fallback through it.  It shares
no code with the CUDA path.

Everything is NumPy in float64, written step by step in the order the sources
give, with no blocking, fusion or reordering.  Sources, by page title:

* "Muon: An optimizer for the hidden layers of neural networks" (README of the
  KellerJordan/Muon repository): sections "Usage" (param groups, lr 0.02,
  weight_decay 0.01, AdamW lr 3e-4, betas (0.9, 0.95), weight_decay 0.01) and
  "Hyperparameter tuning" (momentum 0.95, nesterov True, ns_steps 5).
* "Muon: when the LLM optimizer treats weight matrices as matrices" (blog):
  section 1 (AdamW moment formulas), section 3 (Frobenius normalisation, the
  quintic Newton-Schulz polynomial and its coefficients, p(X) = U p(S) V^T),
  and the PyTorch set-up after the garbled section 4 (torch.optim.Muon with
  momentum 0.95, nesterov, adjust_lr_fn="match_rms_adamw"; the three shape
  scaling conventions).
* "The Newton-Muon Optimizer" (README of zhehangdu/Newton-Muon): section
  "What Is Newton-Muon?" (right-preconditioning by an inverse activation
  second moment; shared QKV estimate; four-block diagonal for the MLP
  contraction; standard Muon after the refresh/apply step).

Readings where the sources are silent (each one is also listed in the design
notes):

* Momentum uses the exponential-moving-average convention that the blog's
  AdamW formulas use, buf <- beta*buf + (1-beta)*g, and the Nesterov look-ahead
  u = (1-beta)*g + beta*buf.  The classic form (buf <- beta*buf + g) differs by
  the constant factor 1/(1-beta), which Frobenius normalisation removes.
* Normalisation divides by ||G||_F + eps with eps = 1e-7.
* A matrix with more rows than columns is orthogonalised through its
  transpose, so that the Gram matrix X X^T is min(rows, cols) square.
* Shape scale: "original" max(1, rows/cols)^0.5 (the lr 0.02 convention of the
  first page) or "match_rms_adamw" 0.2*sqrt(max(rows, cols)); "none" is 1.
* Weight decay is decoupled and multiplies the old weights in the same step.
* AdamW adds eps 1e-8 to the root of the second moment and corrects both
  moments for bias.
* Newton-Muon: S = X^T X / N from N activation rows, optional damping
  S + lambda*I (default 0), exact inverse, applied to the raw gradient before
  momentum; block b of the four-block variant acts on columns
  [b*d, (b+1)*d).
"""

from __future__ import annotations

import math

import numpy as np

# Section 3 of the blog prints the production coefficients of the quintic.
NS_A = 3.4445
NS_B = -4.7750
NS_C = 2.0315
NS_EPS = 1e-7

SCALE_ORIGINAL = "original"
SCALE_MATCH_RMS_ADAMW = "match_rms_adamw"
SCALE_NONE = "none"


def muon_defaults() -> dict:
    """Defaults of the Muon parameter group (first page, "Usage" and
    "Hyperparameter tuning")."""
    return dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.01,
                ns_steps=5, a=NS_A, b=NS_B, c=NS_C, eps=NS_EPS,
                scale=SCALE_ORIGINAL)


def adamw_defaults() -> dict:
    """Defaults of the aux AdamW group (first page, "Usage")."""
    return dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01)


# ---------------------------------------------------------------------------
# Muon
# ---------------------------------------------------------------------------

def nesterov_momentum(grad, buf, beta=0.95, nesterov=True):
    """One momentum update.  Returns (new_buf, u), u being what is
    orthogonalised.  EMA convention, as the blog writes AdamW's first moment
    (section 1); Nesterov look-ahead when nesterov is set (first page,
    "Hyperparameter tuning")."""
    g = np.asarray(grad, dtype=np.float64)
    new_buf = beta * np.asarray(buf, dtype=np.float64) + (1.0 - beta) * g
    if nesterov:
        u = (1.0 - beta) * g + beta * new_buf
    else:
        u = new_buf.copy()
    return new_buf, u


def quintic_scalar(s, a=NS_A, b=NS_B, c=NS_C):
    """p(s) = a s + b s^3 + c s^5, the map the iteration applies to every
    singular value (blog, section 3)."""
    return a * s + b * s ** 3 + c * s ** 5


def newton_schulz(g, steps=5, a=NS_A, b=NS_B, c=NS_C, eps=NS_EPS):
    """Approximate U V^T of g = U S V^T (blog, section 3).

    X = g / (||g||_F + eps), then `steps` times
        A = X X^T ;  B = b A + c A A ;  X = a X + B X,
    which is X <- a X + b (X X^T) X + c (X X^T)^2 X.  A tall g is handled
    through its transpose so that A is min(rows, cols) square.
    """
    x = np.array(g, dtype=np.float64)
    transposed = x.shape[0] > x.shape[1]
    if transposed:
        x = x.T
    x = x / (np.linalg.norm(x) + eps)
    for _ in range(steps):
        gram = x @ x.T
        poly = b * gram + c * (gram @ gram)
        x = a * x + poly @ x
    return x.T if transposed else x


def shape_scale(rows, cols, mode=SCALE_ORIGINAL):
    """Shape-dependent learning-rate factor (blog, PyTorch set-up after
    section 4: three conventions; the first page's lr 0.02 goes with the
    original one)."""
    if mode == SCALE_ORIGINAL:
        return math.sqrt(max(1.0, rows / cols))
    if mode == SCALE_MATCH_RMS_ADAMW:
        return 0.2 * math.sqrt(max(rows, cols))
    if mode == SCALE_NONE:
        return 1.0
    raise ValueError(f"unknown scale mode {mode!r}")


def apply_update(w, o, lr, weight_decay, scale):
    """Decoupled weight decay and the parameter update:
    W <- W (1 - lr wd) - lr scale O."""
    w = np.asarray(w, dtype=np.float64)
    return w * (1.0 - lr * weight_decay) - lr * scale * np.asarray(o, dtype=np.float64)


def muon_step(w, grad, buf, hp=None):
    """One Muon step of one hidden 2-D weight.  Returns (new_w, new_buf, o),
    o being the orthogonalised update before scale and learning rate."""
    p = muon_defaults()
    if hp:
        p.update(hp)
    w = np.asarray(w, dtype=np.float64)
    rows, cols = w.shape
    new_buf, u = nesterov_momentum(grad, buf, p["momentum"], p["nesterov"])
    o = newton_schulz(u, p["ns_steps"], p["a"], p["b"], p["c"], p["eps"])
    new_w = apply_update(w, o, p["lr"], p["weight_decay"],
                         shape_scale(rows, cols, p["scale"]))
    return new_w, new_buf, o


# ---------------------------------------------------------------------------
# Aux AdamW for the non-2-D parameters
# ---------------------------------------------------------------------------

def adamw_step(param, grad, exp_avg, exp_avg_sq, step, hp=None):
    """One AdamW step, step counted from 1.  Moments as in the blog's
    section 1; bias correction, eps and decoupled decay as in torch.optim.AdamW.
    Returns (new_param, new_exp_avg, new_exp_avg_sq)."""
    p = adamw_defaults()
    if hp:
        p.update(hp)
    g = np.asarray(grad, dtype=np.float64)
    m = p["beta1"] * np.asarray(exp_avg, np.float64) + (1.0 - p["beta1"]) * g
    v = p["beta2"] * np.asarray(exp_avg_sq, np.float64) + (1.0 - p["beta2"]) * g * g
    m_hat = m / (1.0 - p["beta1"] ** step)
    v_hat = v / (1.0 - p["beta2"] ** step)
    w = np.asarray(param, np.float64) * (1.0 - p["lr"] * p["weight_decay"])
    w = w - p["lr"] * m_hat / (np.sqrt(v_hat) + p["eps"])
    return w, m, v


# ---------------------------------------------------------------------------
# Newton-Muon
# ---------------------------------------------------------------------------

def second_moment(acts):
    """Activation second moment S = X^T X / N for X of N rows (tokens) by d
    columns ("What Is Newton-Muon?")."""
    x = np.asarray(acts, dtype=np.float64)
    return (x.T @ x) / x.shape[0]


def spd_inverse(s, damping=0.0):
    """(S + damping I)^-1 for a symmetric positive definite S."""
    s = np.asarray(s, dtype=np.float64)
    return np.linalg.inv(s + damping * np.eye(s.shape[0]))


def right_precondition(grad, s_inv_blocks):
    """G <- G S^-1, block-diagonal when several inverses are given: block b
    multiplies the gradient columns [b d, (b+1) d) ("What Is Newton-Muon?",
    four-block diagonal approximation of the MLP contraction)."""
    g = np.asarray(grad, dtype=np.float64)
    blocks = [np.asarray(s, np.float64) for s in s_inv_blocks]
    d = blocks[0].shape[0]
    if g.shape[1] != d * len(blocks):
        raise ValueError("gradient columns must equal blocks * d")
    out = np.empty_like(g)
    for k, s_inv in enumerate(blocks):
        out[:, k * d:(k + 1) * d] = g[:, k * d:(k + 1) * d] @ s_inv
    return out


def newton_muon_step(w, grad, buf, s_inv_blocks, hp=None):
    """Newton-Muon: right-precondition the raw gradient, then the standard
    Muon step ("What Is Newton-Muon?": the only algorithmic change)."""
    return muon_step(w, right_precondition(grad, s_inv_blocks), buf, hp)


# ---------------------------------------------------------------------------
# Counting (the metric's definition of NS work)
# ---------------------------------------------------------------------------

def ns_nominal_flops(rows, cols, steps=5):
    """4 m^2 n + 2 m^3 per iteration with m = min(rows, cols), n = max."""
    m, n = min(rows, cols), max(rows, cols)
    return steps * (4 * m * m * n + 2 * m ** 3)
