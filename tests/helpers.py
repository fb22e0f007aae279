"""Shared test helpers: error measures and host<->device moves.  No method
arithmetic lives here."""

import numpy as np


def rel_fro(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


# Tolerances (relative Frobenius error per matrix):
# * bf16 Newton-Schulz output against the fp64 oracle of the same input.
NS_TOL = 2e-2
# Below 64 rows the bf16 data flow itself (operands rounded to bf16 once per
# stage, fp32 sums), emulated exactly on the CPU over 200 seeds per shape,
# exceeds 2e-2 on up to a quarter of random matrices (max 3.1e-2 at 16x16,
# 6.2e-2 at 4x4): few singular values, each perturbed by about 2^-9 per
# stage and amplified by |p'(s)| up to 1.5 per iteration.  Those shapes get
# the bound that arithmetic supports.


def ns_tol(shape):
    m = min(shape)
    if m >= 64:
        return NS_TOL
    return 4e-2 if m >= 16 else 8e-2
# * fp32 elementwise stages (momentum buffer, staged apply, AdamW).
EW_TOL = 1e-5
# * Newton-Muon stages in fp32 (S^-1, G S^-1, the preconditioned momentum)
#   against the fp64 oracle of the same inputs.
NEWTON_TOL = 1e-5
