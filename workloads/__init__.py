"""Seeded synthetic workloads: shapes and random inputs, nothing else.

This module holds no arithmetic of the method.  It names the matrix shapes of
the workloads the Muon step is measured and checked on and draws their
random inputs, so that the fp64 oracle and the CUDA path are fed identical
data.  Two generators are provided:

* ``np_normal`` draws on the host with NumPy's counter-based Philox generator
  (small cases, parity tests);
* ``torch_normal`` draws directly on a device with torch's generator (the
  full-size workloads, where host generation would dominate); parity checks on
  those copy the sampled matrices back to the host.

A draw is keyed by (workload seed, step, matrix index, role), so any single
matrix can be regenerated without the others.
"""

from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import numpy as np

ROLE_GRAD = 1
ROLE_WEIGHT = 2
ROLE_MOMENTUM = 3
ROLE_ACT = 4
ROLE_AUX = 5


@dataclass(frozen=True)
class Mat:
    """One hidden 2-D weight: name, rows x cols."""
    name: str
    rows: int
    cols: int


@dataclass
class Workload:
    """A set of hidden weights plus how their inputs are drawn."""
    name: str
    mats: list
    grad_dtype: str          # "f32" or "bf16"
    grad_std: float
    weight_std: float
    steps: int
    ns_only: bool = False
    # Newton-Muon: per matrix, the list of activation blocks (index into acts)
    acts: list = field(default_factory=list)       # (name, tokens, width)
    precond: dict = field(default_factory=dict)    # mat name -> (act index, nblocks)
    refresh_every: int = 0


def gpt2_small_mats(layers=12, d=768):
    """GPT-2-small hidden set: per layer Q, K, V, O (d x d), MLP expansion
    (4d x d) and MLP contraction (d x 4d)."""
    out = []
    for l in range(layers):
        out += [Mat(f"h{l}.q", d, d), Mat(f"h{l}.k", d, d), Mat(f"h{l}.v", d, d),
                Mat(f"h{l}.o", d, d), Mat(f"h{l}.fc", 4 * d, d),
                Mat(f"h{l}.proj", d, 4 * d)]
    return out


def llama3_8b_mats(layers=32):
    """Llama-3-8B hidden set: q 4096^2, k and v 1024x4096, o 4096^2,
    gate and up 14336x4096, down 4096x14336."""
    out = []
    for l in range(layers):
        out += [Mat(f"l{l}.q", 4096, 4096), Mat(f"l{l}.k", 1024, 4096),
                Mat(f"l{l}.v", 1024, 4096), Mat(f"l{l}.o", 4096, 4096),
                Mat(f"l{l}.gate", 14336, 4096), Mat(f"l{l}.up", 14336, 4096),
                Mat(f"l{l}.down", 4096, 14336)]
    return out


def square_sweep_mats(size, count=32):
    return [Mat(f"sq{size}.{i}", size, size) for i in range(count)]


def single_256():
    """One 256x256 fp32 gradient, N(0,1); weights N(0,0.02); zero momentum;
    one step."""
    return Workload("single-256x256-f32", [Mat("w", 256, 256)], "f32", 1.0, 0.02, 1)


def gpt2_small():
    """GPT-2-small hidden set, bf16 grads N(0,1e-3), fp32 weights N(0,0.02),
    ten steps with momentum carried."""
    return Workload("gpt2-small-hidden-72", gpt2_small_mats(), "bf16", 1e-3, 0.02, 10)


def square_sweep(size):
    """32 square bf16 matrices, grads N(0,1), Newton-Schulz only."""
    return Workload(f"square-sweep-32x{size}", square_sweep_mats(size), "bf16", 1.0, 0.02,
                    1, ns_only=True)


def llama3_8b():
    """Llama-3-8B hidden set, bf16 grads N(0,1e-3), fp32 weights and momentum."""
    return Workload("llama3-8b-hidden-224", llama3_8b_mats(), "bf16", 1e-3, 0.02, 1)


def llama3_8b_layer():
    """One layer of the Llama-3-8B hidden set (7 matrices): the small case
    the profiler captures; every launch of the full step processes 32 times
    its units."""
    return Workload("llama3-8b-hidden-1-layer", llama3_8b_mats(layers=1), "bf16", 1e-3, 0.02, 1)


def newton_gpt2_small(layers=12, d=768, tokens=8192):
    """Newton-Muon on the GPT-2-small shapes: per layer the activations that
    feed QKV, O, the MLP expansion (tokens x d) and the MLP contraction
    (tokens x 4d, four d-wide blocks), N(0,1), refreshed every 10 steps."""
    w = Workload("newton-gpt2-small", gpt2_small_mats(layers, d), "bf16", 1e-3, 0.02, 10,
                 refresh_every=10)
    for l in range(layers):
        base = len(w.acts)
        w.acts += [(f"h{l}.qkv_in", tokens, d), (f"h{l}.o_in", tokens, d),
                   (f"h{l}.fc_in", tokens, d), (f"h{l}.proj_in", tokens, 4 * d)]
        for nm in ("q", "k", "v"):
            w.precond[f"h{l}.{nm}"] = (base + 0, 1)
        w.precond[f"h{l}.o"] = (base + 1, 1)
        w.precond[f"h{l}.fc"] = (base + 2, 1)
        w.precond[f"h{l}.proj"] = (base + 3, 4)
    return w


WORKLOADS = {
    "single-256": single_256,
    "gpt2-small": gpt2_small,
    "llama3-8b": llama3_8b,
    "llama3-8b-layer": llama3_8b_layer,
    "newton-gpt2-small": newton_gpt2_small,
    "sweep-1024": lambda: square_sweep(1024),
    "sweep-2048": lambda: square_sweep(2048),
    "sweep-4096": lambda: square_sweep(4096),
    "sweep-8192": lambda: square_sweep(8192),
}


# ---------------------------------------------------------------------------
# Seeded draws
# ---------------------------------------------------------------------------

def _key(seed, step, index, role):
    h = hashlib.sha256(f"{seed}/{step}/{index}/{role}".encode()).digest()
    return int.from_bytes(h[:8], "little")


def np_normal(shape, std, seed=0, step=0, index=0, role=ROLE_GRAD, dtype=np.float32):
    """N(0, std^2) draw on the host (Philox), returned as `dtype`."""
    rng = np.random.Generator(np.random.Philox(key=_key(seed, step, index, role)))
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(dtype)


def torch_normal(shape, std, seed=0, step=0, index=0, role=ROLE_GRAD, dtype=None,
                 device="cuda", out=None):
    """N(0, std^2) draw on `device` with torch's generator, cast to `dtype`
    (or written into `out`)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(_key(seed, step, index, role) & ((1 << 63) - 1))
    if out is not None:
        if out.dtype == torch.float32:
            out.normal_(0.0, std, generator=g)
        else:
            tmp = torch.empty(out.shape, dtype=torch.float32, device=out.device)
            tmp.normal_(0.0, std, generator=g)
            out.copy_(tmp)
        return out
    t = torch.empty(shape, dtype=torch.float32, device=device).normal_(0.0, std, generator=g)
    return t if dtype is None or dtype == torch.float32 else t.to(dtype)


def bf16_round_np(x):
    """Round a float32 array to the nearest bfloat16 (ties to even) and return
    it as float32: the value a bf16 gradient tensor holds.  Pure storage
    rounding, used so host-side oracles see exactly the bf16 inputs."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)
