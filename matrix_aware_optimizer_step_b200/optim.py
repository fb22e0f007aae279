"""torch.optim front end: one optimizer over Muon and aux AdamW param groups.

The interface follows the README of the Muon repository ("Muon: An
optimizer for the hidden layers of neural networks", section "Usage"): a
list of param groups, each with ``use_muon``; Muon groups take ``lr``,
``weight_decay`` (and ``momentum``, ``nesterov``, ``ns_steps``), AdamW groups
take ``lr``, ``betas``, ``eps``, ``weight_decay``.  Which parameters are
"hidden" is the caller's choice, as the README says.

This file only keeps optimizer state tensors and hands pointers to the
library: every update runs in libmuon_b200.so.
"""

from __future__ import annotations

from typing import Iterable

import torch

from .binding import MuonContext, default_adamw_hparams, default_hparams

MUON_DEFAULTS = dict(lr=0.02, weight_decay=0.01, momentum=0.95, nesterov=True, ns_steps=5,
                     scale_mode="original")
ADAMW_DEFAULTS = dict(lr=3e-4, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.01)


class MuonWithAuxAdam(torch.optim.Optimizer):
    """Muon for groups with use_muon=True (parameters of two or more
    dimensions, stepped as rows x prod(other dims) matrices), AdamW for the
    rest.  Parameters must be contiguous fp32 CUDA tensors on one device;
    gradients fp32 or bf16.

    Device-side failures (a bounded wait inside a kernel that gave up) are
    flagged on the GPU; from then on the library leaves every parameter and
    state tensor untouched until the flag is read.  step() reads it every
    `check_every` steps (0: never; each read synchronises the device) and
    raises MuonError when it is set; check() reads it on demand."""

    def __init__(self, param_groups: Iterable[dict], device: int = None, check_every: int = 100):
        groups = []
        for g in param_groups:
            g = dict(g)
            if "use_muon" not in g:
                raise ValueError("every param group needs use_muon")
            base = MUON_DEFAULTS if g["use_muon"] else ADAMW_DEFAULTS
            for k, v in base.items():
                g.setdefault(k, v)
            groups.append(g)
        super().__init__(groups, dict())
        for g in self.param_groups:
            for p in g["params"]:
                if not p.is_cuda or p.dtype != torch.float32 or not p.is_contiguous():
                    raise ValueError("parameters must be contiguous fp32 CUDA tensors")
                if g["use_muon"] and p.dim() < 2:
                    raise ValueError("Muon parameters need two or more dimensions")
        first = next(p for g in self.param_groups for p in g["params"])
        self.ctx = MuonContext(first.device.index if device is None else device)
        self.check_every = int(check_every)
        self._steps = 0

    def check(self):
        """Synchronise and raise MuonError if a device-side wait gave up since
        the last check (the library then skipped every update)."""
        self.ctx.check_device()

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for g in self.param_groups:
            params = [p for p in g["params"] if p.grad is not None]
            if not params:
                continue
            if g["use_muon"]:
                self._muon(g, params)
            else:
                self._adamw(g, params)
        self._steps += 1
        if self.check_every and self._steps % self.check_every == 0:
            self.check()
        return loss

    def _muon(self, g, params):
        hp = default_hparams(lr=g["lr"], weight_decay=g["weight_decay"], momentum=g["momentum"],
                             nesterov=g["nesterov"], ns_steps=g["ns_steps"], scale_mode=g["scale_mode"])
        by_shape = {}
        for p in params:
            st = self.state[p]
            if "momentum_buffer" not in st:
                st["momentum_buffer"] = torch.zeros_like(p)
            w = p.view(p.shape[0], -1)
            grad = p.grad.reshape(p.shape[0], -1).contiguous()
            buf = st["momentum_buffer"].view(p.shape[0], -1)
            key = (tuple(w.shape), grad.dtype)
            e = by_shape.setdefault(key, dict(weights=[], grads=[], momentum=[]))
            e["weights"].append(w)
            e["grads"].append(grad)
            e["momentum"].append(buf)
        self.ctx.step(list(by_shape.values()), hp)

    def _adamw(self, g, params):
        b1, b2 = g["betas"]
        hp = default_adamw_hparams(lr=g["lr"], beta1=b1, beta2=b2, eps=g["eps"], weight_decay=g["weight_decay"])
        by_step = {}
        for p in params:
            st = self.state[p]
            if "step" not in st:
                st["step"] = 0
                st["exp_avg"] = torch.zeros_like(p)
                st["exp_avg_sq"] = torch.zeros_like(p)
            st["step"] += 1
            by_step.setdefault(st["step"], []).append(p)
        for step, ps in by_step.items():
            self.ctx.adamw_step([p.view(-1) for p in ps], [p.grad.reshape(-1).contiguous() for p in ps],
                                [self.state[p]["exp_avg"].view(-1) for p in ps],
                                [self.state[p]["exp_avg_sq"].view(-1) for p in ps], step, hp)
