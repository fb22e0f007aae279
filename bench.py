#!/usr/bin/env python
"""Benchmark of the Muon optimizer step on B200.

One step = one Muon step over every hidden 2-D weight of the workload (Nesterov
momentum, Frobenius normalisation, 5 quintic Newton-Schulz iterations in bf16
on tcgen05 tensor cores, shape scale, decoupled decay, update) plus the aux
AdamW step over the non-2-D parameters, all through the C ABI of
libmuon_b200.so.

Default workload: the Llama-3-8B hidden set (32 layers x q 4096x4096, k and v
1024x4096, o 4096x4096, gate and up 14336x4096, down 4096x14336 = 224
matrices, 6.98 G parameters), bf16 gradients N(0, 1e-3), fp32 weights
N(0, 0.02) and momentum carried; aux AdamW over the embedding and output
head (128256x4096 each) and the RMS-norm gains.  `--workload gpt2-small` runs
the GPT-2-small hidden set (12 layers x Q, K, V, O 768x768, MLP 3072x768 and
768x3072 = 72 matrices, 85 M parameters; bf16 gradients drawn for 10 steps and
cycled; aux AdamW over a GPT-2-small-sized set of 39.5 M parameters).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                    [--workload llama3-8b|gpt2-small|single-256|sweep-4096|...]

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank steps an
independent replica of the workload (weak scaling, no data-path collective).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

AUX_GPT2 = [("wte", 50257 * 768), ("wpe", 1024 * 768)] + \
    [(f"h{l}.{n}", 768) for l in range(12) for n in ("ln1.g", "ln1.b", "ln2.g", "ln2.b",
                                                     "attn.proj.b", "mlp.proj.b")] + \
    [(f"h{l}.attn.qkv.b", 3 * 768) for l in range(12)] + \
    [(f"h{l}.mlp.fc.b", 3072) for l in range(12)] + [("lnf.g", 768), ("lnf.b", 768)]

AUX_LLAMA = [("embed", 128256 * 4096), ("lm_head", 128256 * 4096)] + \
    [(f"l{l}.{n}", 4096) for l in range(32) for n in ("attn_norm", "mlp_norm")] + [("norm", 4096)]

GRAD_CYCLE = 10
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # CUDA-core fp32 FMA peak at max clock


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def workload_def(name):
    w = wl.WORKLOADS[name]()
    aux = {"gpt2-small": AUX_GPT2, "llama3-8b": AUX_LLAMA}.get(name, [])
    return w, aux


# ---------------------------------------------------------------------------
# algorithmic work per step
# ---------------------------------------------------------------------------

def step_work(w, aux, ns_steps=5):
    """Nominal NS FLOPs per kernel class and algorithmic HBM bytes of the
    elementwise kernels, per step (Newton-Muon: fp32 FMA FLOPs of the
    preconditioner per step and of the refresh amortised over its period)."""
    gram = poly = upd = 0
    elems = 0
    pre = 0
    pre_bytes = 0          # momentum applied in the preconditioning product's epilogue
    mom_elems = 0          # momentum in the momentum kernel
    for m in w.mats:
        fused = False
        if m.name in w.precond:
            nb = w.precond[m.name][1]
            d = m.cols // nb
            pre += 2 * m.rows * m.cols * d
            # tensor-core preconditioning (block width a multiple of 64) of a
            # matrix the small-matrix kernel does not take: bf16 G read, the
            # momentum buffer read and written, bf16 U written, in one launch
            fused = d % 64 == 0 and max(m.rows, m.cols) > SMALL_MAX
        if fused:
            pre_bytes += m.rows * m.cols * (2 + 4 + 4 + 2)
        else:
            mom_elems += m.rows * m.cols
    refresh_tc = refresh_alu = 0
    for _, tokens, width in w.acts:
        nb = 4 if width > 768 else 1
        d = width // nb
        # second moment on the tensor cores; Cholesky, L^-1 and L^-T L^-1 on
        # the fp32 ALUs, d^3/3 FLOPs each (the LAPACK counts of potrf, trtri
        # and lauum)
        refresh_tc += nb * 2 * tokens * d * d
        refresh_alu += nb * 3 * (d ** 3 // 3)
    small = 0
    fused_bytes = 0
    for m in w.mats:
        a, b = min(m.rows, m.cols), max(m.rows, m.cols)
        if b <= SMALL_MAX:
            # every iteration in one launch of the small-matrix kernel
            small += (4 * a * a * b + 2 * a ** 3) * ns_steps
        else:
            gram += 2 * a * a * b * ns_steps
            poly += 2 * a ** 3 * ns_steps
            upd += 2 * a * a * b * ns_steps
            # the last update with the weight step: bf16 B' (a x a) and X
            # (a x b) read, fp32 W read and written
            fused_bytes += 2 * a * a + 2 * a * b + 8 * a * b
        elems += m.rows * m.cols
    gbytes = 2 if w.grad_dtype == "bf16" else 4
    aux_el = sum(n for _, n in aux)
    per_iter = upd // max(1, ns_steps)
    work = {
        "gram": ("flop", gram), "poly": ("flop", poly), "update": ("flop", upd),
        "ns_small": ("flop", small),
        # the last update with the weight step fused: one iteration's FLOPs
        # and its compulsory HBM bytes (its operands B' and X read once, the
        # fp32 weights read and written once); the update class then holds
        # the other ns_steps - 1 iterations
        "update_apply": ("mixed", (per_iter, fused_bytes)),
        # momentum: read grad + buf, write buf + bf16 U
        "momentum": ("byte", mom_elems * (gbytes + 4 + 4 + 2)),
        # apply: read bf16 O + W, write W
        "apply": ("byte", elems * (2 + 4 + 4)),
        # adamw: read bf16 grad, read+write param, m, v
        "adamw": ("byte", aux_el * (2 + 3 * 8)),
        # tensor cores: G [S_hi; S_lo] executes twice the algorithmic 2 rows cols d;
        # with the momentum in its epilogue it also moves 12 B per element
        "precondition": ("mixed", (pre, pre_bytes)) if pre_bytes else ("flop", pre),
        "newton_refresh": ("seq", (refresh_tc / max(1, w.refresh_every), refresh_alu / max(1, w.refresh_every))),
    }
    if mom_elems == 0:
        # every matrix's momentum is applied by the preconditioning product;
        # what is left in the momentum class is the norm reduction
        del work["momentum"]
    return work, elems, aux_el


PAIR_TILE = 256     # output tile of the tensor-core engine (a CTA pair)
K_BLOCK = 64        # K depth of one pipeline stage
SMALL_MAX = 256     # matrices up to 256 x 256 run every iteration in one launch


def executed_flops(w, ns_steps=5):
    """Tensor-core FLOPs the engine actually issues per step, by product:
    whole 256 x 256 pair tiles over K rounded up to 64; the symmetric Gram
    and polynomial products issue only the tiles on or above the diagonal
    (T (T + 1) / 2 of T^2), the update every tile.  This is the work the
    tensor pipe does, as opposed to the metric's nominal 4 m^2 n + 2 m^3."""
    def rup(x, q):
        return -(-x // q) * q
    out = {"gram": 0, "poly": 0, "update": 0, "ns_small": 0}
    for m in w.mats:
        a, b = min(m.rows, m.cols), max(m.rows, m.cols)
        if b <= SMALL_MAX:
            # one 256 x 256 pair tile per product, K rounded up to 64
            tile = 2 * PAIR_TILE * PAIR_TILE
            out["ns_small"] += tile * (rup(b, K_BLOCK) + 2 * rup(a, K_BLOCK)) * ns_steps
            continue
        t = -(-a // PAIR_TILE)
        tri = t * (t + 1) // 2
        tile = 2 * PAIR_TILE * PAIR_TILE
        out["gram"] += tri * tile * rup(b, K_BLOCK) * ns_steps
        out["poly"] += tri * tile * rup(a, K_BLOCK) * ns_steps
        out["update"] += t * (-(-b // PAIR_TILE)) * tile * rup(a, K_BLOCK) * ns_steps
    return out


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
            time.sleep(1.0)
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def mark(self, which):
        if which == 0:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [ln for t, ln in self.lines if self.t0 - 0.15 <= t <= self.t1 + 0.15]
        if not rows:
            rows = [ln for _, ln in self.lines[-3:]]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 10:
                continue
            try:
                sm.append(float(f[2]))
                mx.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        return os.cpu_count()


def shape_classes(w):
    """Distinct wide shapes (m, n) of the workload in first-seen order, each
    with the first matrix of that shape and the matrix count.  The oracle
    orthogonalises a tall matrix through its transpose, so a shape and its
    transpose cost the same and share a class."""
    cls = {}
    for m in w.mats:
        key = (min(m.rows, m.cols), max(m.rows, m.cols))
        if key not in cls:
            cls[key] = [m, 0]
        cls[key][1] += 1
    return [(k, v[0], v[1]) for k, v in cls.items()]


def time_oracle_matrix(m, rng):
    """Seconds of one oracle Muon step on a fresh rows x cols matrix."""
    import numpy as np
    import oracle
    W = rng.standard_normal((m.rows, m.cols)) * 0.02
    G = rng.standard_normal((m.rows, m.cols)) * 1e-3
    B = np.zeros((m.rows, m.cols))
    t0 = time.perf_counter()
    oracle.muon_step(W, G, B)
    return time.perf_counter() - t0


def time_oracle_adamw(n, rng):
    import numpy as np
    import oracle
    p, g = rng.standard_normal(n), rng.standard_normal(n) * 1e-2
    t0 = time.perf_counter()
    oracle.adamw_step(p, g, np.zeros(n), np.zeros(n), 1)
    return time.perf_counter() - t0


def cpu_baseline(w, aux):
    """The fp64 oracle as it stands, on a bounded sample of the workload:
    one matrix of each distinct wide shape (Muon step), extrapolated to the
    full step by the shape counts, plus AdamW on 1/len(mats) of the aux
    elements, extrapolated by len(mats)."""
    import numpy as np
    rng = np.random.default_rng(0)
    t_step, t_sample, parts = 0.0, 0.0, []
    for (a, b), m, count in shape_classes(w):
        t = time_oracle_matrix(m, rng)
        t_sample += t
        t_step += count * t
        parts.append(f"{m.rows}x{m.cols} x{count}")
    aux_el = sum(n for _, n in aux)
    if aux_el:
        n = max(1, aux_el // len(w.mats))
        t = time_oracle_adamw(n, rng)
        t_sample += t
        t_step += t * aux_el / n
    return {"value": 1.0 / t_step, "unit": "Muon step/s", "cores": blas_threads(), "kind": "oracle",
            "extrapolated": len(w.mats) > len(parts) or bool(aux_el),
            "sample": "fp64 NumPy oracle: one Muon step per distinct wide shape (" + ", ".join(parts) +
                      ") scaled by the shape counts" +
                      (f", plus AdamW on {max(1, aux_el // len(w.mats))} of the {aux_el} aux elements scaled "
                       "to all of them" if aux_el else "") + "; extrapolated to one full step",
            "sample_seconds": round(t_sample, 3)}


# Oracle samples of the reference arm: shapes whose one-matrix Newton-Schulz
# costs at most this many nominal FLOPs (at least the cheapest shape), so a
# --steps K --warmup W run on the host stays within minutes.
REF_SAMPLE_MAX_FLOPS = 5e11


def run_reference(args, w, aux):
    """The oracle as it stands, timed on the host.  Each step is one oracle
    Muon step on one hidden matrix, cycling through the workload's distinct
    wide shapes that are cheap enough to sample, plus AdamW on
    1/len(mats) of the aux elements.  The full-step time is extrapolated:
    a sampled shape counts its mean sample time once per matrix of that
    shape; an unsampled (larger) shape counts its nominal Newton-Schulz
    FLOPs at the sampled shapes' fp64 FLOP rate; AdamW counts len(mats)
    samples."""
    import numpy as np
    import oracle
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    rng = np.random.default_rng(0)
    classes = shape_classes(w)
    cost = {k: oracle.ns_nominal_flops(m.rows, m.cols, 5) for k, m, _ in classes}
    cheapest = min(cost.values())
    sampled = [(k, m, c) for k, m, c in classes if cost[k] <= max(REF_SAMPLE_MAX_FLOPS, cheapest)]
    aux_el = sum(n for _, n in aux)
    share = max(1, aux_el // len(w.mats)) if aux_el else 0
    times = {k: [] for k, _, _ in sampled}
    t_adam = []
    for step in range(args.warmup + args.steps):
        k, m, _ = sampled[step % len(sampled)]
        t = time_oracle_matrix(m, rng)
        ta = time_oracle_adamw(share, rng) if share else 0.0
        if step >= args.warmup:
            times[k].append(t)
            t_adam.append(ta)
    mean = {k: statistics.mean(v) for k, v in times.items() if v}
    rate = sum(cost[k] for k in mean) / sum(mean.values())      # fp64 FLOP/s of the samples
    step_s = 0.0
    for k, m, count in classes:
        step_s += count * (mean[k] if k in mean else cost[k] / rate)
    if share:
        step_s += len(w.mats) * statistics.mean(t_adam)
    v = 1.0 / step_s
    names = ", ".join(f"{m.rows}x{m.cols}" for _, m, _ in sampled)
    sample = (f"each step: one oracle Muon step on one matrix, cycling through the shapes {names}"
              + (f", plus AdamW on {share} aux elements" if share else "")
              + f"; full step = sampled shapes' mean times x their counts"
              + (", larger shapes by nominal NS FLOPs at the sampled fp64 rate" if len(sampled) < len(classes) else "")
              + (f", AdamW x {len(w.mats)}" if share else "") + " (extrapolated)")
    out = {"impl": "reference", "metric": "Muon step/s", "value": v, "unit": "Muon step/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "matrices": len(w.mats)},
           "cpu_baseline": {"value": v, "unit": "Muon step/s", "cores": blas_threads(), "kind": "oracle",
                            "extrapolated": True, "sample": sample},
           "e2e": {"value": v, "unit": "Muon step/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

SOURCE_GROUPS = {"gram": "ns_gemm", "poly": "ns_gemm", "update": "ns_gemm", "update_apply": "ns_gemm",
                 "ns_small": "small_ns",
                 "momentum": "elementwise", "apply": "elementwise", "adamw": "elementwise"}


def kernel_source_hash(group):
    files = {"ns_gemm": ("ns_gemm.cuh", "sm100_ptx.cuh"),
             "small_ns": ("small_ns.cuh", "sm100_ptx.cuh"),
             "elementwise": ("elementwise.cuh", "sm100_ptx.cuh")}[group]
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "matrix_aware_optimizer_step_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def read_traffic(kind, workload):
    """DRAM bytes per step of kernel class `kind` from the committed ncu
    summary profiles/dram_traffic_<workload>.txt, if there is one taken on
    the current source of that kernel (else None).  A summary captured on a
    smaller case of the same kernels gives `scale.<kind>`: the factor from
    the captured units to one step of the workload."""
    p = os.path.join(ROOT, "profiles", f"dram_traffic_{workload}.txt")
    if not os.path.exists(p) or kind not in SOURCE_GROUPS:
        return None
    vals, src, scale = {}, {}, {}
    for ln in open(p):
        ln = ln.strip()
        if ln.startswith("kernel_source_sha256_16."):
            k, v = ln.split()
            src[k.split(".", 1)[1]] = v
        elif ln.startswith("dram_bytes_per_step."):
            k, v = ln.split()
            vals[k.split(".", 1)[1]] = float(v)
        elif ln.startswith("scale."):
            k, v = ln.split()
            scale[k.split(".", 1)[1]] = float(v)
    group = SOURCE_GROUPS[kind]
    if src.get(group) != kernel_source_hash(group) or kind not in vals:
        return None
    return vals[kind] * scale.get(kind, 1.0)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="muon", choices=["muon", "reference"])
    ap.add_argument("--workload", default="llama3-8b", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sharded", action="store_true",
                    help="owner-computes sharding (strong scaling): every rank holds the whole model, steps "
                         "only the matrices muon_partition gives it, and the updated weights are broadcast "
                         "from their owners, stage by stage, overlapping the next stage's step")
    ap.add_argument("--stages", type=int, default=2, help="slices per owner in --sharded mode")
    ap.add_argument("--serial-adamw", action="store_true",
                    help="run the aux AdamW on the Muon stream ahead of the Muon step; by default it runs "
                         "on a second, lowest-priority stream, forked from and joined into the "
                         "(highest-priority) Muon stream every step")
    args = ap.parse_args()
    w, aux = workload_def(args.workload)
    if args.impl == "reference":
        run_reference(args, w, aux)
        return

    import torch
    import matrix_aware_optimizer_step_b200 as mx

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1 or args.sharded:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29533")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), rank=rank, world_size=world,
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    # replicas step independent copies; sharded ranks hold one model
    seed = 1000 if args.sharded else 1000 + rank

    # ---- resident inputs ----
    tdt = torch.bfloat16 if w.grad_dtype == "bf16" else torch.float32
    Ws = [wl.torch_normal((m.rows, m.cols), w.weight_std, seed, 0, i, wl.ROLE_WEIGHT, device=dev)
          for i, m in enumerate(w.mats)]
    if args.sharded:
        from matrix_aware_optimizer_step_b200.binding import partition
        own = partition([(m.rows, m.cols) for m in w.mats], world)
        Bs = [torch.zeros((m.rows, m.cols), device=dev) if own[i] == rank else None for i, m in enumerate(w.mats)]
    else:
        Bs = [torch.zeros((m.rows, m.cols), device=dev) for m in w.mats]
    n_cycle = min(GRAD_CYCLE, max(1, w.steps)) if args.workload != "llama3-8b" else 1
    def flat_set(shapes, dtype):
        # one contiguous buffer per set (every tensor starts on a 16-byte
        # boundary), so a set moves between host and device in one copy
        sizes = [math.prod(sh) for sh in shapes]
        pads = [(n + 7) // 8 * 8 for n in sizes]
        flat = torch.empty(sum(pads), dtype=dtype, device=dev)
        views, off = [], 0
        for sh, n, pn in zip(shapes, sizes, pads):
            views.append(flat[off:off + n].view(sh))
            off += pn
        return flat, views

    G_flat, Gs = [], []
    for s in range(n_cycle):
        f, vs = flat_set([(m.rows, m.cols) for m in w.mats], tdt)
        for i, (m, v) in enumerate(zip(w.mats, vs)):
            wl.torch_normal((m.rows, m.cols), w.grad_std, seed, s, i, wl.ROLE_GRAD, out=v)
        G_flat.append(f)
        Gs.append(vs)
    Ps = [wl.torch_normal((n,), 0.02, seed, 0, 10000 + i, wl.ROLE_WEIGHT, device=dev) for i, (_, n) in enumerate(aux)]
    Ms = [torch.zeros(n, device=dev) for _, n in aux]
    Vs = [torch.zeros(n, device=dev) for _, n in aux]
    AG_flat, AGs = [], []
    for s in range(n_cycle):
        f, vs = flat_set([(n,) for _, n in aux], torch.bfloat16)
        for i, ((_, n), v) in enumerate(zip(aux, vs)):
            wl.torch_normal((n,), 1e-3, seed, s, 10000 + i, wl.ROLE_AUX, out=v)
        AG_flat.append(f)
        AGs.append(vs)

    by_shape = {}
    for i, m in enumerate(w.mats):
        by_shape.setdefault((m.rows, m.cols), []).append(i)

    # Newton-Muon: activations per layer input, one S^-1 buffer per input
    newton = bool(w.acts)
    Acts, Sinv, Split, nblk = [], [], [], []
    if newton:
        for a, (_, tokens, width) in enumerate(w.acts):
            nb = 4 if width > 768 else 1
            d = width // nb
            Acts.append(wl.torch_normal((tokens, width), 1.0, seed, 0, 20000 + a, wl.ROLE_ACT,
                                        dtype=torch.bfloat16, device=dev))
            Sinv.append(torch.empty((nb, d, d), device=dev))
            # the refresh also writes S^-1's bf16 hi/lo split, which the steps
            # until the next refresh use as it is
            Split.append(torch.empty((nb, 2 * d, d), dtype=torch.bfloat16, device=dev))
            nblk.append(nb)

    def groups_for(s):
        gs = []
        for ix in by_shape.values():
            g = dict(weights=[Ws[i] for i in ix], grads=[Gs[s][i] for i in ix],
                     momentum=[Bs[i] for i in ix])
            if newton:
                g["precond"] = [Sinv[w.precond[w.mats[i].name][0]] for i in ix]
                g["precond_split"] = [Split[w.precond[w.mats[i].name][0]] for i in ix]
                g["precond_blocks"] = w.precond[w.mats[ix[0]].name][1]
            gs.append(g)
        return gs

    ctx = mx.MuonContext(local)
    hp = mx.default_hparams()
    ahp = mx.default_adamw_hparams()
    # The aux AdamW touches none of the Muon tensors, so it runs through a
    # second context on a second stream of the lowest priority, forked from
    # and joined back into the Muon stream (highest priority) every step: its
    # blocks are scheduled only where the Muon kernels leave room (registers
    # and HBM bandwidth beside the persistent Newton-Schulz CTAs).  The
    # per-kernel pass below runs it on the Muon stream instead, so each
    # kernel's time is taken without contention.  --serial-adamw runs it on the
    # Muon stream, ahead of the Muon step, throughout.
    serial = args.serial_adamw or not aux
    if serial:
        stream = torch.cuda.current_stream()
        aux_stream = stream
    else:
        torch.cuda.synchronize(dev)
        stream = torch.cuda.Stream(device=dev, priority=-100)
        aux_stream = torch.cuda.Stream(device=dev, priority=0)
        # every other torch operation (the end-to-end staging copies) then
        # runs in order with the Muon step
        torch.cuda.set_stream(stream)
    fork_ev = [torch.cuda.Event() for _ in range(2)]
    join_ev = [torch.cuda.Event() for _ in range(2)]
    ctx_aux = ctx if serial else mx.MuonContext(local)
    pre_groups = [groups_for(s) for s in range(n_cycle)] if not args.sharded else None
    sm = None
    if args.sharded:
        from matrix_aware_optimizer_step_b200.sharded import ShardedMuon
        if newton:
            raise SystemExit("--sharded runs plain Muon workloads")
        sm = ShardedMuon(Ws, ctx=ctx, hp=hp, stages=args.stages)
    adam_step = [0]
    on_side = [not serial]          # AdamW on the side stream (False: on the Muon stream)

    def one_step(k):
        if aux:
            side = on_side[0]
            if side:
                fork_ev[k & 1].record(stream)
                aux_stream.wait_event(fork_ev[k & 1])
            adam_step[0] += 1
            ctx_aux.adamw_step(Ps, AGs[k % n_cycle], Ms, Vs, adam_step[0], ahp, aux_stream if side else stream)
            if side:
                join_ev[k & 1].record(aux_stream)
        if newton and k % w.refresh_every == 0:
            ctx.newton_refresh(Acts, Sinv, nblk, 0.0, stream, splits=Split)
        if sm is not None:
            sm.step(Gs[k % n_cycle], Bs, stream)
        else:
            ctx.step(pre_groups[k % n_cycle], hp, stream)
        if aux and side:
            stream.wait_event(join_ev[k & 1])

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        if dist is None:
            return x
        t = torch.tensor([x], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def timed(k_steps, body, finish=None):
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for k in range(k_steps):
            body(k)
        if finish is not None:
            finish()          # join side streams into `stream` before the end event
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1))

    for k in range(args.warmup):
        one_step(k)
    torch.cuda.synchronize()
    ctx.check_device()

    # ---- headline: device-resident inputs ----
    clocks = ClockSampler(local)
    clocks.start()
    l0 = ctx.launch_count + (ctx_aux.launch_count if ctx_aux is not ctx else 0)
    clocks.mark(0)
    ms = timed(args.steps, lambda k: one_step(args.warmup + k))
    clocks.mark(1)
    launches = ctx.launch_count + (ctx_aux.launch_count if ctx_aux is not ctx else 0) - l0
    clk = clocks.stop()
    ctx.check_device()
    ms_per_step = ms / args.steps
    # replicas: every rank completes a step; sharded: all ranks together complete one
    units = 1 if args.sharded else world
    value = units * 1e3 / ms_per_step

    # ---- per-kernel device times (events on the launching stream) ----
    ctx.profile(True)
    if ctx_aux is not ctx:
        ctx_aux.profile(True)
    on_side[0] = False
    timed(args.steps, lambda k: one_step(args.warmup + args.steps + k))
    on_side[0] = not serial
    kt = ctx.profile_read()
    ctx.profile(False)
    if ctx_aux is not ctx:
        ka = ctx_aux.profile_read()
        ctx_aux.profile(False)
        for kind, (t_ms, nl) in ka.items():
            if nl:
                kt[kind] = (kt[kind][0] + t_ms, kt[kind][1] + nl)
    work, elems, aux_el = step_work(w, aux, hp.ns_steps)
    exe = executed_flops(w, hp.ns_steps)
    fused = kt.get("update_apply", (0, 0))[1] > 0
    if fused:
        work["update"] = ("flop", work["update"][1] - work["update_apply"][1][0])
        exe_last = exe["update"] // max(1, hp.ns_steps)
        exe["update"] -= exe_last
        exe["update_apply"] = exe_last
    pk = peaks()
    # A kernel timed inside a seconds-long loop runs at the power-capped
    # clock: its denominator is the sustained bf16 figure; a short burst
    # takes the burst figure.
    long_run = ms >= 1000.0
    bf16_peak = pk["bf16_sus"] if long_run else pk["bf16"]
    bf16_src = (pk["source"] + (" sustained bf16 (seconds-long cuBLAS loop under the power cap)" if long_run
                                else " burst bf16 (torch.matmul 8192^3)"))
    kernels = {}
    for kind, (t_ms, nl) in kt.items():
        if nl == 0 or kind not in work:
            continue
        unit, per_step = work[kind]
        tot = per_step * args.steps
        if unit == "flop":
            ach = tot / (t_ms * 1e-3) / 1e12
            kernels[kind] = {"ms_per_step": t_ms / args.steps, "launches": nl, "achieved": ach,
                             "unit": "TFLOP/s", "frac": ach / bf16_peak}
        elif unit == "fflop":
            # fp32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz
            ach = tot / (t_ms * 1e-3) / 1e12
            kernels[kind] = {"ms_per_step": t_ms / args.steps, "launches": nl, "achieved": ach,
                             "unit": "TFLOP/s", "bound": "alu", "frac": ach / FP32_PEAK_TFLOPS}
        elif unit == "seq":
            # tensor-core FLOPs then fp32 ALU FLOPs in separate launches: the
            # roofline time is the sum of the two lower bounds
            tc, alu = per_step[0] * args.steps, per_step[1] * args.steps
            t_s = t_ms * 1e-3
            bound_s = tc / (bf16_peak * 1e12) + alu / (FP32_PEAK_TFLOPS * 1e12)
            kernels[kind] = {"ms_per_step": t_ms / args.steps, "launches": nl,
                             "achieved": (tc + alu) / t_s / 1e12, "unit": "TFLOP/s",
                             "frac": bound_s / t_s, "bound": "tensor+alu"}
        elif unit == "mixed":
            # tensor-core FLOPs and HBM bytes in one launch: the roofline time
            # is the larger of the two lower bounds
            fl, by = per_step[0] * args.steps, per_step[1] * args.steps
            t_s = t_ms * 1e-3
            bound_s = max(fl / (bf16_peak * 1e12), by / (pk["hbm"] * 1e9))
            kernels[kind] = {"ms_per_step": t_ms / args.steps, "launches": nl,
                             "achieved": fl / t_s / 1e12, "unit": "TFLOP/s",
                             "achieved_gbs": by / t_s / 1e9, "frac": bound_s / t_s,
                             "bound": "hbm" if by / (pk["hbm"] * 1e9) > fl / (bf16_peak * 1e12) else "tensor"}
        else:
            ach = tot / (t_ms * 1e-3) / 1e9
            kernels[kind] = {"ms_per_step": t_ms / args.steps, "launches": nl, "achieved": ach,
                             "unit": "GB/s", "frac": ach / pk["hbm"]}
        if kind in exe:
            # what the tensor pipe actually ran (whole pair tiles; upper
            # triangle only for the symmetric products)
            ex = exe[kind] * args.steps / (t_ms * 1e-3) / 1e12
            kernels[kind]["executed_tflops"] = ex
            kernels[kind]["executed_frac"] = ex / bf16_peak
    tot_ms = sum(v["ms_per_step"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = v["ms_per_step"] / tot_ms if tot_ms else 0.0
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    d = kernels[dom]
    traffic = read_traffic(dom, args.workload)
    bound = d.get("bound", "tensor" if d["unit"] == "TFLOP/s" else "hbm")
    peak = {"alu": FP32_PEAK_TFLOPS, "hbm": pk["hbm"]}.get(bound, bf16_peak)
    roofline = {"bound": bound, "kernel": dom,
                "achieved": d["achieved"], "peak": peak,
                "unit": d["unit"], "frac": d["frac"],
                "traffic": (traffic / d["launches"] * args.steps) if traffic is not None else None,
                "peak_source": {"hbm": pk["source"] + " HBM copy",
                                "alu": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz",
                                "tensor+alu": bf16_src + " for the tensor-core part, derived fp32 "
                                              "peak for the ALU part; frac = summed lower bounds / time"
                                }.get(bound, bf16_src)}
    if "executed_frac" in d:
        roofline["executed_frac"] = d["executed_frac"]
    ns_kinds = ("gram", "poly", "update", "update_apply", "ns_small")
    ns_flops = work["gram"][1] + work["poly"][1] + work["update"][1] + work["ns_small"][1] + \
        (work["update_apply"][1][0] if "update_apply" in kernels else 0)
    ns_exec = sum(exe.get(k, 0) for k in ns_kinds if k in kernels)
    ns_ms = sum(kernels.get(k, {"ms_per_step": 0})["ms_per_step"] for k in ns_kinds)
    ew_kinds = [k for k in ("momentum", "apply", "adamw") if k in kernels]
    ew_bytes = sum(work[k][1] for k in ew_kinds)
    ew_ms = sum(kernels[k]["ms_per_step"] for k in ew_kinds)

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        hG = [G_flat[s].cpu().pin_memory() for s in range(n_cycle)]
        hAG = [AG_flat[s].cpu().pin_memory() for s in range(n_cycle)] if aux else [None] * n_cycle
        dev_w = Ws + Ps
        w_elems = sum(t.numel() for t in dev_w)
        h_w = torch.empty(w_elems, dtype=torch.float32, pin_memory=True)   # every weight, concatenated
        h2d = G_flat[0].numel() * G_flat[0].element_size() + (AG_flat[0].numel() * 2 if aux else 0)
        d2h = w_elems * 4
        k_e2e = max(3, min(args.steps, 50))
        # Pipelined like a training loop that streams gradients in and weights
        # out: step k's gradients arrive on a copy-in stream (into the device
        # set the step reads; the set is reused every n_cycle steps), the
        # updated weights are copied on the device into a staging buffer and
        # leave for the host on a copy-out stream, so PCIe in both directions
        # overlaps the next step's kernels.  Two staging buffers when device
        # memory holds them, one otherwise (the next step's staging copy then
        # waits for the previous copy-out); with no room for one, the weights
        # leave directly and the next step waits for them before it starts.
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        torch.cuda.synchronize(dev)
        free_b, _ = torch.cuda.mem_get_info(dev)
        margin = 4 << 30
        n_stage = 2 if 2 * w_elems * 4 + margin <= free_b else (1 if w_elems * 4 + margin <= free_b else 0)
        staging = n_stage > 0
        stage = [torch.empty(w_elems, dtype=torch.float32, device=dev) for _ in range(n_stage)]
        h_views, off = [], 0
        for t in dev_w:
            h_views.append(h_w[off:off + t.numel()].view(t.shape))
            off += t.numel()
        in_done = [torch.cuda.Event() for _ in range(n_cycle)]
        used = [torch.cuda.Event() for _ in range(n_cycle)]
        n_out = max(1, n_stage)
        staged = [torch.cuda.Event() for _ in range(n_out)]
        out_done = [torch.cuda.Event() for _ in range(n_out)]

        def e2e_step(k):
            s, b = k % n_cycle, k % n_out
            with torch.cuda.stream(s_in):
                if k >= n_cycle:
                    s_in.wait_event(used[s])          # the step that last read this set is done
                G_flat[s].copy_(hG[s], non_blocking=True)
                if aux:
                    AG_flat[s].copy_(hAG[s], non_blocking=True)
                in_done[s].record(s_in)
            stream.wait_event(in_done[s])
            if not staging and k >= 1:
                stream.wait_event(out_done[0])        # the previous weights have left before they change
            one_step(k)
            used[s].record(stream)
            if staging:
                if k >= n_out:
                    stream.wait_event(out_done[b])    # staging buffer b (n_out steps ago) has left
                torch.cat([t.view(-1) for t in dev_w], out=stage[b])   # one device kernel
            staged[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(staged[b])
                if staging:
                    h_w.copy_(stage[b], non_blocking=True)
                else:
                    for dst, src in zip(h_views, dev_w):
                        dst.copy_(src, non_blocking=True)
                out_done[b].record(s_out)

        def e2e_finish():
            stream.wait_event(out_done[(k_e2e - 1) % n_out])

        ms_e2e = timed(k_e2e, e2e_step, e2e_finish)
        # the host holds the last step's weights (compared tensor by tensor:
        # no second device copy of the whole set)
        if not all(torch.equal(hv, t.cpu()) for hv, t in zip(h_views, dev_w)):
            raise RuntimeError("e2e: host weights differ from the device weights")
        del stage
        torch.cuda.empty_cache()
        e2e = {"value": units * 1e3 * k_e2e / ms_e2e, "unit": "Muon step/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "staging_buffers": n_stage,
               "note": ("every step: gradients host->device (copy-in stream), updated fp32 weights "
                        + ("device->device->host (copy-out stream), overlapped with the next step's kernels"
                           if staging else "device->host (copy-out stream); the next step starts after it"))}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, aux)

    out = {
        "metric": "Muon step/s", "value": value, "unit": "Muon step/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong" if args.sharded else "weak", "vs_baseline": None,
        "dtype": "bf16",
        "elementwise_dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "matrices": len(w.mats), "hidden_params": elems,
                   "aux_params": aux_el, "grad_dtype": w.grad_dtype, "ns_steps": hp.ns_steps,
                   "grad_sets_cycled": n_cycle, "l2": "inputs larger than L2 (no flush)",
                   "aux_adamw": ("same stream" if serial else
                                 "second stream of the lowest priority, joined every step"),
                   "kernels_pass": "aux AdamW on the Muon stream (per-kernel times without contention)",
                   "parallelism": (f"owner-computes x{world}, {args.stages} exchange stages" if args.sharded
                                   else f"replicas x{world}" if world > 1 else "single")},
        "ns_tflops": ns_flops / (ns_ms * 1e-3) / 1e12 if ns_ms else None,
        "ns_tflops_of_step": ns_flops / (ms_per_step * 1e-3) / 1e12,
        "ns_frac_bf16_peak": (ns_flops / (ns_ms * 1e-3) / 1e12) / bf16_peak if ns_ms else None,
        "ns_executed_tflops": ns_exec / (ns_ms * 1e-3) / 1e12 if ns_ms else None,
        "ns_executed_frac": (ns_exec / (ns_ms * 1e-3) / 1e12) / bf16_peak if ns_ms else None,
        "bf16_peak_tflops": bf16_peak, "bf16_peak_source": bf16_src,
        "elementwise_gbs": ew_bytes / (ew_ms * 1e-3) / 1e9 if ew_ms else None,
        "elementwise_frac_hbm": (ew_bytes / (ew_ms * 1e-3) / 1e9) / pk["hbm"] if ew_ms else None,
        "roofline": roofline, "kernels": kernels, "gpu_launches": launches,
        "launches_per_step": launches / args.steps,
        "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
    }
    if ctx_aux is not ctx:
        ctx_aux.close()
    ctx.close()
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
