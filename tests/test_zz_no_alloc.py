"""muon_orthogonalize_noalloc: Newton-Schulz for callers that cannot
allocate device memory (hosts that own every device byte, allocator
callbacks, processes whose memory pool must not grow).

It is called here through the C ABI directly.  It runs the same kernels on
the same scratch layout as the context-based muon_orthogonalize, so on two
calls in a row (the second call finds the first call's leftovers in the
shared scratch array) its output must equal that entry point's bit for bit,
and lie within the Newton-Schulz tolerance of the fp64 oracle; the device's
free memory must not change.  This file is collected last so that a run
stopping at the first failure has run every other test already.
"""

import ctypes

import numpy as np
import pytest

import oracle
import workloads as wl
from helpers import ns_tol, rel_fro, to_np

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def _call(lib, hp, x, out, code):
    return lib.muon_orthogonalize_noalloc(
        ctypes.c_void_p(x.data_ptr()), code, x.shape[0], x.shape[1],
        ctypes.c_void_p(out.data_ptr()), ctypes.byref(hp),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_context_entry_point_twice():
    import matrix_aware_optimizer_step_b200 as mx
    lib = mx.load_library()
    hp = mx.default_hparams()
    cases = [((768, 3072), torch.bfloat16, mx.MUON_BF16, 1),
             ((300, 200), torch.float32, mx.MUON_F32, 2)]
    with mx.MuonContext(0) as ctx:
        refs, xs, hosts = [], [], []
        for shape, dt, _, seed in cases:
            h = wl.np_normal(shape, 1.0, seed=seed)
            if dt == torch.bfloat16:
                h = wl.bf16_round_np(h)
            hosts.append(h)
            x = torch.from_numpy(h).cuda().to(dt).contiguous()
            ref = torch.empty(shape, device="cuda")
            ctx.orthogonalize([x], [ref], hp)
            xs.append(x)
            refs.append(ref)
        outs = [torch.full(shape, float("nan"), device="cuda") for shape, _, _, _ in cases]
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        for (shape, _, code, _), x, out in zip(cases, xs, outs):
            assert _call(lib, hp, x, out, code) == 0
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        for (shape, _, _, _), out, ref, h in zip(cases, outs, refs, hosts):
            assert torch.isfinite(out).all()
            assert torch.equal(out, ref)
            assert rel_fro(to_np(out), oracle.newton_schulz(h.astype(np.float64), 5)) < ns_tol(shape)
        assert free_after == free_before


def test_noalloc_rejects_what_does_not_fit_or_is_invalid():
    import matrix_aware_optimizer_step_b200 as mx
    lib = mx.load_library()
    hp = mx.default_hparams()
    big = torch.zeros((2048, 2048), device="cuda")
    out = torch.zeros((2048, 2048), device="cuda")
    assert _call(lib, hp, big, out, mx.MUON_F32) == 3          # MUON_ERR_WORKSPACE
    assert torch.count_nonzero(out) == 0
    small = torch.ones((8, 8), device="cuda")
    o8 = torch.zeros((8, 8), device="cuda")
    bad = mx.default_hparams(ns_steps=-1)
    assert _call(lib, bad, small, o8, mx.MUON_F32) == 1        # MUON_ERR_INVALID_ARG
    assert lib.muon_orthogonalize_noalloc(None, 0, 8, 8, ctypes.c_void_p(o8.data_ptr()),
                                          ctypes.byref(hp), None) == 1
    torch.cuda.synchronize()
    assert torch.count_nonzero(o8) == 0
