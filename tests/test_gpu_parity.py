"""CUDA path against the fp64 oracle, through the C ABI, on seeded inputs.

Bars: bf16 Newton-Schulz output within 2e-2 relative Frobenius error per
matrix; fp32 momentum buffer, staged apply (the oracle's apply fed the GPU's
own orthogonalised update) and AdamW within 1e-5.
"""

import numpy as np
import pytest

import oracle
import workloads as wl
from helpers import EW_TOL, NEWTON_TOL, NS_TOL, ns_tol, rel_fro, to_np

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    import matrix_aware_optimizer_step_b200 as m
    return m


@pytest.fixture(scope="module")
def ctx(mx):
    c = mx.MuonContext(0)
    yield c
    c.close()


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(dtype).contiguous()


NS_SHAPES = [(256, 256), (5, 3), (3, 5), (1, 1), (1, 7), (127, 129), (129, 127), (300, 200),
             (200, 300), (768, 768), (768, 3072), (3072, 768), (1024, 1024), (640, 2000),
             (136, 1000), (520, 520)]


@pytest.mark.parametrize("shape", NS_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_orthogonalize_vs_oracle(ctx, shape, dtype):
    x = wl.np_normal(shape, 1.0, seed=7, index=shape[0] * 10007 + shape[1])
    if dtype == "bf16":
        x = wl.bf16_round_np(x)
    xt = dev(x, torch.bfloat16 if dtype == "bf16" else torch.float32)
    out = torch.empty(shape, dtype=torch.float32, device="cuda")
    ctx.orthogonalize([xt], [out])
    torch.cuda.synchronize()
    ctx.check_device()
    want = oracle.newton_schulz(x.astype(np.float64), 5)
    err = rel_fro(to_np(out), want)
    assert err < ns_tol(shape), f"{shape} {dtype}: {err}"


@pytest.mark.parametrize("case", [((3072, 768), "f32"), ((3072, 768), "bf16"), ((1000, 336), "f32"),
                                  ((520, 264), "bf16"), ((264, 520), "f32")],
                         ids=lambda c: f"{c[0][0]}x{c[0][1]}-{c[1]}")
def test_orthogonalize_zero_steps_exact_layout(ctx, mx, case):
    """With no iteration the output is U / (||U||_F + eps) where U is stored
    in bf16 in the wide layout and read back.  Element for element it is the
    bf16-rounded input times one scale, so a misplaced element of the layout
    write (transposing for the tall shapes, whole and ragged tiles) fails
    here even where the Newton-Schulz tolerance could absorb it."""
    shape, dt = case
    x = wl.np_normal(shape, 1.0, seed=10, index=shape[0]).astype(np.float32)
    if dt == "bf16":
        x = wl.bf16_round_np(x)
    out = torch.empty(shape, dtype=torch.float32, device="cuda")
    ctx.orthogonalize([dev(x, torch.bfloat16 if dt == "bf16" else torch.float32)], [out],
                      mx.default_hparams(ns_steps=0))
    torch.cuda.synchronize()
    ctx.check_device()
    want = wl.bf16_round_np(x).astype(np.float64) / (np.linalg.norm(x.astype(np.float64)) + oracle.NS_EPS)
    got = to_np(out)
    assert np.max(np.abs(got - want)) <= 1e-5 * np.max(np.abs(want)), shape


def test_step_tall_f32_gradients(ctx, mx):
    """fp32 gradients on tall matrices past the single-launch size (whole
    and ragged 64 x 64 tiles), two steps, with and without Nesterov."""
    shapes = [(1000, 336), (3072, 768), (520, 264)]
    _step_case(ctx, mx, shapes, 2, "f32")
    _step_case(ctx, mx, shapes, 2, "f32", hp_over=dict(nesterov=0), seed=1)


def test_orthogonalize_batched_groups(ctx):
    """Many matrices of mixed shapes in one call: every one matches."""
    shapes = [(384, 384)] * 5 + [(384, 1536)] * 3 + [(1536, 384)] * 3 + [(64, 64)] * 7
    xs, outs = [], []
    for i, s in enumerate(shapes):
        x = wl.np_normal(s, 1e-3, seed=8, index=i)
        xs.append(x)
    xt = [dev(x) for x in xs]
    outs = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    ctx.orthogonalize(xt, outs)
    torch.cuda.synchronize()
    for x, o in zip(xs, outs):
        assert rel_fro(to_np(o), oracle.newton_schulz(x, 5)) < ns_tol(x.shape)


@pytest.mark.parametrize("steps", [0, 1, 2, 3, 7])
def test_orthogonalize_ns_steps(ctx, mx, steps):
    x = wl.np_normal((200, 456), 1.0, seed=9)
    out = torch.empty((200, 456), dtype=torch.float32, device="cuda")
    ctx.orthogonalize([dev(x)], [out], mx.default_hparams(ns_steps=steps))
    torch.cuda.synchronize()
    assert rel_fro(to_np(out), oracle.newton_schulz(x, steps)) < NS_TOL


@pytest.mark.parametrize("coeffs", [(1.5, -0.5, 0.0), (2.0, -1.5, 0.5)], ids=["cubic_c0", "quintic_alt"])
def test_orthogonalize_custom_coefficients(ctx, mx, coeffs):
    """Other coefficient sets through the ABI, including c = 0 (the cubic
    iteration), against the oracle with the same coefficients."""
    a, b, c = coeffs
    hp = mx.default_hparams(ns_a=a, ns_b=b, ns_c=c, ns_steps=8)
    x = wl.np_normal((256, 384), 1.0, seed=31)
    out = torch.empty((256, 384), device="cuda")
    ctx.orthogonalize([dev(x, torch.bfloat16)], [out], hp)
    torch.cuda.synchronize()
    want = oracle.newton_schulz(wl.bf16_round_np(x), 8, a=a, b=b, c=c)
    assert rel_fro(to_np(out), want) < NS_TOL


def test_small_matrix_step_is_one_launch(ctx, mx):
    """A 256 x 256 step is ONE launch: the kernel forms the momentum and the
    Frobenius norm, runs all five iterations and applies the weight step
    from the fp32 accumulator; momentum within 1e-5 and the applied update
    within the Newton-Schulz tolerance of the oracle."""
    shape = (256, 256)
    g = wl.np_normal(shape, 1.0, seed=40, index=0)
    w0 = wl.np_normal(shape, 0.02, seed=40, index=0, role=wl.ROLE_WEIGHT)
    w, b = dev(w0), torch.zeros(shape, device="cuda")
    n0 = ctx.launch_count
    ctx.step([dict(weights=[w], grads=[dev(g)], momentum=[b])])
    torch.cuda.synchronize()
    ctx.check_device()
    assert ctx.launch_count - n0 == 1
    w1, b1, o1 = oracle.muon_step(w0, g, np.zeros(shape))
    assert rel_fro(to_np(b), b1) < EW_TOL
    upd = (w0.astype(np.float64) * (1 - 0.02 * 0.01) - to_np(w)) / 0.02
    assert rel_fro(upd, o1) < NS_TOL


@pytest.mark.parametrize("case", [((256, 256), "f32", 2), ((250, 17), "bf16", 3), ((17, 250), "f32", 2),
                                  ((1, 1), "f32", 2), ((129, 127), "bf16", 2)],
                         ids=lambda c: f"{c[0][0]}x{c[0][1]}-{c[1]}")
def test_small_matrix_momentum_in_kernel_over_steps(ctx, mx, case):
    """The momentum the small-matrix kernel forms itself, carried over
    steps, wide and tall, fused weight step or not (widths not a multiple
    of 4 take the separate apply pass): the buffer within 1e-5 of the
    oracle's, the update within the Newton-Schulz tolerance."""
    shape, dt, steps = case
    _step_case(ctx, mx, [shape], steps, dt, grad_std=1.0)
    w0 = wl.np_normal(shape, 0.02, seed=44, index=0, role=wl.ROLE_WEIGHT)
    w, b = dev(w0), torch.zeros(shape, device="cuda")
    buf = np.zeros(shape)
    wd = w0.astype(np.float64)
    for step in range(steps):
        g = wl.np_normal(shape, 1.0, seed=44, step=step, index=0)
        if dt == "bf16":
            g = wl.bf16_round_np(g)
        ctx.step([dict(weights=[w], grads=[dev(g, torch.bfloat16 if dt == "bf16" else torch.float32)],
                       momentum=[b])])
        torch.cuda.synchronize()
        w_prev = wd
        wd, buf, o = oracle.muon_step(w_prev, g, buf)
        assert rel_fro(to_np(b), buf) < EW_TOL, step
        scale = oracle.shape_scale(shape[0], shape[1], "original")
        upd = (w_prev * (1 - 0.02 * 0.01) - to_np(w)) / (0.02 * scale)
        assert rel_fro(upd, o) < ns_tol(shape), step
        wd = to_np(w)


def test_small_matrices_batched_past_the_pair_count(ctx, mx):
    """More small matrices than CTA pairs (each pair takes several in turn),
    of several shapes in one call, tall ones included, for the
    Newton-Schulz-only path and a fused step."""
    shapes = [(64, 200)] * 160 + [(256, 256)] * 2 + [(252, 20)] * 3 + [(96, 96)] * 5
    xs = [wl.np_normal(sh, 1.0, seed=41, index=i) for i, sh in enumerate(shapes)]
    outs = [torch.empty(sh, device="cuda") for sh in shapes]
    ctx.orthogonalize([dev(x, torch.bfloat16) for x in xs], outs)
    torch.cuda.synchronize()
    ctx.check_device()
    for i in list(range(0, 160, 13)) + list(range(160, len(shapes))):
        want = oracle.newton_schulz(wl.bf16_round_np(xs[i]), 5)
        assert rel_fro(to_np(outs[i]), want) < ns_tol(shapes[i]), (i, shapes[i])
    w0 = [wl.np_normal(sh, 0.02, seed=41, index=i, role=wl.ROLE_WEIGHT) for i, sh in enumerate(shapes)]
    wt = [dev(x) for x in w0]
    bt = [torch.zeros(sh, device="cuda") for sh in shapes]
    gt = [dev(x * 1e-3) for x in xs]
    by = {}
    for i, sh in enumerate(shapes):
        by.setdefault(sh, []).append(i)
    ctx.step([dict(weights=[wt[i] for i in ix], grads=[gt[i] for i in ix], momentum=[bt[i] for i in ix])
              for ix in by.values()])
    torch.cuda.synchronize()
    ctx.check_device()
    for i in list(range(0, 160, 29)) + list(range(160, len(shapes))):
        sh = shapes[i]
        _, _, o = oracle.muon_step(w0[i], (xs[i] * 1e-3).astype(np.float32), np.zeros(sh))
        scale = oracle.shape_scale(sh[0], sh[1], "original")
        upd = (w0[i].astype(np.float64) * (1 - 0.02 * 0.01) - to_np(wt[i])) / (0.02 * scale)
        assert rel_fro(upd, o) < ns_tol(sh), (i, sh)


def _step_case(ctx, mx, shapes, steps, grad_dtype, hp_over=None, seed=0, grad_std=1e-3):
    """Run `steps` Muon steps on GPU and oracle side by side; check momentum
    and staged apply every step, and the update against the oracle's."""
    hp_over = hp_over or {}
    hp = mx.default_hparams(**hp_over)
    ohp = {"scale": {0: "original", 1: "match_rms_adamw", 2: "none"}[hp.scale_mode],
           "lr": hp.lr, "weight_decay": hp.weight_decay, "momentum": hp.momentum,
           "nesterov": bool(hp.nesterov), "ns_steps": hp.ns_steps}
    tdt = torch.bfloat16 if grad_dtype == "bf16" else torch.float32
    w = [wl.np_normal(s, 0.02, seed=seed, index=i, role=wl.ROLE_WEIGHT).astype(np.float64)
         for i, s in enumerate(shapes)]
    buf = [np.zeros(s) for s in shapes]
    wt = [dev(x) for x in w]
    bt = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    ot = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    for step in range(steps):
        g = []
        for i, s in enumerate(shapes):
            x = wl.np_normal(s, grad_std, seed=seed, step=step, index=i)
            g.append(wl.bf16_round_np(x) if grad_dtype == "bf16" else x)
        gt = [dev(x, tdt) for x in g]
        w_prev = [to_np(t) for t in wt]
        by = {}
        for i, s in enumerate(shapes):
            by.setdefault(s, []).append(i)
        groups = [dict(weights=[wt[i] for i in ix], grads=[gt[i] for i in ix],
                       momentum=[bt[i] for i in ix], update_out=[ot[i] for i in ix])
                  for ix in by.values()]
        ctx.step(groups, hp)
        torch.cuda.synchronize()
        for i, s in enumerate(shapes):
            nb, u = oracle.nesterov_momentum(g[i], buf[i], ohp["momentum"], ohp["nesterov"])
            assert rel_fro(to_np(bt[i]), nb) < EW_TOL, f"momentum {s} step {step}"
            o_ref = oracle.newton_schulz(u, ohp["ns_steps"])
            o_gpu = to_np(ot[i])
            assert rel_fro(o_gpu, o_ref) < ns_tol(s), f"update {s} step {step}"
            scale = oracle.shape_scale(s[0], s[1], ohp["scale"])
            w_staged = oracle.apply_update(w_prev[i], o_gpu, ohp["lr"], ohp["weight_decay"], scale)
            assert rel_fro(to_np(wt[i]), w_staged) < EW_TOL, f"apply {s} step {step}"
            buf[i] = nb
        # carry the oracle buffer from its own arithmetic; weights from the GPU
    return wt, bt


def test_step_fused_apply_vs_oracle_and_unfused(ctx, mx):
    """Without update_out the last Newton-Schulz product applies the weight
    step in its epilogue (O stays in fp32 and never reaches memory).  Three
    steps on square, wide, tall and ragged shapes (widths a multiple of 4):
    momentum matches the oracle, the applied update (W_prev (1 - lr wd) -
    W_new) / (lr scale) matches the oracle's Newton-Schulz output, and on the
    first step it matches the unfused path's update_out up to bf16 rounding.
    A set holding a width that is not a multiple of 4 takes the unfused path."""
    hp = mx.default_hparams()
    decay = 1 - hp.lr * hp.weight_decay
    for shapes in ([(256, 256), (768, 3072), (3072, 768), (1000, 336), (520, 1028), (72, 8)],
                   [(130, 34), (96, 200)]):
        w = [wl.np_normal(s, 0.02, seed=21, index=i, role=wl.ROLE_WEIGHT) for i, s in enumerate(shapes)]
        wa = [dev(x) for x in w]
        wb = [dev(x) for x in w]
        ba = [torch.zeros(s, device="cuda") for s in shapes]
        bb = [torch.zeros(s, device="cuda") for s in shapes]
        ob = [torch.empty(s, device="cuda") for s in shapes]
        buf = [np.zeros(s) for s in shapes]
        for step in range(3):
            g = [wl.bf16_round_np(wl.np_normal(s, 1e-3, seed=21, step=step, index=i)) for i, s in enumerate(shapes)]
            gt = [dev(x, torch.bfloat16) for x in g]
            prev_a = [to_np(t) for t in wa]
            ctx.step([dict(weights=[wa[i]], grads=[gt[i]], momentum=[ba[i]]) for i in range(len(shapes))], hp)
            if step == 0:
                ctx.step([dict(weights=[wb[i]], grads=[gt[i]], momentum=[bb[i]], update_out=[ob[i]])
                          for i in range(len(shapes))], hp)
            torch.cuda.synchronize()
            ctx.check_device()
            for i, s in enumerate(shapes):
                nb, u = oracle.nesterov_momentum(g[i], buf[i])
                assert rel_fro(to_np(ba[i]), nb) < EW_TOL, (s, step)
                buf[i] = nb
                scale = oracle.shape_scale(s[0], s[1])
                upd = (prev_a[i] * decay - to_np(wa[i])) / (hp.lr * scale)
                assert rel_fro(upd, oracle.newton_schulz(u, 5)) < ns_tol(s), (s, step)
                if step == 0:
                    assert rel_fro(upd, to_np(ob[i])) < 5e-3, s
                    assert torch.equal(ba[i], bb[i]), s


def test_step_single_256_f32(ctx, mx):
    """One 256x256 fp32 gradient N(0,1), weights N(0,0.02), zero momentum,
    one step with the defaults."""
    _step_case(ctx, mx, [(256, 256)], 1, "f32", grad_std=1.0)


def test_step_gpt2_layer_bf16_multi_step(ctx, mx):
    """One GPT-2-small layer (Q, K, V, O, MLP in/out), bf16 gradients, three
    steps with momentum carried."""
    shapes = [(768, 768)] * 4 + [(3072, 768), (768, 3072)]
    _step_case(ctx, mx, shapes, 3, "bf16")


@pytest.mark.parametrize("over", [dict(scale_mode="match_rms_adamw"), dict(scale_mode="none"),
                                  dict(nesterov=0), dict(ns_steps=0), dict(ns_steps=3),
                                  dict(momentum=0.0, weight_decay=0.0),
                                  dict(lr=0.1, weight_decay=0.3)])
def test_step_hparam_variants(ctx, mx, over):
    _step_case(ctx, mx, [(96, 160), (160, 96), (33, 33)], 2, "f32", hp_over=over)


def test_step_ragged_edge_shapes(ctx, mx):
    shapes = [(1, 1), (1, 9), (9, 1), (3, 5), (5, 3), (65, 63), (130, 260), (260, 130), (257, 513)]
    _step_case(ctx, mx, shapes, 2, "bf16", grad_std=1.0)


def test_empty_and_zero(ctx, mx):
    # no groups, and a group of count 0, are no-ops
    ctx.step([], mx.default_hparams())
    # zero gradient: O = 0, W only decays
    w = torch.full((16, 24), 1.0, device="cuda")
    g = torch.zeros((16, 24), device="cuda")
    b = torch.zeros((16, 24), device="cuda")
    ctx.step([dict(weights=[w], grads=[g], momentum=[b])])
    torch.cuda.synchronize()
    assert torch.allclose(w, torch.full_like(w, 1.0 - 0.02 * 0.01), rtol=0, atol=1e-7)


def test_invalid_arguments_leave_tensors_untouched(ctx, mx):
    w = torch.ones((8, 8), device="cuda")
    g = torch.ones((8, 8), device="cuda")
    b = torch.zeros((8, 8), device="cuda")
    with pytest.raises(mx.MuonError) as e:
        ctx.step([dict(weights=[w], grads=[g], momentum=[b])], mx.default_hparams(ns_steps=-1))
    assert e.value.status == 1
    with pytest.raises(mx.MuonError):
        ctx.step([dict(weights=[w], grads=[g], momentum=[b])], mx.default_hparams(momentum=1.0))
    with pytest.raises(ValueError):
        ctx.step([dict(weights=[w], grads=[g[1:].contiguous()[:, :7].contiguous()], momentum=[b])])
    # the C ABI itself rejects a NULL tensor pointer
    import ctypes
    lib = mx.load_library()
    arr = (mx.binding.Group * 1)()
    arr[0].rows, arr[0].cols, arr[0].count, arr[0].grad_dtype = 8, 8, 1, 0
    nul = (ctypes.c_void_p * 1)(None)
    ok = (ctypes.c_void_p * 1)(w.data_ptr())
    arr[0].weights = ctypes.cast(ok, ctypes.c_void_p)
    arr[0].grads = ctypes.cast(nul, ctypes.c_void_p)
    arr[0].momentum = ctypes.cast(ok, ctypes.c_void_p)
    hp = mx.default_hparams()
    assert lib.muon_step(ctx._ctx, arr, 1, ctypes.byref(hp), None) == 1
    torch.cuda.synchronize()
    assert torch.all(w == 1) and torch.all(b == 0)


def test_nonfinite_gradient_is_rejected(ctx, mx):
    w = torch.ones((64, 96), device="cuda")
    g = torch.randn((64, 96), device="cuda")
    g[3, 5] = float("nan")
    b = torch.zeros((64, 96), device="cuda")
    with pytest.raises(mx.MuonError) as e:
        ctx.step([dict(weights=[w], grads=[g], momentum=[b])], mx.default_hparams(check_finite=1))
    assert e.value.status == 5
    assert torch.all(w == 1) and torch.all(b == 0)
    g[3, 5] = 0.0
    ctx.step([dict(weights=[w], grads=[g], momentum=[b])], mx.default_hparams(check_finite=1))
    torch.cuda.synchronize()
    assert not torch.all(w == 1)


def test_bounded_wait_reports_timeout_and_context_survives(ctx, mx):
    """Failure detection without a fault: a kernel waits on an mbarrier that
    nothing completes; its bounded wait gives up after 2 s, the timeout
    surfaces as MUON_ERR_TIMEOUT from check_device, the flag is cleared, and
    the context keeps computing correct results."""
    ctx.check_device()
    ctx.selftest_wait()
    with pytest.raises(mx.MuonError) as e:
        ctx.check_device()
    assert e.value.status == mx.binding.MUON_ERR_TIMEOUT
    ctx.check_device()
    g = wl.np_normal((256, 256), 1.0, seed=17, index=0)
    out = torch.empty((256, 256), device="cuda")
    ctx.orthogonalize([dev(g)], [out])
    torch.cuda.synchronize()
    ctx.check_device()
    assert rel_fro(to_np(out), oracle.newton_schulz(g, 5)) < NS_TOL


def test_engine_abort_sequence_reports_timeout_and_context_survives(ctx, mx):
    """Failure detection inside the Newton-Schulz engine without a fault: a
    Gram launch whose MMA thread never issues makes the TMA producer, the MMA
    thread and the epilogue of both CTAs give up after their bounded waits
    and run their abort sequences; MUON_ERR_TIMEOUT is reported once, and the
    same context then computes correct results (TMEM was released, no copy
    was left in flight)."""
    ctx.check_device()
    ctx.selftest_gemm()
    with pytest.raises(mx.MuonError) as e:
        ctx.check_device()
    assert e.value.status == mx.binding.MUON_ERR_TIMEOUT
    ctx.check_device()
    for shape in ((512, 768), (256, 256)):
        g = wl.np_normal(shape, 1.0, seed=43, index=shape[0])
        out = torch.empty(shape, device="cuda")
        ctx.orthogonalize([dev(g)], [out])
        torch.cuda.synchronize()
        ctx.check_device()
        assert rel_fro(to_np(out), oracle.newton_schulz(g, 5)) < NS_TOL


def test_timeout_halts_later_steps_until_checked(ctx, mx):
    """A bounded wait that gave up leaves the context's error flag set; every
    kernel of a later step then returns without writing, so the weights and
    momentum stay as they were (no half-computed update reaches them).
    check_device reports MUON_ERR_TIMEOUT and clears the flag, and the next
    step updates normally."""
    ctx.check_device()
    shape = (256, 384)
    w0 = wl.np_normal(shape, 0.02, seed=18, index=0, role=wl.ROLE_WEIGHT)
    g = wl.bf16_round_np(wl.np_normal(shape, 1e-3, seed=18, index=0))
    w, b = dev(w0), torch.zeros(shape, device="cuda")
    gt = dev(g, torch.bfloat16)
    p, pg = dev(np.ones(1000)), dev(np.ones(1000))
    pm, pv = torch.zeros(1000, device="cuda"), torch.zeros(1000, device="cuda")
    ctx.selftest_wait()
    ctx.step([dict(weights=[w], grads=[gt], momentum=[b])])
    ctx.adamw_step([p], [pg], [pm], [pv], 1)
    torch.cuda.synchronize()
    assert torch.equal(w, dev(w0)) and torch.count_nonzero(b) == 0
    assert torch.all(p == 1) and torch.count_nonzero(pm) == 0
    with pytest.raises(mx.MuonError) as e:
        ctx.check_device()
    assert e.value.status == mx.binding.MUON_ERR_TIMEOUT
    o = torch.empty(shape, device="cuda")
    ctx.step([dict(weights=[w], grads=[gt], momentum=[b], update_out=[o])])
    torch.cuda.synchronize()
    ctx.check_device()
    w1, b1, o1 = oracle.muon_step(w0, g, np.zeros(shape))
    assert rel_fro(to_np(b), b1) < EW_TOL
    assert rel_fro(to_np(o), o1) < NS_TOL


def test_nonfinite_flag_clears_for_the_next_unchecked_step(ctx, mx):
    """After a step rejected for a non-finite gradient, a step without the
    finite check still runs (the flag only halts the step that raised it)."""
    w = torch.ones((64, 96), device="cuda")
    g = torch.randn((64, 96), device="cuda")
    g[0, 0] = float("inf")
    b = torch.zeros((64, 96), device="cuda")
    with pytest.raises(mx.MuonError):
        ctx.step([dict(weights=[w], grads=[g], momentum=[b])], mx.default_hparams(check_finite=1))
    g[0, 0] = 0.0
    ctx.step([dict(weights=[w], grads=[g], momentum=[b])])
    torch.cuda.synchronize()
    assert not torch.all(w == 1) and torch.count_nonzero(b) > 0


def test_workspace_cap_and_caller_workspace(ctx, mx):
    """A bounded workspace (chunked execution) and a caller-owned workspace
    give the same result as the library's own."""
    shapes = [(256, 512)] * 6 + [(512, 256)] * 3 + [(128, 128)] * 4
    xs = [dev(wl.np_normal(s, 1.0, seed=10, index=i)) for i, s in enumerate(shapes)]
    ref = [torch.empty(s, device="cuda") for s in shapes]
    ctx.orthogonalize(xs, ref)
    per = 2 * 256 * 512 * 2 + 2 * 256 * 256 * 2 + 4096
    small = mx.MuonContext(0, workspace_bytes=3 * per)
    out = [torch.empty(s, device="cuda") for s in shapes]
    small.orthogonalize(xs, out)
    torch.cuda.synchronize()
    for a, b in zip(ref, out):
        assert torch.equal(a, b)
    small.close()
    wst = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")
    ctx.set_workspace(wst)
    out2 = [torch.empty(s, device="cuda") for s in shapes]
    ctx.orthogonalize(xs, out2)
    torch.cuda.synchronize()
    ctx.set_workspace(None)
    for a, b in zip(ref, out2):
        assert torch.equal(a, b)


def test_fused_step_chunked_matches_unchunked(ctx, mx):
    """The fused weight step under a bounded workspace (several chunks, each
    with its own descriptor table and last-product launch) leaves the same
    weights and momentum, bit for bit, as one unbounded call."""
    shapes = [(256, 512)] * 6 + [(512, 256)] * 3 + [(128, 128)] * 4
    w0 = [wl.np_normal(s, 0.02, seed=11, index=i, role=wl.ROLE_WEIGHT) for i, s in enumerate(shapes)]
    g = [dev(wl.bf16_round_np(wl.np_normal(s, 1e-3, seed=11, index=i)), torch.bfloat16)
         for i, s in enumerate(shapes)]
    per = 2 * 256 * 512 * 2 + 2 * 256 * 256 * 2 + 4096 + 256 * 512 * 4
    small = mx.MuonContext(0, workspace_bytes=3 * per)
    results = []
    for c in (ctx, small):
        w = [dev(x) for x in w0]
        b = [torch.zeros(s, device="cuda") for s in shapes]
        for _ in range(2):
            c.step([dict(weights=[w[i]], grads=[g[i]], momentum=[b[i]]) for i in range(len(shapes))])
        torch.cuda.synchronize()
        results.append((w, b))
    small.close()
    for (wa, ba), (wb, bb) in [(results[0], results[1])]:
        for x, y in zip(wa, wb):
            assert torch.equal(x, y)
        for x, y in zip(ba, bb):
            assert torch.equal(x, y)


def test_adamw_vs_oracle(ctx, mx):
    sizes = [1, 3, 768, 1000, 50257 * 8 + 3, 12345]
    ps = [wl.np_normal((n,), 0.02, seed=11, index=i, role=wl.ROLE_WEIGHT) for i, n in enumerate(sizes)]
    pt = [dev(p) for p in ps]
    mt = [torch.zeros(n, device="cuda") for n in sizes]
    vt = [torch.zeros(n, device="cuda") for n in sizes]
    m = [np.zeros(n) for n in sizes]
    v = [np.zeros(n) for n in sizes]
    w = [p.astype(np.float64) for p in ps]
    for step in range(1, 4):
        gs = [wl.bf16_round_np(wl.np_normal((n,), 1e-2, seed=11, step=step, index=i))
              for i, n in enumerate(sizes)]
        gt = [dev(g, torch.bfloat16) if i % 2 == 0 else dev(g) for i, g in enumerate(gs)]
        ctx.adamw_step(pt, gt, mt, vt, step)
        torch.cuda.synchronize()
        for i in range(len(sizes)):
            w_prev = to_np(pt[i]) if False else None
            w[i], m[i], v[i] = oracle.adamw_step(w[i], gs[i], m[i], v[i], step)
            assert rel_fro(to_np(mt[i]), m[i]) < EW_TOL
            assert rel_fro(to_np(vt[i]), v[i]) < EW_TOL
            assert rel_fro(to_np(pt[i]), w[i]) < EW_TOL


def test_newton_refresh_vs_oracle(ctx, mx):
    """S^-1 of the activation second moment: one block, four blocks, a
    ragged block width (partial panel) and the GPT-2 width 768."""
    tokens = 2048
    acts = [wl.bf16_round_np(wl.np_normal((tokens, 192), 1.0, seed=12, index=0, role=wl.ROLE_ACT)),
            wl.bf16_round_np(wl.np_normal((tokens, 4 * 96), 1.0, seed=12, index=1, role=wl.ROLE_ACT)),
            wl.bf16_round_np(wl.np_normal((tokens, 104), 1.0, seed=12, index=2, role=wl.ROLE_ACT)),
            wl.bf16_round_np(wl.np_normal((8192, 768), 1.0, seed=12, index=3, role=wl.ROLE_ACT))]
    nblocks = [1, 4, 1, 1]
    at = [dev(a, torch.bfloat16) for a in acts]
    si = [torch.empty((nb, a.shape[1] // nb, a.shape[1] // nb), device="cuda") for a, nb in zip(acts, nblocks)]
    ctx.newton_refresh(at, si, nblocks)
    torch.cuda.synchronize()
    ctx.check_device()
    for a, nb, s in zip(acts, nblocks, si):
        d = a.shape[1] // nb
        for b in range(nb):
            want = oracle.spd_inverse(oracle.second_moment(a[:, b * d:(b + 1) * d]))
            assert rel_fro(to_np(s[b]), want) < NEWTON_TOL


def test_newton_refresh_many_blocks_repeatable(ctx, mx):
    """A refresh of 84 blocks of width 768 (the GPT-2-small layer inputs:
    36 single-block activations and 12 four-block ones) launches far more
    Cholesky panel blocks than the GPU holds at once, so blocks of one
    matrix run at different times: three refreshes in a row give the same
    bits, and sampled blocks match the oracle."""
    tokens = 4096
    acts, outs, nbl = [], [], []
    for a in range(48):
        width, nb = (3072, 4) if a % 4 == 3 else (768, 1)
        x = wl.bf16_round_np(wl.np_normal((tokens, width), 1.0, seed=42, index=a, role=wl.ROLE_ACT))
        acts.append(x)
        nbl.append(nb)
    at = [dev(x, torch.bfloat16) for x in acts]
    runs = []
    for _ in range(3):
        outs = [torch.empty((nb, 768, 768), device="cuda") for nb in nbl]
        ctx.newton_refresh(at, outs, nbl)
        torch.cuda.synchronize()
        ctx.check_device()
        runs.append(outs)
    for other in runs[1:]:
        for x, y in zip(runs[0], other):
            assert torch.equal(x, y)
    for a in (0, 3, 17, 46, 47):
        for b in range(nbl[a]):
            want = oracle.spd_inverse(oracle.second_moment(acts[a][:, b * 768:(b + 1) * 768]))
            assert rel_fro(to_np(runs[0][a][b]), want) < NEWTON_TOL, (a, b)


def _s_inv_blocks(tokens, d, nb, seed, index):
    a = wl.bf16_round_np(wl.np_normal((tokens, nb * d), 1.0, seed=seed, index=index, role=wl.ROLE_ACT))
    return [oracle.spd_inverse(oracle.second_moment(a[:, b * d:(b + 1) * d])) for b in range(nb)]


# (rows, d, nb): tensor-core block widths (multiples of 64) with ragged row
# counts, then widths the fp32 tile kernel takes (multiples of 8 only).
PRECOND_CASES = [(200, 128, 1), (96, 64, 4), (300, 192, 2), (77, 104, 1), (130, 40, 2), (1, 8, 3)]


@pytest.mark.parametrize("case", PRECOND_CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}")
def test_newton_precondition_vs_oracle(ctx, mx, case):
    """The stand-alone right-preconditioning G S^-1 against the oracle's
    block-diagonal product, three gradients sharing one S^-1."""
    rows, d, nb = case
    blocks = _s_inv_blocks(512, d, nb, seed=14, index=d + nb)
    st = dev(np.stack(blocks))
    gs = [wl.bf16_round_np(wl.np_normal((rows, nb * d), 1e-3, seed=14, index=i)) for i in range(3)]
    out = [torch.full((rows, nb * d), float("nan"), device="cuda") for _ in gs]
    ctx.newton_precondition([dev(g, torch.bfloat16) for g in gs], [st] * 3, nb, out)
    torch.cuda.synchronize()
    ctx.check_device()
    for g, o in zip(gs, out):
        assert rel_fro(to_np(o), oracle.right_precondition(g, blocks)) < NEWTON_TOL


def test_newton_precondition_matches_step_and_batches(ctx, mx):
    """The stand-alone product equals the preconditioned gradient the step
    folds into its momentum (momentum starts at zero, beta = 0), for two
    S^-1 each shared by two gradients; a workspace that holds one S^-1's
    hi/lo stacks at a time (two staging batches) gives the same bits."""
    d, nb, rows = 128, 2, 256
    sa = dev(np.stack(_s_inv_blocks(1024, d, nb, seed=15, index=0)))
    sb = dev(np.stack(_s_inv_blocks(1024, d, nb, seed=15, index=1)))
    ss = [sa, sa, sb, sb]
    shape = (rows, nb * d)
    gt = [dev(wl.bf16_round_np(wl.np_normal(shape, 1e-3, seed=15, index=i)), torch.bfloat16) for i in range(4)]
    ref = [torch.empty(shape, device="cuda") for _ in gt]
    ctx.newton_precondition(gt, ss, nb, ref)
    wt = [torch.zeros(shape, device="cuda") for _ in gt]
    bt = [torch.zeros(shape, device="cuda") for _ in gt]
    ctx.step([dict(weights=wt, grads=gt, momentum=bt, precond=ss, precond_blocks=nb)],
             mx.default_hparams(momentum=0.0, nesterov=0, lr=0.0))
    torch.cuda.synchronize()
    for a, b in zip(ref, bt):
        assert torch.equal(a, b)
    stack = nb * 2 * d * d * 2
    wst = torch.empty(stack + 1024, dtype=torch.uint8, device="cuda")
    ctx.set_workspace(wst)
    out = [torch.empty(shape, device="cuda") for _ in gt]
    ctx.newton_precondition(gt, ss, nb, out)
    torch.cuda.synchronize()
    ctx.set_workspace(None)
    for a, b in zip(ref, out):
        assert torch.equal(a, b)


def test_newton_precondition_rejects_bad_arguments(ctx, mx):
    g = torch.zeros((64, 128), device="cuda", dtype=torch.bfloat16)
    s = torch.eye(128, device="cuda")[None].contiguous()
    o = torch.full((64, 128), 7.0, device="cuda")
    with pytest.raises(mx.MuonError):      # fp32 gradient
        ctx.newton_precondition([g.float()], [s], 1, [o])
    with pytest.raises(mx.MuonError):      # block width 128 / 3 not whole
        ctx.newton_precondition([g], [torch.zeros(3 * 42 * 42, device="cuda")], 3, [o])
    arr, keep = ctx.make_groups([dict(grads=[g], precond=[s], precond_blocks=1)])
    assert ctx._lib.muon_newton_precondition(ctx._ctx, arr, 1, None) == mx.binding.MUON_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.all(o == 7.0)


@pytest.mark.parametrize("case", [[((1001, 256), 2)], [((1001, 100), 1)], [((640, 90), 2), ((512, 128), 1)],
                                  [((1500, 301), 1)]],
                         ids=["in-place-ragged-tokens", "transposed-width-100", "transposed-odd-block-then-even",
                              "odd-width-301"])
def test_newton_refresh_paths(ctx, mx, case):
    """The second moment read in place (widths multiples of 8, here with a
    token count that is not) and through transposed copies (a width or block
    width that is not a multiple of 8; an odd block width followed, in the
    same call, by a block whose kernels take 16-byte vector paths) all match
    the oracle.  Width 301 runs doubling levels of 32, 64, 128 and 256 rows
    (ragged second blocks of 13 and 45 rows) on the element-by-element load
    paths of the inverse's kernels."""
    acts, outs = [], []
    for k, (shape, nb) in enumerate(case):
        a = wl.bf16_round_np(wl.np_normal(shape, 1.0, seed=16, index=shape[1] + k, role=wl.ROLE_ACT))
        d = shape[1] // nb
        acts.append((a, nb, d))
        outs.append(torch.empty((nb, d, d), device="cuda"))
    ctx.newton_refresh([dev(a, torch.bfloat16) for a, _, _ in acts], outs, [nb for _, nb, _ in acts])
    torch.cuda.synchronize()
    ctx.check_device()
    for (a, nb, d), s in zip(acts, outs):
        for b in range(nb):
            want = oracle.spd_inverse(oracle.second_moment(a[:, b * d:(b + 1) * d]))
            assert rel_fro(to_np(s[b]), want) < NEWTON_TOL


@pytest.mark.parametrize("case", [[((2048, 192), 1)], [((1001, 256), 2)], [((777, 100), 1)],
                                  [((1024, 128), 1, "bf16"), ((1024, 128), 1), ((512, 192), 2)]],
                         ids=["fp32-2048x192", "fp32-ragged-tokens-two-blocks", "fp32-odd-width",
                              "bf16-and-fp32-in-one-call"])
def test_newton_refresh_fp32_activations(ctx, mx, case):
    """fp32 activations (split into bf16 high and low parts whose three
    significant cross products the tensor cores sum in fp32) against the
    oracle's second moment of the same fp32 values; bf16 activations in the
    same call keep their own path."""
    acts, outs = [], []
    for k, spec in enumerate(case):
        shape, nb = spec[0], spec[1]
        a = wl.np_normal(shape, 1.0, seed=19, index=shape[1] + 7 * k, role=wl.ROLE_ACT)
        if len(spec) > 2:
            a = wl.bf16_round_np(a)
        acts.append((a, nb, shape[1] // nb, torch.bfloat16 if len(spec) > 2 else torch.float32))
        outs.append(torch.empty((nb, shape[1] // nb, shape[1] // nb), device="cuda"))
    ctx.newton_refresh([dev(a, dt) for a, _, _, dt in acts], outs, [nb for _, nb, _, _ in acts])
    torch.cuda.synchronize()
    ctx.check_device()
    for (a, nb, d, _), s in zip(acts, outs):
        for b in range(nb):
            want = oracle.spd_inverse(oracle.second_moment(a[:, b * d:(b + 1) * d].astype(np.float64)))
            assert rel_fro(to_np(s[b]), want) < NEWTON_TOL


def test_newton_muon_step_vs_oracle(ctx, mx):
    """Right-preconditioned step: shared S^-1 for Q/K/V-like matrices and a
    four-block S^-1 for the contraction."""
    d = 128
    tokens = 1024
    rng_acts = [wl.bf16_round_np(wl.np_normal((tokens, d), 1.0, seed=13, index=0, role=wl.ROLE_ACT)),
                wl.bf16_round_np(wl.np_normal((tokens, 4 * d), 1.0, seed=13, index=1, role=wl.ROLE_ACT))]
    s_in = [oracle.spd_inverse(oracle.second_moment(rng_acts[0]))]
    s_out = [oracle.spd_inverse(oracle.second_moment(rng_acts[1][:, b * d:(b + 1) * d])) for b in range(4)]
    si_a = dev(np.stack(s_in))
    si_b = dev(np.stack(s_out))
    shapes = [(d, d), (d, d), (d, d), (d, 4 * d)]
    ws = [wl.np_normal(s, 0.02, seed=13, index=i, role=wl.ROLE_WEIGHT) for i, s in enumerate(shapes)]
    gs = [wl.bf16_round_np(wl.np_normal(s, 1e-3, seed=13, index=i)) for i, s in enumerate(shapes)]
    wt = [dev(x) for x in ws]
    gt = [dev(x, torch.bfloat16) for x in gs]
    bt = [torch.zeros(s, device="cuda") for s in shapes]
    ot = [torch.empty(s, device="cuda") for s in shapes]
    groups = [dict(weights=wt[:3], grads=gt[:3], momentum=bt[:3], update_out=ot[:3],
                   precond=[si_a] * 3, precond_blocks=1),
              dict(weights=wt[3:], grads=gt[3:], momentum=bt[3:], update_out=ot[3:],
                   precond=[si_b], precond_blocks=4)]
    ctx.step(groups)
    torch.cuda.synchronize()
    for i, s in enumerate(shapes):
        blocks = s_in if i < 3 else s_out
        pg = oracle.right_precondition(gs[i], blocks)
        nb, u = oracle.nesterov_momentum(pg, np.zeros(s))
        assert rel_fro(to_np(bt[i]), nb) < NEWTON_TOL, f"preconditioned momentum {i}"
        assert rel_fro(to_np(ot[i]), oracle.newton_schulz(u, 5)) < NS_TOL


def test_newton_momentum_in_preconditioning_epilogue_edges(ctx, mx):
    """The preconditioning product that applies the momentum in its
    epilogue, on the shapes that exercise its edges: a tall matrix with a
    row count that is not a multiple of 32 (the wide layout is U^T and the
    last row tile is partly outside the matrix), a wide matrix with fewer
    than 256 rows, and two column blocks; Nesterov off and beta 0.9, two
    steps with the momentum carried, against the oracle at the fp32 bar (and
    the Newton-Schulz output at its own)."""
    hp = mx.default_hparams(momentum=0.9, nesterov=0)
    cases = [((1001, 256), 1), ((200, 768), 1), ((640, 256), 2)]
    tokens = 2048
    sinv_np, sinv_dev = [], []
    for i, ((rows, cols), nb) in enumerate(cases):
        d = cols // nb
        acts = wl.bf16_round_np(wl.np_normal((tokens, cols), 1.0, seed=33, index=i, role=wl.ROLE_ACT))
        blocks = [oracle.spd_inverse(oracle.second_moment(acts[:, b * d:(b + 1) * d])) for b in range(nb)]
        sinv_np.append(blocks)
        sinv_dev.append(dev(np.stack(blocks)))
    shapes = [c[0] for c in cases]
    wt = [dev(wl.np_normal(s, 0.02, seed=33, index=i, role=wl.ROLE_WEIGHT)) for i, s in enumerate(shapes)]
    bt = [torch.zeros(s, device="cuda") for s in shapes]
    ot = [torch.empty(s, device="cuda") for s in shapes]
    bufs = [np.zeros(s) for s in shapes]
    for step in range(2):
        gs = [wl.bf16_round_np(wl.np_normal(s, 1e-3, seed=33, step=step, index=i)) for i, s in enumerate(shapes)]
        gt = [dev(x, torch.bfloat16) for x in gs]
        ctx.step([dict(weights=[wt[i]], grads=[gt[i]], momentum=[bt[i]], update_out=[ot[i]],
                       precond=[sinv_dev[i]], precond_blocks=cases[i][1]) for i in range(len(cases))], hp)
        torch.cuda.synchronize()
        ctx.check_device()
        for i, s in enumerate(shapes):
            pg = oracle.right_precondition(gs[i], sinv_np[i])
            nb_, u = oracle.nesterov_momentum(pg, bufs[i], beta=0.9, nesterov=False)
            bufs[i] = nb_
            assert rel_fro(to_np(bt[i]), nb_) < NEWTON_TOL, (s, step)
            assert rel_fro(to_np(ot[i]), oracle.newton_schulz(u, 5)) < ns_tol(s), (s, step)


def test_newton_refresh_writes_split_and_step_uses_it(ctx, mx):
    """A refresh asked for the bf16 hi/lo split of each S^-1 writes exactly
    S_hi = bf16(S^-1) and S_lo = bf16(S^-1 - S_hi), block by block; a step
    given that split as precond_split is bit-identical to one that splits
    S^-1 itself (weights and momentum), over two steps, for a one-block and a
    four-block preconditioner shared by several matrices."""
    tokens = 2048
    specs = [(768, 1), (512, 4)]
    acts, sinv, splits, nblk = [], [], [], []
    for a, (width, nb) in enumerate(specs):
        d = width // nb
        acts.append(dev(wl.bf16_round_np(wl.np_normal((tokens, width), 1.0, seed=35, index=a, role=wl.ROLE_ACT)),
                        torch.bfloat16))
        sinv.append(torch.empty((nb, d, d), device="cuda"))
        splits.append(torch.empty((nb, 2 * d, d), dtype=torch.bfloat16, device="cuda"))
        nblk.append(nb)
    ctx.newton_refresh(acts, sinv, nblk, splits=splits)
    torch.cuda.synchronize()
    ctx.check_device()
    for s, sp, (width, nb) in zip(sinv, splits, specs):
        d = width // nb
        hi = s.to(torch.bfloat16)
        lo = (s - hi.float()).to(torch.bfloat16)
        assert torch.equal(sp[:, :d, :], hi)
        assert torch.equal(sp[:, d:, :], lo)
    shapes = [(768, 768), (768, 768), (1024, 768), (640, 512)]
    use = [0, 0, 0, 1]
    w0 = [dev(wl.np_normal(s, 0.02, seed=35, index=i, role=wl.ROLE_WEIGHT)) for i, s in enumerate(shapes)]
    wa, wb = [t.clone() for t in w0], [t.clone() for t in w0]
    ba, bb = [torch.zeros(s, device="cuda") for s in shapes], [torch.zeros(s, device="cuda") for s in shapes]
    for step in range(2):
        gt = [dev(wl.bf16_round_np(wl.np_normal(s, 1e-3, seed=35, step=step, index=i)), torch.bfloat16)
              for i, s in enumerate(shapes)]
        for w, bufs, with_split in ((wa, ba, False), (wb, bb, True)):
            groups = []
            for i, s in enumerate(shapes):
                g = dict(weights=[w[i]], grads=[gt[i]], momentum=[bufs[i]], precond=[sinv[use[i]]],
                         precond_blocks=nblk[use[i]])
                if with_split:
                    g["precond_split"] = [splits[use[i]]]
                groups.append(g)
            ctx.step(groups)
        torch.cuda.synchronize()
        ctx.check_device()
        for i in range(len(shapes)):
            assert torch.equal(ba[i], bb[i]), (shapes[i], step)
            assert torch.equal(wa[i], wb[i]), (shapes[i], step)
