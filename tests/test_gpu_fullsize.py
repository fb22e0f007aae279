"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (grouped calls over all matrices of the workload).

Where the fp64 oracle can afford it, whole matrices are compared (every
shape of one Llama-3-8B layer, one GPT-2-small layer per step).  Everywhere
else the checks are ones the oracle can make element by element or that
hold at any size: the momentum buffer and the staged apply on sampled
elements, finiteness, and the norm of the orthogonalised update (its
singular values lie in the quintic's band, so ||O||_F / sqrt(m) does too).
"""

import numpy as np
import pytest

import oracle
import workloads as wl
from helpers import EW_TOL, NS_TOL, rel_fro

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    import matrix_aware_optimizer_step_b200 as m
    return m


def _np(t):
    return t.detach().double().cpu().numpy()


def _sample_idx(numel, k, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.choice(numel, size=min(k, numel), replace=False)).cuda()


def _band_ok(o, rows, cols):
    m = min(rows, cols)
    r = float(torch.linalg.vector_norm(o.float()).item()) / np.sqrt(m)
    return 0.6 < r < 1.25, r


def test_llama3_8b_step_full_size(mx):
    """One Llama-3-8B-shaped step (224 matrices, bf16 grads N(0,1e-3), fp32
    weights N(0,0.02), zero momentum), run in three calls of whole layers.
    Every matrix: momentum and staged apply on 4096 sampled elements,
    finiteness, the singular-value band; the seven matrices of layers 0 and
    31: the whole Newton-Schulz output against the fp64 oracle."""
    dev = torch.device("cuda")
    mats = wl.llama3_8b_mats()
    hp = mx.default_hparams()
    layer_sets = [list(range(0, 77)), list(range(77, 154)), list(range(154, 224))]
    with mx.MuonContext(0) as ctx:
        for part, ids in enumerate(layer_sets):
            W, G, B, O, samp = {}, {}, {}, {}, {}
            for i in ids:
                m = mats[i]
                W[i] = wl.torch_normal((m.rows, m.cols), 0.02, 3, 0, i, wl.ROLE_WEIGHT, device=dev)
                G[i] = wl.torch_normal((m.rows, m.cols), 1e-3, 3, 0, i, wl.ROLE_GRAD, dtype=torch.bfloat16, device=dev)
                B[i] = torch.zeros((m.rows, m.cols), device=dev)
                O[i] = torch.empty((m.rows, m.cols), device=dev)
                idx = _sample_idx(m.rows * m.cols, 4096, seed=i)
                samp[i] = (idx, W[i].view(-1)[idx].double().cpu().numpy(), G[i].view(-1)[idx].double().cpu().numpy())
            # every matrix of the first and the last layer against the full oracle
            full = {i: (W[i].double().cpu().numpy(), G[i].double().cpu().numpy()) for i in ids
                    if i < 7 or i >= len(mats) - 7}
            groups = {}
            for i in ids:
                groups.setdefault((mats[i].rows, mats[i].cols), []).append(i)
            ctx.step([dict(weights=[W[i] for i in ix], grads=[G[i] for i in ix], momentum=[B[i] for i in ix],
                           update_out=[O[i] for i in ix]) for ix in groups.values()], hp)
            torch.cuda.synchronize()
            ctx.check_device()
            for i in ids:
                m = mats[i]
                idx, w0, g0 = samp[i]
                nb, _ = oracle.nesterov_momentum(g0, np.zeros_like(g0))
                assert rel_fro(B[i].view(-1)[idx].double().cpu().numpy(), nb) < EW_TOL, m.name
                assert bool(torch.isfinite(O[i]).all()), m.name
                ok, r = _band_ok(O[i], m.rows, m.cols)
                assert ok, (m.name, r)
                o_s = O[i].view(-1)[idx].double().cpu().numpy()
                want = oracle.apply_update(w0, o_s, hp.lr, hp.weight_decay, oracle.shape_scale(m.rows, m.cols))
                assert rel_fro(W[i].view(-1)[idx].double().cpu().numpy(), want) < EW_TOL, m.name
            for i, (w0, g0) in full.items():
                _, u = oracle.nesterov_momentum(g0, np.zeros_like(g0))
                err = rel_fro(_np(O[i]), oracle.newton_schulz(u, 5))
                assert err < NS_TOL, (mats[i].name, err)
            del W, G, B, O
            torch.cuda.empty_cache()


def test_gpt2_small_ten_steps_full_size(mx):
    """All 72 GPT-2-small hidden matrices, bf16 grads N(0,1e-3) drawn per
    step, momentum carried over 10 steps.  Every step: the whole momentum
    buffer and the staged apply of every matrix against the oracle, and the
    full Newton-Schulz of one layer (rotating) against the oracle."""
    dev = torch.device("cuda")
    mats = wl.gpt2_small_mats()
    hp = mx.default_hparams()
    W = [wl.torch_normal((m.rows, m.cols), 0.02, 4, 0, i, wl.ROLE_WEIGHT, device=dev) for i, m in enumerate(mats)]
    B = [torch.zeros((m.rows, m.cols), device=dev) for m in mats]
    O = [torch.empty((m.rows, m.cols), device=dev) for m in mats]
    bufs = [np.zeros((m.rows, m.cols)) for m in mats]
    groups = {}
    for i, m in enumerate(mats):
        groups.setdefault((m.rows, m.cols), []).append(i)
    with mx.MuonContext(0) as ctx:
        for step in range(10):
            G = [wl.torch_normal((m.rows, m.cols), 1e-3, 4, step, i, wl.ROLE_GRAD, dtype=torch.bfloat16, device=dev)
                 for i, m in enumerate(mats)]
            w_prev = [_np(w) for w in W]
            ctx.step([dict(weights=[W[i] for i in ix], grads=[G[i] for i in ix], momentum=[B[i] for i in ix],
                           update_out=[O[i] for i in ix]) for ix in groups.values()], hp)
            torch.cuda.synchronize()
            layer = step % 12
            for i, m in enumerate(mats):
                g = _np(G[i])
                nb, u = oracle.nesterov_momentum(g, bufs[i])
                assert rel_fro(_np(B[i]), nb) < EW_TOL, (m.name, step)
                bufs[i] = nb
                o = _np(O[i])
                want = oracle.apply_update(w_prev[i], o, hp.lr, hp.weight_decay, oracle.shape_scale(m.rows, m.cols))
                assert rel_fro(_np(W[i]), want) < EW_TOL, (m.name, step)
                if i // 6 == layer:
                    assert rel_fro(o, oracle.newton_schulz(u, 5)) < NS_TOL, (m.name, step)


@pytest.mark.parametrize("size", [1024, 2048, 4096, 8192])
def test_square_sweep_full_size(mx, size):
    """32 square bf16 matrices N(0,1), Newton-Schulz only.  One matrix per
    size against the full oracle up to 2048; every matrix: finite, in band."""
    dev = torch.device("cuda")
    n = 32
    X = [wl.torch_normal((size, size), 1.0, 6, 0, i, wl.ROLE_GRAD, dtype=torch.bfloat16, device=dev) for i in range(n)]
    O = [torch.empty((size, size), device=dev) for _ in range(n)]
    with mx.MuonContext(0) as ctx:
        ctx.orthogonalize(X, O)
        torch.cuda.synchronize()
        ctx.check_device()
    for i in range(n):
        assert bool(torch.isfinite(O[i]).all())
        ok, r = _band_ok(O[i], size, size)
        assert ok, (size, i, r)
    if size <= 2048:
        err = rel_fro(_np(O[5]), oracle.newton_schulz(_np(X[5]), 5))
        assert err < NS_TOL, (size, err)


def test_newton_muon_gpt2_small_ten_steps_full_size(mx):
    """Newton-Muon on the GPT-2-small shapes at full size: per layer the
    activations feeding Q/K/V (one shared estimate), O, the MLP expansion
    (8192 x 768 each) and the MLP contraction (8192 x 3072, four 768-wide
    blocks), N(0,1) bf16; S^-1 refreshed at step 0 for all 84 blocks, then
    10 steps with momentum carried ("The Newton-Muon Optimizer", "What Is
    Newton-Muon?").  Every step: the momentum of every matrix (the
    preconditioned gradient's moving average) against the fp64 oracle within
    the fp32 bar, the staged apply of every matrix, and the whole
    Newton-Schulz output of one layer (rotating)."""
    from helpers import NEWTON_TOL
    dev = torch.device("cuda")
    w = wl.newton_gpt2_small()
    mats = w.mats
    hp = mx.default_hparams()
    acts, sinv, nblk = [], [], []
    for a, (_, tokens, width) in enumerate(w.acts):
        nb = 4 if width > 768 else 1
        acts.append(wl.torch_normal((tokens, width), 1.0, 8, 0, a, wl.ROLE_ACT, dtype=torch.bfloat16, device=dev))
        sinv.append(torch.empty((nb, width // nb, width // nb), device=dev))
        nblk.append(nb)
    W = [wl.torch_normal((m.rows, m.cols), 0.02, 8, 0, i, wl.ROLE_WEIGHT, device=dev) for i, m in enumerate(mats)]
    B = [torch.zeros((m.rows, m.cols), device=dev) for m in mats]
    O = [torch.empty((m.rows, m.cols), device=dev) for m in mats]
    groups = {}
    for i, m in enumerate(mats):
        groups.setdefault((m.rows, m.cols), []).append(i)
    # the oracle's inverses from the same bf16 activations, in fp64
    s_or = []
    for a, nb in zip(acts, nblk):
        x = _np(a)
        d = x.shape[1] // nb
        s_or.append([oracle.spd_inverse(oracle.second_moment(x[:, b * d:(b + 1) * d])) for b in range(nb)])
    bufs = [np.zeros((m.rows, m.cols)) for m in mats]
    with mx.MuonContext(0) as ctx:
        ctx.newton_refresh(acts, sinv, nblk)
        torch.cuda.synchronize()
        ctx.check_device()
        worst = max(rel_fro(_np(sinv[a][b]), s_or[a][b]) for a in range(len(acts)) for b in range(nblk[a]))
        assert worst < NEWTON_TOL, worst
        for step in range(10):
            G = [wl.torch_normal((m.rows, m.cols), 1e-3, 8, step, i, wl.ROLE_GRAD, dtype=torch.bfloat16,
                                 device=dev) for i, m in enumerate(mats)]
            w_prev = [_np(x) for x in W]
            gs = []
            for ix in groups.values():
                a0, nb = w.precond[mats[ix[0]].name]
                gs.append(dict(weights=[W[i] for i in ix], grads=[G[i] for i in ix], momentum=[B[i] for i in ix],
                               update_out=[O[i] for i in ix],
                               precond=[sinv[w.precond[mats[i].name][0]] for i in ix], precond_blocks=nb))
            ctx.step(gs, hp)
            torch.cuda.synchronize()
            ctx.check_device()
            layer = step % 12
            for i, m in enumerate(mats):
                a, _ = w.precond[m.name]
                pg = oracle.right_precondition(_np(G[i]), s_or[a])
                nb_, u = oracle.nesterov_momentum(pg, bufs[i])
                assert rel_fro(_np(B[i]), nb_) < NEWTON_TOL, (m.name, step)
                bufs[i] = nb_
                o = _np(O[i])
                want = oracle.apply_update(w_prev[i], o, hp.lr, hp.weight_decay, oracle.shape_scale(m.rows, m.cols))
                assert rel_fro(_np(W[i]), want) < EW_TOL, (m.name, step)
                if i // 6 == layer:
                    assert rel_fro(o, oracle.newton_schulz(u, 5)) < NS_TOL, (m.name, step)


@pytest.mark.parametrize("shape", [(16384, 131136), (131136, 16384)], ids=["wide", "tall"])
def test_single_matrix_past_2_31_elements(mx, shape):
    """One matrix of 2.15 G elements (more than 2^31, so every element,
    tile and byte offset needs 64 bits), bf16 gradient N(0,1e-3), fp32
    weights N(0,0.02), zero momentum, one step; both orientations (the tall
    one goes through the transposing momentum tile).  Unfused first, with the
    update written out: the momentum and the staged apply on sampled elements
    (among them the first, the last and those around index 2^31) against the
    oracle, the update finite and in the quintic's band.  Then the same step
    fused: the applied update on the same elements against the unfused one,
    up to bf16 rounding, and the momentum bit for bit."""
    dev = torch.device("cuda")
    rows, cols = shape
    numel = rows * cols
    assert numel > 2 ** 31
    hp = mx.default_hparams()
    decay = 1.0 - hp.lr * hp.weight_decay
    scale = oracle.shape_scale(rows, cols)
    G = wl.torch_normal(shape, 1e-3, 9, 0, 0, wl.ROLE_GRAD, dtype=torch.bfloat16, device=dev)
    W = wl.torch_normal(shape, 0.02, 9, 0, 0, wl.ROLE_WEIGHT, device=dev)
    B = torch.zeros(shape, device=dev)
    O = torch.empty(shape, device=dev)
    special = [0, 1, 2 ** 31 - 1, 2 ** 31, 2 ** 31 + 1, 2 ** 31 + 12345, numel - cols, numel - 1]
    rng = np.random.default_rng(31)
    idx_np = np.unique(np.concatenate([rng.integers(0, numel, 4096), np.array(special)]))
    idx = torch.from_numpy(idx_np).to(dev)
    w0 = W.view(-1)[idx].double().cpu().numpy()
    g0 = G.view(-1)[idx].double().cpu().numpy()
    with mx.MuonContext(0) as ctx:
        ctx.step([dict(weights=[W], grads=[G], momentum=[B], update_out=[O])], hp)
        torch.cuda.synchronize()
        ctx.check_device()
        nb, _ = oracle.nesterov_momentum(g0, np.zeros_like(g0))
        b1 = B.view(-1)[idx].clone()
        assert rel_fro(b1.double().cpu().numpy(), nb) < EW_TOL
        assert bool(torch.isfinite(O).all())
        ok, r = _band_ok(O, rows, cols)
        assert ok, r
        o1 = O.view(-1)[idx].double().cpu().numpy()
        want = oracle.apply_update(w0, o1, hp.lr, hp.weight_decay, scale)
        assert rel_fro(W.view(-1)[idx].double().cpu().numpy(), want) < EW_TOL
        del O
        torch.cuda.empty_cache()
        # the same step with the weight update fused into the last product
        wl.torch_normal(shape, 0.02, 9, 0, 0, wl.ROLE_WEIGHT, device=dev, out=W)
        B.zero_()
        ctx.step([dict(weights=[W], grads=[G], momentum=[B])], hp)
        torch.cuda.synchronize()
        ctx.check_device()
        assert torch.equal(B.view(-1)[idx], b1)
        upd = (w0 * decay - W.view(-1)[idx].double().cpu().numpy()) / (hp.lr * scale)
        assert rel_fro(upd, o1) < 5e-3
