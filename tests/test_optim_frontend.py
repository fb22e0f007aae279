"""MuonWithAuxAdam: the README's param-group interface driving the library."""

import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")


def test_rejects_bad_groups_without_gpu():
    from matrix_aware_optimizer_step_b200.optim import MuonWithAuxAdam
    p = torch.nn.Parameter(torch.zeros(4, 4))
    with pytest.raises(ValueError):
        MuonWithAuxAdam([dict(params=[p])])                    # no use_muon
    with pytest.raises(ValueError):
        MuonWithAuxAdam([dict(params=[p], use_muon=True)])     # CPU tensor


@pytest.mark.gpu
def test_matches_library_calls_and_trains_a_toy_model():
    """The first step equals direct library calls bit for bit (Muon matrix)
    and the fp64 AdamW oracle (an aux tensor); then the model trains."""
    import matrix_aware_optimizer_step_b200 as mx
    from matrix_aware_optimizer_step_b200.optim import MuonWithAuxAdam
    torch.manual_seed(0)
    model = torch.nn.Sequential(torch.nn.Linear(64, 256), torch.nn.GELU(), torch.nn.Linear(256, 256),
                                torch.nn.GELU(), torch.nn.Linear(256, 8)).cuda()
    hidden = [model[2].weight]
    rest = [p for n, p in model.named_parameters() if p is not model[2].weight]
    opt = MuonWithAuxAdam([dict(params=hidden, use_muon=True, lr=0.02, weight_decay=0.01),
                           dict(params=rest, use_muon=False, lr=3e-3, betas=(0.9, 0.95), weight_decay=0.01)])
    x = torch.randn(512, 64, device="cuda")
    y = torch.randn(512, 8, device="cuda")
    loss = torch.nn.functional.mse_loss(model(x), y)
    loss.backward()
    w_ref = model[2].weight.detach().clone()
    g_ref = model[2].weight.grad.detach().clone()
    b_ref = torch.zeros_like(w_ref)
    b0 = model[0].bias.detach().double().cpu().numpy()
    gb = model[0].bias.grad.double().cpu().numpy()
    opt.step()
    with mx.MuonContext(0) as ctx:
        ctx.step([dict(weights=[w_ref], grads=[g_ref], momentum=[b_ref])], mx.default_hparams())
    torch.cuda.synchronize()
    assert torch.equal(model[2].weight.detach(), w_ref)
    assert torch.equal(opt.state[model[2].weight]["momentum_buffer"], b_ref)
    bb, _, _ = oracle.adamw_step(b0, gb, np.zeros_like(gb), np.zeros_like(gb), 1,
                                 dict(lr=3e-3, beta1=0.9, beta2=0.95, weight_decay=0.01))
    assert np.abs(model[0].bias.detach().double().cpu().numpy() - bb).max() < 1e-6
    first = loss.item()
    for _ in range(40):
        opt.zero_grad(set_to_none=True)
        loss = torch.nn.functional.mse_loss(model(x), y)
        loss.backward()
        opt.step()
    assert loss.item() < 0.7 * first


@pytest.mark.gpu
def test_device_timeout_leaves_parameters_untouched_and_check_raises():
    """After a bounded device-side wait gave up, optimizer steps change no
    parameter and no state; the periodic check raises MUON_ERR_TIMEOUT, and
    stepping resumes afterwards."""
    import matrix_aware_optimizer_step_b200 as mx
    from matrix_aware_optimizer_step_b200.optim import MuonWithAuxAdam
    torch.manual_seed(1)
    w = torch.nn.Parameter(torch.randn(128, 192, device="cuda") * 0.02)
    b = torch.nn.Parameter(torch.zeros(192, device="cuda"))
    opt = MuonWithAuxAdam([dict(params=[w], use_muon=True), dict(params=[b], use_muon=False)], check_every=2)
    w.grad = torch.randn_like(w) * 1e-3
    b.grad = torch.randn_like(b) * 1e-3
    w0, b0 = w.detach().clone(), b.detach().clone()
    opt.ctx.selftest_wait()
    opt.step()                                   # no check yet: halted on the device
    torch.cuda.synchronize()
    assert torch.equal(w, w0) and torch.equal(b, b0)
    assert torch.count_nonzero(opt.state[w]["momentum_buffer"]) == 0
    with pytest.raises(mx.MuonError) as e:
        opt.step()                               # second step: the check raises
    assert e.value.status == mx.binding.MUON_ERR_TIMEOUT
    assert torch.equal(w, w0) and torch.equal(b, b0)
    opt.step()
    torch.cuda.synchronize()
    assert not torch.equal(w, w0) and not torch.equal(b, b0)
