"""ShardedMuon's default path (the library's step on the owned matrices)
on one GPU as a world of one rank: identical to calling the step directly."""

import os
import socket

import numpy as np
import pytest

import workloads as wl

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def test_sharded_world_of_one_equals_direct_step():
    import torch.distributed as dist

    import matrix_aware_optimizer_step_b200 as mx
    from matrix_aware_optimizer_step_b200.sharded import ShardedMuon
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        shapes = [(256, 256), (256, 256), (512, 256), (256, 512)]
        w = [torch.from_numpy(wl.np_normal(sh, 0.02, seed=21, index=i, role=wl.ROLE_WEIGHT)).cuda()
             for i, sh in enumerate(shapes)]
        g = [torch.from_numpy(wl.np_normal(sh, 1e-3, seed=21, index=i)).cuda().to(torch.bfloat16)
             for i, sh in enumerate(shapes)]
        w2 = [x.clone() for x in w]
        b = [torch.zeros_like(x) for x in w]
        b2 = [torch.zeros_like(x) for x in w]
        with mx.MuonContext(0) as ctx:
            sm = ShardedMuon(w, ctx=ctx, hp=mx.default_hparams())
            assert sm.owned == list(range(len(shapes)))
            sm.step(g, b)
            groups = {}
            for i, sh in enumerate(shapes):
                groups.setdefault(sh, []).append(i)
            ctx.step([dict(weights=[w2[i] for i in ix], grads=[g[i] for i in ix], momentum=[b2[i] for i in ix])
                      for ix in groups.values()])
            torch.cuda.synchronize()
        for x, y in zip(w, w2):
            assert torch.equal(x, y)
    finally:
        dist.destroy_process_group()
