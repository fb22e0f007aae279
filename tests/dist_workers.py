"""Worker functions for the multi-process (gloo, CPU) tests of the sharded
step.  Module level so that spawned processes can import them."""

import os
import sys
import traceback

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def _init(rank, world, port, timeout_s=60):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))
    return dist


SHAPES = [(48, 48), (48, 48), (96, 48), (48, 96), (32, 80), (80, 32), (48, 48), (16, 16)]


def _inputs():
    import workloads as wl
    ws = [wl.np_normal(s, 0.02, seed=5, index=i, role=wl.ROLE_WEIGHT).astype("float64")
          for i, s in enumerate(SHAPES)]
    gs = [[wl.np_normal(s, 1e-3, seed=5, step=k, index=i).astype("float64") for i, s in enumerate(SHAPES)]
          for k in range(3)]
    return ws, gs


def sharded_step_worker(rank, world, port, out_dir, stages=2):
    """Three sharded steps (each owner's matrices in `stages` slices whose
    exchange is issued right after the slice's step); every rank writes its
    final weights and the issue order of its last step."""
    try:
        import numpy as np
        import torch

        import oracle
        from matrix_aware_optimizer_step_b200.sharded import ShardedMuon
        dist = _init(rank, world, port)
        ws, gs = _inputs()
        weights = [torch.from_numpy(w.copy()) for w in ws]
        storages = {w.untyped_storage().data_ptr() for w in weights}
        sm = ShardedMuon(weights, stages=stages)
        # the weights now live in one flat buffer per (owner, stage)
        assert len({w.untyped_storage().data_ptr() for w in weights}) < len(storages)
        momentum = [torch.zeros_like(w) if i in sm.owned else None for i, w in enumerate(weights)]

        def local_step(owned, grads, mom):
            for i in owned:
                w1, b1, _ = oracle.muon_step(weights[i].numpy(), grads[i].numpy(), mom[i].numpy())
                weights[i].copy_(torch.from_numpy(w1))
                mom[i].copy_(torch.from_numpy(b1))

        sm.local_step = local_step
        for k in range(3):
            sm.step([torch.from_numpy(g) for g in gs[k]], momentum)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), owner=np.array(sm.owner),
                 *[w.numpy() for w in weights])
        with open(os.path.join(out_dir, f"trace{rank}.txt"), "w") as f:
            f.write(repr(sm.trace))
        dist.barrier()
        dist.destroy_process_group()
    except Exception:
        traceback.print_exc()
        raise


def dying_rank_worker(rank, world, port, out_dir):
    """Rank 1 raises before the exchange; rank 0 must get an error from its
    collective within the process-group timeout instead of hanging."""
    import torch

    from matrix_aware_optimizer_step_b200.sharded import ShardedMuon
    dist = _init(rank, world, port, timeout_s=5)
    ws, gs = _inputs()
    weights = [torch.from_numpy(w.copy()) for w in ws]
    sm = ShardedMuon(weights, local_step=lambda owned, g, m: None)
    if rank == 1:
        os._exit(3)          # leaves without joining the exchange
    try:
        sm.exchange()
        status = "no-error"
    except Exception as e:   # timeout or connection closed
        status = "error:" + type(e).__name__
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(status)
    os._exit(0)
