"""materialize_lm_weight on the CPU with two gloo ranks: the gathered head equals
the full head, the head's gradient is the SUM of the ranks' full-weight
gradients sliced to each rank's shard (uneven shards too), and a trainable
sharded head without a matching reduction group is refused."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, rows, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from torch.distributed.device_mesh import init_device_mesh
    from torch.distributed.tensor import Shard, distribute_tensor

    from lm_head_projection_flce_b200.distributed import materialize_lm_weight

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mesh = init_device_mesh("cpu", (world,))
        g = torch.Generator().manual_seed(0)
        full = torch.randn(rows, 4, generator=g)
        dt = distribute_tensor(full, mesh, [Shard(0)])
        dt.requires_grad_(True)
        res = {}
        # a trainable sharded head without a group is refused
        try:
            materialize_lm_weight(dt, None)
            res["refused"] = False
        except ValueError:
            res["refused"] = True
        w = materialize_lm_weight(dt, dist.group.WORLD)
        res["gathered_ok"] = bool(torch.equal(w, full))
        coeffs = [torch.randn(rows, 4, generator=torch.Generator().manual_seed(100 + r))
                  for r in range(world)]
        (w * coeffs[rank]).sum().backward()
        want = sum(coeffs)
        per = -(-rows // world)
        lo, hi = rank * per, min(rows, (rank + 1) * per)
        local_grad = dt.grad.to_local()
        res["grad_ok"] = bool(torch.allclose(local_grad, want[lo:hi], atol=1e-6))
        res["grad_rows"] = int(local_grad.shape[0])
        plain = torch.randn(3, 2)
        res["plain_identity"] = materialize_lm_weight(plain, None) is plain
        out.put((rank, res))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _mismatch_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from torch.distributed.device_mesh import init_device_mesh
    from torch.distributed.tensor import Shard, distribute_tensor

    from lm_head_projection_flce_b200.distributed import materialize_lm_weight

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mesh = init_device_mesh("cpu", (world,))
        dt = distribute_tensor(torch.zeros(8, 2), mesh, [Shard(0)])
        dt.requires_grad_(True)
        groups = [dist.new_group([r]) for r in range(world)]
        try:
            materialize_lm_weight(dt, groups[rank])
            out.put((rank, False))
        except ValueError:
            out.put((rank, True))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _spawn(target, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, *args, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    return dict(q.get(timeout=10) for _ in range(world))


@pytest.mark.parametrize("rows", [10, 11])
def test_gather_and_summed_gradient_two_ranks(rows):
    res = _spawn(_worker, 2, rows)
    for r in (0, 1):
        assert res[r]["refused"] and res[r]["gathered_ok"] and res[r]["grad_ok"]
        assert res[r]["plain_identity"]
    assert res[0]["grad_rows"] + res[1]["grad_rows"] == rows


def test_group_size_must_match_the_mesh():
    res = _spawn(_mismatch_worker, 2)
    assert res == {0: True, 1: True}
