"""The data-parallel wrapper on one GPU over NCCL (a one-rank group: the
all-gather and reduce-scatter are identities), against the plain fused path:
same loss, same dhidden, same head gradient delivered into the DTensor shard."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(port, out, head_dtype="bf16", fused_head_cast=False):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from torch.distributed.device_mesh import init_device_mesh
    from torch.distributed.tensor import Shard, distribute_tensor

    from lm_head_projection_flce_b200 import flce
    from lm_head_projection_flce_b200 import workloads as W
    from lm_head_projection_flce_b200.distributed import data_parallel_fused_linear_cross_entropy

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev)
    try:
        w = W.custom(700, 520, 5000, 5120, softcap=30.0, ignore_frac=0.1, w_sigma=0.05, seed=41,
                     w_dtype=head_dtype)
        d = W.generate(w)
        hid = d["hidden"].to(dev).requires_grad_(True)
        lab = d["labels"].to(dev)
        mesh = init_device_mesh("cuda", (1,))
        dt = distribute_tensor(d["weight"].to(dev), mesh, [Shard(0)])
        dt.requires_grad_(True)
        loss = data_parallel_fused_linear_cross_entropy(
            hid, dt, lab, num_label_tokens=d["num_label_tokens"], grad_reduce_group=dist.group.WORLD,
            softcap=w.softcap, unpadded_vocab=w.vocab, fused_head_cast=fused_head_cast)
        loss.backward()
        h2 = d["hidden"].to(dev).requires_grad_(True)
        w2 = d["weight"].to(dev).requires_grad_(True)
        ref = flce.fused_linear_cross_entropy(h2, w2, lab, softcap=w.softcap, unpadded_vocab=w.vocab,
                                              num_label_tokens=d["num_label_tokens"])
        ref.backward()
        torch.cuda.synchronize(dev)
        out.put({"loss": abs(float(loss) - float(ref)) <= 1e-6 * abs(float(ref)),
                 "dh": bool(torch.equal(hid.grad, h2.grad)),
                 "dw": bool(torch.equal(dt.grad.to_local(), w2.grad))})
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("head_dtype,fused", [("bf16", False), ("f32", False), ("f32", True)])
def test_data_parallel_wrapper_single_rank_nccl(head_dtype, fused):
    """The wrapper over a one-rank group equals the plain fused loss bit for bit,
    for a BF16 head and for FP32 master weights (whose BF16 copy the autograd
    wrapper keeps from the forward for the backward, or which the GEMMs round
    in the kernel with fused_head_cast)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_worker, args=(_free_port(), q, head_dtype, fused))
    p.start()
    p.join(timeout=300)
    assert p.exitcode == 0
    assert q.get(timeout=10) == {"loss": True, "dh": True, "dw": True}
