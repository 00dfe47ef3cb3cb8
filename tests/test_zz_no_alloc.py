"""The forward entry point that allocates nothing (flce_forward_noalloc).

Some callers cannot give this library scratch memory: a plugin running inside
a framework whose allocator owns all device memory and has no way to lend a
workspace, or a service that forbids device allocations after start-up because
an allocation failing mid-run cannot be recovered.  For them the forward keeps
its scratch in a fixed 32 MiB array inside the library.  These tests call that
entry point through the C ABI and check it against flce_forward, which takes a
caller-provided workspace, on consecutive calls that reuse the same array.

This file is collected last so that a run stopping at its first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from lm_head_projection_flce_b200 import flce
from lm_head_projection_flce_b200 import workloads as W

from gpu_common import LOSS_REL, LSE_ABS, gpu_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return gpu_device()


def _inputs(w, dev, labels=None):
    d = W.generate(w)
    lab = d["labels"] if labels is None else labels
    return d["hidden"].to(dev), d["weight"].to(dev), lab.to(dev), d


def _with_workspace(w, hid, wt, lab, reduction, nlt):
    loss, lse = flce.forward(hid, wt, lab, softcap=w.softcap, unpadded_vocab=w.vocab,
                             reduction=reduction, num_label_tokens=nlt)
    return loss.clone(), lse.clone()


def _no_alloc(w, hid, wt, lab, reduction, nlt):
    lib = flce.load_library()
    n, h = hid.shape
    loss = torch.full((n if reduction == "none" else 1,), float("nan"), device=hid.device)
    lse = torch.full((n,), float("nan"), device=hid.device)
    st = lib.flce_forward_noalloc(
        ctypes.c_void_p(hid.data_ptr()), ctypes.c_void_p(wt.data_ptr()),
        flce.W_DTYPES[wt.dtype], ctypes.c_void_p(lab.data_ptr()), n, h, wt.shape[0], w.vocab,
        -100, float(w.softcap), flce.REDUCTIONS[reduction], int(nlt or 0),
        ctypes.c_void_p(loss.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream(hid.device).cuda_stream))
    assert st == flce.FLCE_OK, flce.STATUS.get(st, st)
    return loss, lse


def _same(a, b):
    (loss_a, lse_a), (loss_b, lse_b) = a, b
    torch.cuda.synchronize()
    la = loss_a.double().cpu().numpy().reshape(-1)
    lb = loss_b.double().cpu().numpy().reshape(-1)
    assert float(np.max(np.abs(lse_a.double().cpu().numpy() - lse_b.double().cpu().numpy()))) <= LSE_ABS
    if la.size == 1:
        assert abs(la[0] - lb[0]) <= LOSS_REL * abs(lb[0])
    else:
        assert float(np.max(np.abs(la - lb))) <= LSE_ABS


CASES = [
    # (workload, reduction, normalise by label tokens)
    (W.custom(1100, 1024, 8269, 8269, ignore_frac=0.05, seed=31), "sum", True),
    (W.custom(333, 328, 1000, 1024, softcap=30.0, ignore_frac=0.1, seed=32), "none", False),
    (W.TINY, "sum", False),
]


def test_no_alloc_forward_matches_workspace_forward_on_consecutive_calls(dev):
    # Larger problem first, so the smaller ones run over a scratch array that
    # still holds the previous call's partials.
    for w, red, norm in CASES + CASES[:1]:
        hid, wt, lab, d = _inputs(w, dev)
        nlt = d["num_label_tokens"] if norm else None
        ref = _with_workspace(w, hid, wt, lab, red, nlt)
        first = _no_alloc(w, hid, wt, lab, red, nlt)
        _same(first, ref)
        # second call in a row with different labels: nothing left over leaks in
        lab2 = torch.roll(lab, 1)
        ref2 = _with_workspace(w, hid, wt, lab2, red, nlt)
        second = _no_alloc(w, hid, wt, lab2, red, nlt)
        _same(second, ref2)
    assert flce.get_error(dev) == flce.FLCE_OK


def test_no_alloc_forward_refuses_problems_beyond_its_scratch(dev):
    lib = flce.load_library()
    fake = ctypes.c_void_p(1 << 20)      # never touched: the size check comes first
    # 32768 tokens x 151936 rows needs ~156 MB of logsumexp partials > 32 MiB
    st = lib.flce_forward_noalloc(fake, fake, 0, fake, 32768, 4096, 151936, 151936, -100, 0.0,
                                  0, 0, fake, fake, None)
    assert st == 2                       # FLCE_ERR_WORKSPACE
    # the same with an FP32 head (rounded inside the GEMM, so it adds nothing to
    # the scratch; tests/test_gpu_fused_cast.py runs one whose copy would not fit)
    st = lib.flce_forward_noalloc(fake, fake, 1, fake, 32768, 4096, 151936, 151936, -100, 0.0,
                                  0, 0, fake, fake, None)
    assert st == 2
    # the binding surfaces the same refusal as an error: 20000 tokens x 65536 rows
    # need 256 x 20000 x 8 B = 41 MB of partials
    hid = torch.zeros(20000, 8, dtype=torch.bfloat16, device=dev)
    wt = torch.zeros(65536, 8, dtype=torch.bfloat16, device=dev)
    lab = torch.zeros(20000, dtype=torch.int64, device=dev)
    with pytest.raises(flce.FlceError):
        flce.forward_noalloc(hid, wt, lab)
    # and the same shape is accepted by the workspace entry point
    loss, _ = flce.forward(hid, wt, lab)
    torch.cuda.synchronize(dev)
    assert abs(float(loss) - 20000 * np.log(65536)) <= 1e-4 * 20000 * np.log(65536)
