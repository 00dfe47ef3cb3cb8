"""GPU tests of the in-kernel FP32 -> BF16 head rounding (FLCE_FUSED_HEAD_CAST).

The inkling2 page (Inkling2FusedLinearCrossEntropy class docstring) rounds an
FP32 head to BF16 before use, as FSDP's cast does.  With the flag, the GEMMs
that read the head load its FP32 rows and round them in shared memory instead
of reading a BF16 copy from the workspace.  The rounding is the copy's
(nearest even) and the MMAs run in the same order, so every output must equal
the copy path's bit for bit; the fused results are also held to the oracle.
"""
import pytest
import torch

from lm_head_projection_flce_b200 import flce
from lm_head_projection_flce_b200 import workloads as W

from gpu_common import assert_parity, gpu_device, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return gpu_device()


def _step(hid, wt, lab, w, dev, *, fused, ws_bytes=None, reduction=None, grad=None):
    red = reduction or w.reduction
    ws = None
    if ws_bytes is not None:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        ws.fill_(0xFF)  # stale bytes must not matter
    kw = dict(softcap=w.softcap, unpadded_vocab=w.vocab, reduction=red, workspace=ws,
              fused_head_cast=fused)
    loss, lse = flce.forward(hid, wt, lab, **kw)
    if grad is None:
        grad = torch.ones(1) if red != "none" else torch.linspace(-1.0, 2.0, w.n_tokens)
    dh, dw = flce.backward(hid, wt, lab, lse, grad.to(dev), **kw)
    torch.cuda.synchronize(dev)
    return loss, lse, dh, dw


# Ragged edges in every dimension: H = 328 and 520 end in a partial k-block
# (the second 32-wide FP32 box of the last one lies wholly past H), V = 1000 /
# 5000 / 8269 end in partial head tiles, and the minimum workspace streams the
# vocabulary in 256-wide chunks (the dhidden GEMM's MN-major FP32 boxes then
# start every 256 head rows).
CASES = {
    "ragged_softcap": (W.custom(333, 328, 1000, 1024, w_dtype="f32", softcap=30.0,
                                ignore_frac=0.1, seed=11), None),
    "many_chunks": (W.custom(700, 520, 5000, 5120, w_dtype="f32", softcap=30.0,
                             ignore_frac=0.1, w_sigma=0.05, seed=13), "min"),
    "multi_tile": (W.custom(1100, 1024, 8269, 8269, w_dtype="f32", ignore_frac=0.05, seed=12),
                   None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fused_head_cast_equals_the_copy_path(dev, name):
    w, size = CASES[name]
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    args = (w.n_tokens, w.hidden, w.padded_vocab, w.vocab, torch.float32)
    copy_ws = flce.workspace_size(*args, minimum=size == "min")
    fused_ws = flce.workspace_size(*args, minimum=size == "min", fused_head_cast=True)
    # the fused workspace lacks exactly the V x H BF16 copy (rounded up to 1 KiB)
    copy_bytes = -(-w.vocab * w.hidden * 2 // 1024) * 1024
    assert copy_ws - fused_ws == copy_bytes
    a = _step(hid, wt, lab, w, dev, fused=False, ws_bytes=copy_ws)
    b = _step(hid, wt, lab, w, dev, fused=True, ws_bytes=fused_ws)
    assert flce.get_error(dev) == flce.FLCE_OK
    for x, y, what in zip(a, b, ("loss", "lse", "dhidden", "dW")):
        assert torch.equal(x, y), what
    got = {"loss": b[0].double().cpu().numpy(), "lse": b[1].double().cpu().numpy(),
           "dh": b[2].double().cpu().numpy(), "dw": b[3].double().cpu().numpy(),
           "status": flce.FLCE_OK}
    assert_parity(got, run_oracle(d, w))


def test_fused_head_cast_reductions_and_bf16_head(dev):
    """Per-token losses and gradients ('none'), and a BF16 head, where the flag
    changes nothing."""
    w = W.custom(300, 264, 3000, 3072, w_dtype="f32", softcap=5.0, ignore_frac=0.2, seed=31)
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    a = _step(hid, wt, lab, w, dev, fused=False, reduction="none")
    b = _step(hid, wt, lab, w, dev, fused=True, reduction="none")
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    wb = wt.to(torch.bfloat16)
    a = _step(hid, wb, lab, w, dev, fused=False)
    b = _step(hid, wb, lab, w, dev, fused=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_fused_head_cast_autograd(dev):
    w = W.custom(257, 256, 2000, 2048, w_dtype="f32", softcap=30.0, ignore_frac=0.1, seed=32)
    d = W.generate(w)
    grads = []
    for fused in (False, True):
        h = d["hidden"].to(dev).requires_grad_(True)
        wt = d["weight"].to(dev).requires_grad_(True)
        loss = flce.fused_linear_cross_entropy(h, wt, d["labels"].to(dev), softcap=w.softcap,
                                               unpadded_vocab=w.vocab, fused_head_cast=fused)
        loss.backward()
        grads.append((loss.detach(), h.grad, wt.grad))
    torch.cuda.synchronize(dev)
    for x, y in zip(*grads):
        assert torch.equal(x, y)


def test_noalloc_forward_takes_fp32_heads_of_any_size(dev):
    """The forward without allocation rounds an FP32 head in the GEMM, so a
    head whose BF16 copy alone (20011 x 1024 x 2 = 41 MB) exceeds its 32 MiB
    scratch array runs, and equals flce_forward."""
    w = W.custom(600, 1024, 20011, 20480, w_dtype="f32", softcap=30.0, ignore_frac=0.05,
                 seed=33)
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    loss_a, lse_a = flce.forward(hid, wt, lab, softcap=w.softcap, unpadded_vocab=w.vocab)
    loss_b, lse_b = flce.forward_noalloc(hid, wt, lab, softcap=w.softcap, unpadded_vocab=w.vocab)
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_OK
    assert torch.equal(loss_a, loss_b) and torch.equal(lse_a, lse_b)


def test_fused_head_cast_full_size_fp32_head(dev):
    """The FP32-head workload at full size (N 8192, H 5376, V 256000 of 262144,
    softcap 30): the fused path equals the copy path bit for bit."""
    w = W.WORKLOADS["n8192_h5376_v256000_vp262144_softcap30_f32head"]
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    del d
    a = _step(hid, wt, lab, w, dev, fused=False)
    b = _step(hid, wt, lab, w, dev, fused=True)
    assert flce.get_error(dev) == flce.FLCE_OK
    for x, y, what in zip(a, b, ("loss", "lse", "dhidden", "dW")):
        assert torch.equal(x, y), what
