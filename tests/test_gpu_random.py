"""Randomised GPU parity sweep: shapes (ragged in N, H, V and Vp), head dtype,
softcap, reduction, num_label_tokens, ignore_index values (including one that
is a large positive number), ignored fraction and workspace size (hence the
backward's vocabulary chunking), each against the FP64 oracle."""
import numpy as np
import pytest
import torch

from lm_head_projection_flce_b200 import flce
from lm_head_projection_flce_b200 import workloads as W
from oracle import flce_oracle as O

from gpu_common import assert_parity, gpu_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return gpu_device()


def _draw(i):
    r = np.random.default_rng(500 + i)
    n = int(r.integers(1, 700))
    h = int(8 * r.integers(1, 80))
    v = int(r.integers(1, 4000))
    vp = v + int(r.integers(0, 3)) * int(r.integers(0, 300))
    return dict(n=n, h=h, v=v, vp=vp,
                w_dtype=str(r.choice(["bf16", "f32"])),
                softcap=float(r.choice([0.0, 0.0, 5.0, 30.0])),
                reduction=str(r.choice(["sum", "sum", "mean", "none"])),
                norm=bool(r.integers(0, 2)),
                ignore_index=int(r.choice([-100, -1, 10 ** 6])),
                ignore_frac=float(r.choice([0.0, 0.1, 0.5])),
                ws_frac=float(r.choice([0.0, 0.5, 1.0])),
                w_sigma=float(r.choice([0.02, 0.1])),
                seed=600 + i)


@pytest.mark.parametrize("i", range(24))
def test_random_case(dev, i):
    c = _draw(i)
    w = W.custom(c["n"], c["h"], c["v"], c["vp"], w_dtype=c["w_dtype"], softcap=c["softcap"],
                 ignore_frac=c["ignore_frac"], w_sigma=c["w_sigma"], seed=c["seed"])
    d = W.generate(w)
    labels = d["labels"].clone()
    labels[labels == W.IGNORE_INDEX] = c["ignore_index"]
    red = c["reduction"]
    nlt = d["num_label_tokens"] if (red == "sum" and c["norm"] and d["num_label_tokens"] > 0) else None
    wdt = torch.float32 if c["w_dtype"] == "f32" else torch.bfloat16
    lo = flce.workspace_size(c["n"], c["h"], c["vp"], c["v"], wdt, minimum=True)
    hi = flce.workspace_size(c["n"], c["h"], c["vp"], c["v"], wdt)
    ws_bytes = int(lo + c["ws_frac"] * (hi - lo))
    hid, wt, lab = d["hidden"].to(dev), d["weight"].to(dev), labels.to(dev)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    grad = torch.linspace(-1, 1, c["n"]) if red == "none" else torch.tensor([1.25])
    loss, lse = flce.forward(hid, wt, lab, ignore_index=c["ignore_index"], softcap=c["softcap"],
                             unpadded_vocab=c["v"], reduction=red, num_label_tokens=nlt, workspace=ws)
    dh, dw = flce.backward(hid, wt, lab, lse, grad.to(dev), ignore_index=c["ignore_index"],
                           softcap=c["softcap"], unpadded_vocab=c["v"], reduction=red,
                           num_label_tokens=nlt, workspace=ws)
    torch.cuda.synchronize(dev)
    got = {"loss": loss.double().cpu().numpy(), "lse": lse.double().cpu().numpy(),
           "dh": dh.double().cpu().numpy(), "dw": dw.double().cpu().numpy(),
           "status": flce.get_error(dev)}
    hw = d["weight"].numpy() if wdt == torch.float32 else d["weight"].double().numpy()
    kw = dict(ignore_index=c["ignore_index"], softcap=c["softcap"], unpadded_vocab=c["v"],
              reduction=red, num_label_tokens=nlt)
    fwd = O.forward(d["hidden"].double().numpy(), hw, labels.numpy(), **kw)
    rdh, rdw = O.backward(d["hidden"].double().numpy(), hw, labels.numpy(),
                          grad_loss=grad.double().numpy(), **kw)
    assert_parity(got, {"loss": np.asarray(fwd.loss), "lse": fwd.lse, "dh": rdh, "dw": rdw}), c
    if wdt == torch.float32:
        # The head rounded inside the GEMMs instead: a workspace smaller by exactly the
        # copy keeps the same vocabulary chunking, so every result matches bit for bit.
        copy = -(-c["v"] * c["h"] * 2 // 1024) * 1024
        ws_f = torch.empty(max(ws_bytes - copy, 16), dtype=torch.uint8, device=dev)
        kw_f = dict(ignore_index=c["ignore_index"], softcap=c["softcap"], unpadded_vocab=c["v"],
                    reduction=red, num_label_tokens=nlt, workspace=ws_f, fused_head_cast=True)
        loss_f, lse_f = flce.forward(hid, wt, lab, **kw_f)
        dh_f, dw_f = flce.backward(hid, wt, lab, lse_f, grad.to(dev), **kw_f)
        torch.cuda.synchronize(dev)
        assert flce.get_error(dev) == flce.FLCE_OK
        for x, y in ((loss, loss_f), (lse, lse_f), (dh, dh_f), (dw, dw_f)):
            assert torch.equal(x, y), c


def _draw_ce(i):
    r = np.random.default_rng(900 + i)
    n = int(r.choice([int(r.integers(1, 64)), int(r.integers(64, 600)), int(r.integers(600, 1500))]))
    v = int(r.choice([int(r.integers(1, 3000)), int(r.integers(30000, 140000))]))
    v = max(1, min(v, 40_000_000 // n))        # keep the FP64 oracle to a few seconds
    return dict(n=n, v=v, pad=int(r.choice([0, 0, 1, 3, 17])),
                dtype=str(r.choice(["bf16", "f32"])),
                scale=float(r.choice([1.0, 3.0, 8.0])),
                reduction=str(r.choice(["sum", "sum", "mean", "none"])),
                norm=bool(r.integers(0, 2)), mask=bool(r.integers(0, 2)),
                ignore_frac=float(r.choice([0.0, 0.1, 0.5])), seed=950 + i)


@pytest.mark.parametrize("i", range(16))
def test_random_ce_case(dev, i):
    """Cross entropy on given logits: row counts below and above the resident
    CTA slots (segmented and whole-row launches), long and short rows, row
    strides, masks, both dtypes, every reduction, against the FP64 oracle."""
    c = _draw_ce(i)
    g = torch.Generator().manual_seed(c["seed"])
    n, v, ld = c["n"], c["v"], c["v"] + c["pad"]
    dtype = torch.float32 if c["dtype"] == "f32" else torch.bfloat16
    full = (torch.randn(n, ld, generator=g) * c["scale"]).to(dtype)
    labels = torch.randint(0, v, (n,), generator=g)
    k = int(c["ignore_frac"] * n + 0.5)
    if k:
        labels[torch.randperm(n, generator=g)[:k]] = W.IGNORE_INDEX
    mask = (torch.rand(n, generator=g) > 0.2).to(torch.uint8) if c["mask"] else None
    red = c["reduction"]
    valid = (labels != W.IGNORE_INDEX) & (mask.bool() if mask is not None else True)
    nvalid = int(valid.sum())
    nlt = nvalid if (red == "sum" and c["norm"] and nvalid > 0) else None
    z = full.to(dev)[:, :v]
    m = mask.to(dev) if mask is not None else None
    grad = torch.linspace(-1, 1, n) if red == "none" else torch.tensor([0.75])
    loss, lse = flce.ce_forward(z, labels.to(dev), mask=m, reduction=red, num_label_tokens=nlt)
    dz = flce.ce_backward(z, labels.to(dev), lse, grad.to(dev), mask=m, reduction=red,
                          num_label_tokens=nlt)
    torch.cuda.synchronize(dev)
    zf = full[:, :v].double().numpy()
    mk = mask.numpy() if mask is not None else None
    ref = O.ce_forward(zf, labels.numpy(), mask=mk, reduction=red, num_label_tokens=nlt)
    rdz = O.ce_backward(zf, labels.numpy(), mask=mk, reduction=red, num_label_tokens=nlt,
                        grad_loss=grad.double().numpy())
    got = {"loss": loss.double().cpu().numpy(), "lse": lse.double().cpu().numpy(),
           "dh": dz.double().cpu().numpy(), "dw": np.zeros(1), "status": flce.get_error(dev)}
    assert_parity(got, {"loss": np.asarray(ref.loss), "lse": ref.lse, "dh": rdz,
                        "dw": np.zeros(1)}), c
