"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the FP64 oracle on the same seeded inputs, and compare them within the
stated tolerances:

  per-token |lse_gpu - lse_ref|            <= 2e-3
  |loss_gpu - loss_ref| / |loss_ref|       <= 1e-4
  max|dh_gpu - dh_ref|, max|dW_gpu - dW_ref| <= 1e-2 * max|ref|
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from lm_head_projection_flce_b200 import build as B
from lm_head_projection_flce_b200 import flce
from lm_head_projection_flce_b200 import workloads as W
from oracle import flce_oracle as O

LSE_ABS = 2e-3
LOSS_REL = 1e-4
GRAD_REL = 1e-2


def gpu_device() -> torch.device:
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    flce.load_library()  # raises loudly if the library is missing
    return torch.device("cuda", 0)


def to_oracle(d: dict):
    hidden = d["hidden"].double().numpy()
    w = d["weight"]
    weight = w.numpy() if w.dtype == torch.float32 else w.double().numpy()
    return hidden, weight, d["labels"].numpy()


def run_gpu(d: dict, w: W.Workload, dev, *, reduction=None, grad=None, ws_bytes=None,
            num_label_tokens=None):
    red = reduction or w.reduction
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    ws = None
    if ws_bytes is not None:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    loss, lse = flce.forward(hid, wt, lab, softcap=w.softcap, unpadded_vocab=w.vocab,
                             reduction=red, num_label_tokens=num_label_tokens, workspace=ws)
    if grad is None:
        grad = torch.ones(1) if red != "none" else torch.ones(w.n_tokens)
    dh, dw = flce.backward(hid, wt, lab, lse, grad.to(dev), softcap=w.softcap,
                           unpadded_vocab=w.vocab, reduction=red,
                           num_label_tokens=num_label_tokens, workspace=ws)
    torch.cuda.synchronize(dev)
    status = flce.get_error(dev)
    return {"loss": loss.double().cpu().numpy(), "lse": lse.double().cpu().numpy(),
            "dh": dh.double().cpu().numpy(), "dw": dw.double().cpu().numpy(),
            "status": status}


def run_oracle(d: dict, w: W.Workload, *, reduction=None, grad=None, num_label_tokens=None):
    red = reduction or w.reduction
    h, wt, lab = to_oracle(d)
    g = 1.0 if grad is None else grad.double().numpy()
    kw = dict(ignore_index=W.IGNORE_INDEX, softcap=w.softcap, unpadded_vocab=w.vocab,
              reduction=red, num_label_tokens=num_label_tokens)
    fwd = O.forward(h, wt, lab, **kw)
    dh, dw = O.backward(h, wt, lab, grad_loss=g, **kw)
    return {"loss": np.asarray(fwd.loss), "lse": fwd.lse, "dh": dh, "dw": dw,
            "token_loss": fwd.token_loss}


def max_rel(got, ref) -> float:
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return err / scale if scale > 0 else err


def assert_parity(got: dict, ref: dict, *, check_grads=True):
    assert got["status"] == flce.FLCE_OK, flce.STATUS[got["status"]]
    if ref["lse"].size:
        lse_err = float(np.max(np.abs(got["lse"] - ref["lse"])))
        assert lse_err <= LSE_ABS, f"lse abs err {lse_err}"
    loss_g, loss_r = np.asarray(got["loss"]).reshape(-1), np.asarray(ref["loss"]).reshape(-1)
    if loss_r.size == 1:
        if np.isnan(loss_r[0]):
            assert np.isnan(loss_g[0])
        elif loss_r[0] == 0.0:
            assert loss_g[0] == 0.0
        else:
            rel = abs(loss_g[0] - loss_r[0]) / abs(loss_r[0])
            assert rel <= LOSS_REL, f"loss rel err {rel} ({loss_g[0]} vs {loss_r[0]})"
    else:
        err = float(np.max(np.abs(loss_g - loss_r))) if loss_r.size else 0.0
        assert err <= LSE_ABS, f"token loss abs err {err}"
    if check_grads:
        e_dh = max_rel(got["dh"], ref["dh"])
        e_dw = max_rel(got["dw"], ref["dw"])
        assert e_dh <= GRAD_REL, f"dh rel err {e_dh}"
        assert e_dw <= GRAD_REL, f"dW rel err {e_dw}"
