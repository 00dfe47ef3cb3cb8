"""GPU parity at the five workloads' full sizes, in the launch configuration the
benchmark uses (default workspace, so the same vocabulary chunking).

The oracle cannot afford a full FP64 backward at these sizes, so on every
workload:
  * the FP64 forward runs in full: every token's lse and token loss, and the
    total loss from them, are compared with the GPU's (the oracle computes the
    logits 512 token rows at a time; about four minutes of FP64 BLAS for all
    five workloads on a 16-core host);
  * dhidden is compared on 256 sampled token rows (a dhidden row needs only
    its own logits row), ignored tokens and both ends included;
  * dW is compared on 256 sampled head rows (a head row's gradient needs every
    token's logsumexp, which the full forward above provides), including the
    labels' rows, rows 0 and V - 1 and, with a padded head, rows >= V;
  * and properties that hold at any size: rows >= V exactly 0; doubling the
    upstream gradient doubles dW and dhidden bit for bit; without a softcap
    the head rows' gradients sum to ~0.
"""
import numpy as np
import pytest
import torch

from lm_head_projection_flce_b200 import flce
from lm_head_projection_flce_b200 import workloads as W
from oracle import flce_oracle as O

from gpu_common import GRAD_REL, LOSS_REL, LSE_ABS, gpu_device

pytestmark = pytest.mark.gpu

CONFIGS = [W.TINY, W.LLAMA_HEAD, W.SOFTCAP_F32_HEAD, W.LONG_SEQ, W.LARGE_HEAD]


@pytest.fixture(scope="module")
def dev():
    return gpu_device()


def _oracle_head(d, w):
    """The oracle's FP64 compute head (rows < V), prepared once per workload."""
    wt = d["weight"]
    raw = wt.numpy() if wt.dtype == torch.float32 else wt.to(torch.float64).numpy()
    head = O.compute_head(raw, w.vocab)
    return np.ascontiguousarray(head)


def _sample_rows(rng, labels, n, k):
    ign = np.nonzero(labels == W.IGNORE_INDEX)[0]
    pick = set(rng.choice(n, size=min(k, n), replace=False).tolist())
    pick.update(ign[:4].tolist())
    pick.update([0, n - 1])
    return np.array(sorted(pick), dtype=np.int64)


@pytest.mark.parametrize("w", CONFIGS, ids=[c.name for c in CONFIGS])
def test_full_size_parity(dev, w):
    d = W.generate(w)
    n, h, vp, v = w.n_tokens, w.hidden, w.padded_vocab, w.vocab
    nlt = d["num_label_tokens"] if w.normalize_by_label_tokens else None
    hid, wt, lab = d["hidden"].to(dev), d["weight"].to(dev), d["labels"].to(dev)
    kw = dict(softcap=w.softcap, unpadded_vocab=v, reduction=w.reduction, num_label_tokens=nlt)

    loss, lse = flce.forward(hid, wt, lab, **kw)
    tok, _ = flce.forward(hid, wt, lab, softcap=w.softcap, unpadded_vocab=v, reduction="none")
    dh, dw = flce.backward(hid, wt, lab, lse, torch.ones(1, device=dev), **kw)
    dh2, dw2 = flce.backward(hid, wt, lab, lse, torch.full((1,), 2.0, device=dev), **kw)
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_OK

    # ---- properties at any size
    assert torch.equal(dh2, 2 * dh) and torch.equal(dw2, 2 * dw)
    del dh2, dw2
    if vp > v:
        assert torch.all(dw[v:] == 0)
    assert torch.isfinite(dw).all() and torch.isfinite(dh).all()
    tok_sum = float(tok.double().sum())
    want_total = tok_sum / nlt if nlt else tok_sum
    assert abs(float(loss) - want_total) <= 1e-5 * abs(want_total)
    if w.softcap == 0:
        # sum_v dz[n, v] = 0 for every token, so sum_v dW[v, :] = 0 up to the BF16
        # rounding of G (<= 2^-9 relative, sum_v |dz[n, v]| <= 2 s_n) and of dW itself.
        scale = np.where(d["labels"].numpy() != W.IGNORE_INDEX,
                         1.0 / nlt if nlt else 1.0, 0.0)
        sh = (torch.from_numpy(scale)[:, None] * d["hidden"].double().abs()).sum(dim=0).max().item()
        col = dw[:v].double().sum(dim=0).abs().max().item()
        bound = 2.0 ** -7 * sh + 2.0 ** -8 * dw[:v].double().abs().sum(dim=0).max().item()
        assert col <= bound, (col, bound)

    # ---- sampled rows against the oracle
    hidden = d["hidden"].to(torch.float64).numpy()
    labels = d["labels"].numpy()
    head = _oracle_head(d, w)
    rng = np.random.default_rng(w.seed)
    o_kw = dict(ignore_index=W.IGNORE_INDEX, softcap=w.softcap, unpadded_vocab=v)
    lse_g = lse.double().cpu().numpy()
    tok_g = tok.double().cpu().numpy()

    # ---- the oracle's full forward: every token's lse and loss, and the total
    lse_all = np.empty(n)
    tok_all = np.empty(n)
    step = 512
    for s in range(0, n, step):
        idx = np.arange(s, min(n, s + step))
        lse_all[idx], tok_all[idx] = O.forward_rows(hidden, head, labels, idx, **o_kw)
    assert float(np.max(np.abs(lse_g - lse_all))) <= LSE_ABS
    assert float(np.max(np.abs(tok_g - tok_all))) <= LSE_ABS
    ref_total = O.reduce_losses(tok_all, labels != W.IGNORE_INDEX, w.reduction, nlt)
    assert abs(float(loss) - ref_total) <= LOSS_REL * abs(ref_total)

    # ---- sampled dhidden rows
    dh_rows = _sample_rows(rng, labels, n, 256)
    dh_r = O.dh_rows(hidden, head, labels, dh_rows, reduction=w.reduction,
                     num_label_tokens=nlt, **o_kw)
    dh_g = dh[torch.from_numpy(dh_rows).to(dev)].double().cpu().numpy()
    assert float(np.max(np.abs(dh_g - dh_r))) <= GRAD_REL * float(np.max(np.abs(dh_r)))

    # ---- sampled dW rows (the labels' rows included, and padded rows if any)
    live = labels[labels != W.IGNORE_INDEX]
    pad = [v, vp - 1] if vp > v else []
    vrows = np.unique(np.concatenate([rng.choice(v, size=min(224, v), replace=False),
                                      live[:28], [0, v - 1], pad])).astype(np.int64)
    dw_r = O.dw_rows(hidden, head, labels, vrows, lse_all, reduction=w.reduction,
                     num_label_tokens=nlt, **o_kw)
    dw_g = dw[torch.from_numpy(vrows).to(dev)].double().cpu().numpy()
    assert float(np.max(np.abs(dw_g - dw_r))) <= GRAD_REL * float(np.max(np.abs(dw_r)))
