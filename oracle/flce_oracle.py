"""FP64 CPU oracle for the fused LM-head projection + cross-entropy.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, the package smoke check and the benchmark's CPU-baseline and
reference (``--impl reference``) legs call it.  It shares no code, constant or helper with the CUDA path; the two
meet only in the seeded input generators, which hold none of the arithmetic.

What is computed, and where the pages fix it:

* Projection of BF16 hidden states against the BF16 head rows with (here:
  better than) FP32 accumulation; softcap and cross entropy in floating point
  wider than BF16; rows past ``unpadded_vocab`` never enter the softmax; an
  FP32 head is rounded to BF16 first ("nemo_automodel.components.models.
  inkling2.loss", Inkling2FusedLinearCrossEntropy, class docstring).
* ``ignore_index`` positions contribute zero loss and zero gradient
  ("nemo_automodel.components.loss.chunked_ce", _ChunkedCrossEntropySum.forward,
  parameter ``labels``).
* ``reduction='sum'`` by default, and ``num_label_tokens`` divides a
  sum-reduced loss ("nemo_automodel.components.loss.linear_ce",
  FusedLinearCrossEntropy constructor and ``forward`` parameter
  ``num_label_tokens``); other reductions follow PyTorch ("Compute fused
  linear cross entropy matching PyTorch behavior", same section).
* The backward returns gradients w.r.t. the hidden states and the (padded)
  head; the softmax is recomputed rather than stored
  ("nemo_automodel.components.loss.chunked_ce", _ChunkedCrossEntropySum.backward).

Readings taken where the pages are silent:
softcap is ``c*tanh(z/c)`` with ``c = 0`` meaning off; logits are not rounded
to BF16 before the softcap; a label outside ``[0, unpadded_vocab)`` that is not
``ignore_index`` is invalid (this oracle raises); labels are not shifted;
``mean`` divides by the number of non-ignored labels (NaN when there are none,
as PyTorch gives); ``num_label_tokens`` is only valid with ``sum``; head rows
``>= unpadded_vocab`` receive an exactly-zero gradient.

Arrays: ``hidden`` is ``[N, H]`` float64 holding BF16 values; ``weight`` is
``[Vp, H]`` and is either float64 holding BF16 values or float32 (an FP32 head,
rounded to BF16 here); ``labels`` is int64 ``[N]``.  All arithmetic is FP64.
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = [
    "bf16_round", "compute_head", "project", "apply_softcap", "logsumexp_rows",
    "token_losses", "reduce_losses", "token_scales", "logit_grad",
    "ForwardResult", "forward", "backward", "forward_rows", "dh_rows", "dw_rows",
    "check_labels", "ce_labels", "ce_forward", "ce_backward",
]


# --------------------------------------------------------------------------
# Inputs
# --------------------------------------------------------------------------

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round FP32 values to BF16 with round-to-nearest-even; return them as FP64.

    BF16 keeps the upper 16 bits of the FP32 encoding.  Round-to-nearest-even
    on the 16 dropped bits: add 0x7FFF plus the lowest kept bit, then truncate.
    NaNs are kept as (quiet) NaNs.  This is the FP32->BF16 cast the inkling2 page
    names for an FP32 head ("the cast FSDP applies", i.e. ``tensor.to(bfloat16)``).
    """
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    # For every non-NaN encoding u <= 0xFF800000, so u + 0x7FFF + 1 stays below 2**32.
    keep_lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = ((u + np.uint32(0x7FFF) + keep_lsb) >> np.uint32(16)) << np.uint32(16)
    nan = np.isnan(f)
    if nan.any():
        r[nan] = (u[nan] & np.uint32(0xFFFF0000)) | np.uint32(0x00400000)
    return r.view(np.float32).astype(np.float64)


def compute_head(weight: np.ndarray, unpadded_vocab: int) -> np.ndarray:
    """The BF16 compute head: the first ``unpadded_vocab`` rows, FP32 rounded to BF16.

    inkling2 page, ``materialize_lm_weight`` return value: a BF16 tensor of shape
    ``[unpadded_vocab_size, hidden]``.
    """
    rows = weight[:unpadded_vocab]
    if rows.dtype == np.float32:
        out = np.empty(rows.shape, dtype=np.float64)
        for s in range(0, rows.shape[0], 8192):      # elementwise; blocks only bound memory
            out[s:s + 8192] = bf16_round(rows[s:s + 8192])
        return out
    return np.asarray(rows, dtype=np.float64)


def check_labels(labels: np.ndarray, unpadded_vocab: int, ignore_index: int) -> np.ndarray:
    """Mask of labels that take part in the loss; raises on out-of-range labels."""
    labels = np.asarray(labels, dtype=np.int64)
    valid = labels != ignore_index
    bad = valid & ((labels < 0) | (labels >= unpadded_vocab))
    if bad.any():
        raise ValueError(f"{int(bad.sum())} labels outside [0, {unpadded_vocab}) "
                         f"that are not ignore_index={ignore_index}")
    return valid


# --------------------------------------------------------------------------
# Forward steps
# --------------------------------------------------------------------------

def project(hidden: np.ndarray, head: np.ndarray) -> np.ndarray:
    """Logits ``z[n, v] = sum_h hidden[n, h] * head[v, h]`` in FP64 (a library matmul)."""
    return np.asarray(hidden, dtype=np.float64) @ np.asarray(head, dtype=np.float64).T


def apply_softcap(z: np.ndarray, softcap: float) -> np.ndarray:
    """``c * tanh(z / c)`` for ``c > 0``; the identity for ``c == 0``."""
    if softcap > 0:
        return softcap * np.tanh(z / softcap)
    return z


def logsumexp_rows(zc: np.ndarray) -> np.ndarray:
    """``log(sum_v exp(zc[n, v]))`` per row, shifted by the row max for range."""
    m = zc.max(axis=1, keepdims=True)
    return (m + np.log(np.exp(zc - m).sum(axis=1, keepdims=True)))[:, 0]


def token_losses(lse: np.ndarray, zc: np.ndarray, labels: np.ndarray,
                 valid: np.ndarray) -> np.ndarray:
    """Per-token NLL ``lse[n] - zc[n, y_n]`` for valid labels, exactly 0 otherwise."""
    out = np.zeros(lse.shape[0], dtype=np.float64)
    idx = np.nonzero(valid)[0]
    out[idx] = lse[idx] - zc[idx, labels[idx]]
    return out


def reduce_losses(tok: np.ndarray, valid: np.ndarray, reduction: str,
                  num_label_tokens: int | None):
    """Reduce per-token losses: 'sum' (optionally / num_label_tokens), 'mean', 'none'."""
    if num_label_tokens is not None and reduction != "sum":
        raise ValueError("num_label_tokens normalises a sum-reduced loss only")
    if reduction == "sum":
        total = float(np.sum(tok))
        if num_label_tokens is not None:
            total /= float(num_label_tokens)
        return total
    if reduction == "mean":
        count = int(valid.sum())
        return float(np.sum(tok)) / count if count > 0 else float("nan")
    if reduction == "none":
        return tok.copy()
    raise ValueError(f"unknown reduction {reduction!r}")


@dataclasses.dataclass
class ForwardResult:
    loss: object              # float for sum/mean, float64 [N] for none
    lse: np.ndarray           # float64 [N]: logsumexp of the capped logits
    token_loss: np.ndarray    # float64 [N]: 0 at ignored positions


def forward(hidden, weight, labels, *, ignore_index: int = -100,
            softcap: float = 0.0, unpadded_vocab: int | None = None,
            reduction: str = "sum", num_label_tokens: int | None = None) -> ForwardResult:
    """Loss of the fused projection + cross entropy, in the order the pages state it."""
    labels = np.asarray(labels, dtype=np.int64)
    v = weight.shape[0] if unpadded_vocab is None else int(unpadded_vocab)
    valid = check_labels(labels, v, ignore_index)
    head = compute_head(weight, v)
    z = project(hidden, head)
    zc = apply_softcap(z, softcap)
    lse = logsumexp_rows(zc) if zc.shape[0] else np.zeros(0)
    tok = token_losses(lse, zc, labels, valid)
    return ForwardResult(reduce_losses(tok, valid, reduction, num_label_tokens), lse, tok)


# --------------------------------------------------------------------------
# Backward
# --------------------------------------------------------------------------

def token_scales(valid: np.ndarray, reduction: str, num_label_tokens: int | None,
                 grad_loss) -> np.ndarray:
    """d(loss)/d(token loss n): the upstream gradient through the reduction.

    Exactly 0 at ignored positions, which contribute zero loss and zero
    gradient (chunked_ce page, _ChunkedCrossEntropySum.forward, ``labels``);
    with ``mean`` and no valid label there is nothing to scale, so all are 0.
    """
    if reduction == "none":
        g = np.asarray(grad_loss, dtype=np.float64).reshape(-1)
        return np.where(valid, g, 0.0)
    g = float(np.asarray(grad_loss, dtype=np.float64).reshape(-1)[0])
    if reduction == "sum":
        if num_label_tokens is not None:
            g /= float(num_label_tokens)
        return np.where(valid, g, 0.0)
    if reduction == "mean":
        count = int(valid.sum())
        return np.where(valid, g / count if count else 0.0, 0.0)
    raise ValueError(f"unknown reduction {reduction!r}")


def logit_grad(z: np.ndarray, lse: np.ndarray, labels: np.ndarray, valid: np.ndarray,
               scale: np.ndarray, softcap: float) -> np.ndarray:
    """``dL/dz[n, v] = s_n * (softmax(zc)[n, v] - [v == y_n]) * dzc/dz``.

    ``dzc/dz = 1 - tanh(z/c)^2`` under a softcap, 1 without one.  Ignored rows
    are exactly 0 (their scale is 0).
    """
    zc = apply_softcap(z, softcap)
    p = np.exp(zc - lse[:, None])
    idx = np.nonzero(valid)[0]
    p[idx, labels[idx]] -= 1.0
    if softcap > 0:
        t = np.tanh(z / softcap)
        p *= (1.0 - t * t)
    return p * scale[:, None]


def backward(hidden, weight, labels, *, ignore_index: int = -100,
             softcap: float = 0.0, unpadded_vocab: int | None = None,
             reduction: str = "sum", num_label_tokens: int | None = None,
             grad_loss=1.0):
    """Gradients ``(dhidden [N,H], dweight [Vp,H])`` in FP64; rows >= V of dweight are 0."""
    labels = np.asarray(labels, dtype=np.int64)
    vp = weight.shape[0]
    v = vp if unpadded_vocab is None else int(unpadded_vocab)
    valid = check_labels(labels, v, ignore_index)
    head = compute_head(weight, v)
    z = project(hidden, head)
    lse = logsumexp_rows(apply_softcap(z, softcap)) if z.shape[0] else np.zeros(0)
    s = token_scales(valid, reduction, num_label_tokens, grad_loss)
    dz = logit_grad(z, lse, labels, valid, s, softcap)
    dh = dz @ head
    dw = np.zeros((vp, head.shape[1]), dtype=np.float64)
    dw[:v] = dz.T @ np.asarray(hidden, dtype=np.float64)
    return dh, dw


# --------------------------------------------------------------------------
# Row-sampled forms for large problems (same arithmetic, fewer rows)
# --------------------------------------------------------------------------

def forward_rows(hidden, weight, labels, rows, *, ignore_index=-100, softcap=0.0,
                 unpadded_vocab=None):
    """``(lse, token_loss)`` for the token rows ``rows`` only (each row is independent)."""
    rows = np.asarray(rows, dtype=np.int64)
    v = weight.shape[0] if unpadded_vocab is None else int(unpadded_vocab)
    lab = np.asarray(labels, dtype=np.int64)[rows]
    valid = check_labels(lab, v, ignore_index)
    head = compute_head(weight, v)
    zc = apply_softcap(project(np.asarray(hidden)[rows], head), softcap)
    lse = logsumexp_rows(zc)
    return lse, token_losses(lse, zc, lab, valid)


def dh_rows(hidden, weight, labels, rows, *, ignore_index=-100, softcap=0.0,
            unpadded_vocab=None, reduction="sum", num_label_tokens=None, grad_loss=1.0):
    """Rows ``rows`` of dhidden.  A row of dhidden needs only its own logits row.

    For ``mean`` the valid count is taken over all ``labels``; for ``none``
    ``grad_loss`` is the full ``[N]`` upstream gradient.
    """
    rows = np.asarray(rows, dtype=np.int64)
    labels = np.asarray(labels, dtype=np.int64)
    v = weight.shape[0] if unpadded_vocab is None else int(unpadded_vocab)
    valid_all = check_labels(labels, v, ignore_index)
    s = token_scales(valid_all, reduction, num_label_tokens, grad_loss)[rows]
    head = compute_head(weight, v)
    z = project(np.asarray(hidden)[rows], head)
    lse = logsumexp_rows(apply_softcap(z, softcap))
    dz = logit_grad(z, lse, labels[rows], valid_all[rows], s, softcap)
    return dz @ head


def dw_rows(hidden, weight, labels, vrows, lse_all, *, ignore_index=-100, softcap=0.0,
            unpadded_vocab=None, reduction="sum", num_label_tokens=None, grad_loss=1.0):
    """Rows ``vrows`` of dweight, given the oracle's ``lse`` for every token.

    A head row's gradient sums over all tokens, so it needs every token's
    logsumexp; ``lse_all`` must come from :func:`forward` / :func:`forward_rows`.
    Rows ``>= unpadded_vocab`` are 0.
    """
    vrows = np.asarray(vrows, dtype=np.int64)
    labels = np.asarray(labels, dtype=np.int64)
    vp = weight.shape[0]
    v = vp if unpadded_vocab is None else int(unpadded_vocab)
    valid = check_labels(labels, v, ignore_index)
    s = token_scales(valid, reduction, num_label_tokens, grad_loss)
    out = np.zeros((vrows.shape[0], weight.shape[1]), dtype=np.float64)
    live = np.nonzero(vrows < v)[0]
    if live.size == 0:
        return out
    head_rows = compute_head(weight[vrows[live]], len(live))
    z = project(hidden, head_rows)                  # [N, |live|]
    zc = apply_softcap(z, softcap)
    p = np.exp(zc - np.asarray(lse_all)[:, None])
    onehot = (labels[:, None] == vrows[live][None, :]) & valid[:, None]
    g = p - onehot
    if softcap > 0:
        t = np.tanh(z / softcap)
        g *= (1.0 - t * t)
    g *= s[:, None]
    out[live] = g.T @ np.asarray(hidden, dtype=np.float64)
    return out


# --------------------------------------------------------------------------
# Cross entropy on given logits ("nemo_automodel.components.loss.chunked_ce":
# ChunkedCrossEntropy.forward, _ChunkedCrossEntropySum.forward/backward)
# --------------------------------------------------------------------------

def ce_labels(labels, mask, ignore_index: int = -100) -> np.ndarray:
    """Labels with every position whose mask is zero replaced by ``ignore_index``
    (ChunkedCrossEntropy.forward, parameter ``mask``: nonzero positions
    contribute, zero positions are ignored)."""
    labels = np.array(labels, dtype=np.int64, copy=True)
    if mask is not None:
        labels[np.asarray(mask) == 0] = ignore_index
    return labels


def ce_forward(logits, labels, *, mask=None, ignore_index: int = -100,
               reduction: str = "sum", num_label_tokens: int | None = None) -> ForwardResult:
    """Cross entropy of given logits ``[N, V]`` (any float dtype, upcast to FP64)."""
    z = np.asarray(logits, dtype=np.float64)
    lab = ce_labels(labels, mask, ignore_index)
    valid = check_labels(lab, z.shape[1], ignore_index)
    lse = logsumexp_rows(z) if z.shape[0] else np.zeros(0)
    tok = token_losses(lse, z, lab, valid)
    return ForwardResult(reduce_losses(tok, valid, reduction, num_label_tokens), lse, tok)


def ce_backward(logits, labels, *, mask=None, ignore_index: int = -100,
                reduction: str = "sum", num_label_tokens: int | None = None,
                grad_loss=1.0) -> np.ndarray:
    """Gradient of that loss w.r.t. the logits (_ChunkedCrossEntropySum.backward)."""
    z = np.asarray(logits, dtype=np.float64)
    lab = ce_labels(labels, mask, ignore_index)
    valid = check_labels(lab, z.shape[1], ignore_index)
    lse = logsumexp_rows(z) if z.shape[0] else np.zeros(0)
    s = token_scales(valid, reduction, num_label_tokens, grad_loss)
    return logit_grad(z, lse, lab, valid, s, 0.0)
