"""Pins of the FP64 oracle to facts other than itself (CPU only).

Each ``pin_*`` checks the oracle against a closed form, an invariant, a
library routine it does not call, finite differences or brute force on tiny
inputs.  ``test_pins_catch_planted_mistakes`` plants plausible mistakes in the
oracle (on the CPU) and checks that at least one pin fails for each.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import flce_oracle as O

II = -100


def _bf16_vals(rng, shape, sigma=1.0):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * sigma)
    return x.to(torch.bfloat16).to(torch.float64).numpy()


def _problem(seed, n, h, v, vp=None, ignore=(), sigma_w=0.3):
    rng = np.random.default_rng(seed)
    vp = v if vp is None else vp
    hidden = _bf16_vals(rng, (n, h))
    weight = _bf16_vals(rng, (vp, h), sigma_w)
    labels = rng.integers(0, v, size=n).astype(np.int64)
    for i in ignore:
        labels[i] = II
    return hidden, weight, labels


# ---------------------------------------------------------------------------
# Pins
# ---------------------------------------------------------------------------

def pin_zero_weights(o):
    """W = 0: every logit is 0, so lse = log V (never log Vp) under any softcap,
    the loss is #valid*log V, dh = 0 and dW[v] = sum_n s_n (1/V - [y_n = v]) h[n]."""
    rng = np.random.default_rng(1)
    n, h, v, vp = 6, 4, 5, 8
    hidden = _bf16_vals(rng, (n, h))
    weight = np.zeros((vp, h))
    weight[v:] = 50.0                      # padded rows must never enter the softmax
    labels = np.array([0, 4, II, 2, 2, II], dtype=np.int64)
    for c in (0.0, 3.0):
        r = o.forward(hidden, weight, labels, softcap=c, unpadded_vocab=v)
        assert np.allclose(r.lse, math.log(v), rtol=0, atol=1e-14)
        assert abs(r.loss - 4 * math.log(v)) < 1e-12
        dh, dw = o.backward(hidden, np.where(np.arange(vp)[:, None] < v, 0.0, weight),
                            labels, softcap=c, unpadded_vocab=v)
        assert np.all(dh == 0.0)
        want = np.zeros((vp, h))
        for i in range(n):
            if labels[i] == II:
                continue
            for j in range(v):
                want[j] += (1.0 / v - (1.0 if labels[i] == j else 0.0)) * hidden[i]
        assert np.allclose(dw, want, rtol=0, atol=1e-12)


def pin_permutation_head(o):
    """Head = rows of a permutation matrix: z[n, v] = hidden[n, pi(v)] exactly, so
    the loss is a closed form of the hidden values (catches a transposed head)."""
    rng = np.random.default_rng(2)
    n, v = 5, 6
    pi = [2, 0, 5, 1, 3, 4]                # not an involution
    hidden = _bf16_vals(rng, (n, v), 1.5)
    weight = np.zeros((v + 2, v))
    for r, col in enumerate(pi):
        weight[r, col] = 1.0
    weight[v:] = 7.0
    labels = np.array([3, 1, II, 5, 0], dtype=np.int64)
    for c in (0.0, 2.0):
        cap = (lambda x: c * math.tanh(x / c)) if c > 0 else (lambda x: x)
        r = o.forward(hidden, weight, labels, softcap=c, unpadded_vocab=v, reduction="none")
        for i in range(n):
            zs = [cap(hidden[i, pi[j]]) for j in range(v)]
            lse = math.log(math.fsum(math.exp(t) for t in zs))
            assert abs(r.lse[i] - lse) < 1e-12
            want = 0.0 if labels[i] == II else lse - zs[labels[i]]
            assert abs(r.loss[i] - want) < 1e-12


def pin_two_class_closed_form(o):
    """Two classes with head [[1], [-1]] and hidden [[a]]: logits (a', -a') with
    a' = cap(a); loss(label 0) = softplus(-2a'), and by calculus
    dloss/da = -2*sigmoid(-2a')*cap'(a), dloss/dW = (dz0*a, dz1*a) with
    dz0 = -sigmoid(-2a')*cap'(a) = -dz1."""
    for a in (-1.25, 0.5, 3.0):
        for c in (0.0, 2.0):
            ap = c * math.tanh(a / c) if c > 0 else a
            capd = 1.0 - math.tanh(a / c) ** 2 if c > 0 else 1.0
            hidden = np.array([[a]])
            weight = np.array([[1.0], [-1.0]])
            labels = np.array([0])
            r = o.forward(hidden, weight, labels, softcap=c)
            assert abs(r.loss - math.log1p(math.exp(-2 * ap))) < 1e-13
            sig = 1.0 / (1.0 + math.exp(2 * ap))
            dh, dw = o.backward(hidden, weight, labels, softcap=c)
            assert abs(dh[0, 0] - (-2.0 * sig * capd)) < 1e-13
            assert abs(dw[0, 0] - (-sig * capd * a)) < 1e-13
            assert abs(dw[1, 0] - (sig * capd * a)) < 1e-13


def pin_torch_cross_entropy(o):
    """softcap = 0, V = Vp: torch's cross_entropy on FP64 logits (the library the
    linear_ce page says it matches), for sum, mean and none with ignore_index."""
    hidden, weight, labels = _problem(3, 9, 12, 17, ignore=(2, 7))
    z = torch.from_numpy(hidden) @ torch.from_numpy(weight).T
    y = torch.from_numpy(labels)
    for red in ("sum", "mean", "none"):
        r = o.forward(hidden, weight, labels, reduction=red)
        want = F.cross_entropy(z, y, ignore_index=II, reduction=red).numpy()
        assert np.allclose(r.loss, want, rtol=1e-13, atol=1e-13)
    r = o.forward(hidden, weight, labels, reduction="sum", num_label_tokens=5)
    want = F.cross_entropy(z, y, ignore_index=II, reduction="sum").item() / 5
    assert abs(r.loss - want) < 1e-13
    assert np.allclose(r.lse, torch.logsumexp(z, dim=1).numpy(), rtol=0, atol=1e-13)


def pin_torch_autograd(o):
    """Gradients equal torch autograd of the same loss built from library ops."""
    n, h, v, vp = 7, 6, 11, 13
    hidden, weight, labels = _problem(4, n, h, v, vp, ignore=(1,))
    gvec = np.linspace(-1.0, 2.0, n)
    cases = [("sum", None, 1.7), ("sum", 4, 0.9), ("mean", None, 1.3), ("none", None, gvec)]
    for c in (0.0, 2.5):
        for red, nlt, g in cases:
            ht = torch.tensor(hidden, requires_grad=True)
            wt = torch.tensor(weight, requires_grad=True)
            z = ht @ wt[:v].T
            zc = c * torch.tanh(z / c) if c > 0 else z
            loss = F.cross_entropy(zc, torch.from_numpy(labels), ignore_index=II, reduction=red)
            if nlt is not None:
                loss = loss / nlt
            loss.backward(torch.as_tensor(g, dtype=torch.float64).reshape(loss.shape))
            dh, dw = o.backward(hidden, weight, labels, softcap=c, unpadded_vocab=v,
                                reduction=red, num_label_tokens=nlt, grad_loss=g)
            assert np.allclose(dh, ht.grad.numpy(), rtol=1e-11, atol=1e-13)
            assert np.allclose(dw, wt.grad.numpy(), rtol=1e-11, atol=1e-13)


def pin_finite_differences(o):
    """Central differences (step 1e-6) of the oracle's own loss on N=3, H=5, V=7
    (two padded head rows) agree with its backward, with and without softcap."""
    rng = np.random.default_rng(5)
    n, h, v, vp = 3, 5, 7, 9
    hidden = rng.standard_normal((n, h))
    weight = rng.standard_normal((vp, h)) * 0.7
    labels = np.array([4, II, 6], dtype=np.int64)
    eps = 1e-6
    for c in (0.0, 2.0):
        for red, nlt in (("sum", None), ("sum", 3), ("mean", None)):
            def loss(hh, ww):
                return o.forward(hh, ww, labels, softcap=c, unpadded_vocab=v,
                                 reduction=red, num_label_tokens=nlt).loss
            dh, dw = o.backward(hidden, weight, labels, softcap=c, unpadded_vocab=v,
                                reduction=red, num_label_tokens=nlt)
            for (arr, grad) in ((hidden, dh), (weight, dw)):
                for idx in np.ndindex(arr.shape):
                    old = arr[idx]
                    arr[idx] = old + eps
                    lp = loss(hidden, weight)
                    arr[idx] = old - eps
                    lm = loss(hidden, weight)
                    arr[idx] = old
                    fd = (lp - lm) / (2 * eps)
                    assert abs(fd - grad[idx]) < 1e-7 + 1e-6 * abs(fd), (idx, fd, grad[idx])


def pin_ignored_tokens(o):
    """Ignored positions add exactly 0 to the loss, get exactly-zero dh rows, and
    changing their hidden rows changes neither the loss nor dW."""
    hidden, weight, labels = _problem(6, 8, 6, 10, ignore=(0, 5))
    for c in (0.0, 4.0):
        r = o.forward(hidden, weight, labels, softcap=c, reduction="none")
        assert r.loss[0] == 0.0 and r.loss[5] == 0.0
        dh, dw = o.backward(hidden, weight, labels, softcap=c)
        assert np.all(dh[0] == 0.0) and np.all(dh[5] == 0.0)
        h2 = hidden.copy()
        h2[[0, 5]] = 9.0
        r2 = o.forward(h2, weight, labels, softcap=c)
        assert r2.loss == o.forward(hidden, weight, labels, softcap=c).loss
        _, dw2 = o.backward(h2, weight, labels, softcap=c)
        assert np.allclose(dw2, dw, rtol=0, atol=1e-14)


def pin_row_sum(o):
    """sum_v dz[n, v] = 0 without softcap; sum_v dz/(1 - tanh^2) = 0 with it."""
    hidden, weight, labels = _problem(7, 6, 5, 9, ignore=(3,))
    valid = labels != II
    for c in (0.0, 1.5):
        z = o.project(hidden, weight)
        zc = c * np.tanh(z / c) if c > 0 else z
        lse = np.log(np.exp(zc).sum(axis=1))
        dz = o.logit_grad(z, lse, labels, valid, np.where(valid, 1.3, 0.0), c)
        if c > 0:
            dz = dz / (1.0 - np.tanh(z / c) ** 2)
        assert np.allclose(dz.sum(axis=1), 0.0, atol=1e-13)
        assert np.all(dz[3] == 0.0)


def pin_padded_rows(o):
    """dW rows >= V are exactly 0, and padded rows' contents never change the loss."""
    hidden, weight, labels = _problem(8, 5, 4, 6, vp=9)
    w2 = weight.copy()
    w2[6:] = -40.0
    for c in (0.0, 5.0):
        a = o.forward(hidden, weight, labels, softcap=c, unpadded_vocab=6)
        b = o.forward(hidden, w2, labels, softcap=c, unpadded_vocab=6)
        assert a.loss == b.loss
        _, dw = o.backward(hidden, weight, labels, softcap=c, unpadded_vocab=6)
        assert np.all(dw[6:] == 0.0) and np.any(dw[:6] != 0.0)


def pin_softcap_bound(o):
    """|c*tanh(z/c)| <= c for any z; a very large c reproduces the uncapped loss."""
    z = np.concatenate([np.linspace(-1e6, 1e6, 1001), [0.0, 1e-30, -1e-30]])
    for c in (0.5, 30.0):
        zc = o.apply_softcap(z, c)
        assert np.all(np.abs(zc) <= c)
    hidden, weight, labels = _problem(9, 4, 3, 5)
    a = o.forward(hidden, weight, labels, softcap=0.0).loss
    b = o.forward(hidden, weight, labels, softcap=1e9).loss
    assert abs(a - b) < 1e-6


def pin_reductions(o):
    """sum = sum of per-token losses; mean divides by #valid (NaN when none);
    num_label_tokens divides a sum; it is refused with other reductions."""
    hidden, weight, labels = _problem(10, 7, 4, 6, ignore=(1, 2))
    tok = o.forward(hidden, weight, labels, reduction="none").loss
    s = o.forward(hidden, weight, labels, reduction="sum").loss
    assert abs(s - math.fsum(tok)) < 1e-12
    assert abs(o.forward(hidden, weight, labels, reduction="mean").loss - s / 5) < 1e-12
    assert abs(o.forward(hidden, weight, labels, num_label_tokens=11).loss - s / 11) < 1e-12
    with pytest.raises(ValueError):
        o.forward(hidden, weight, labels, reduction="mean", num_label_tokens=3)
    allign = np.full_like(labels, II)
    assert o.forward(hidden, weight, allign, reduction="sum").loss == 0.0
    assert math.isnan(o.forward(hidden, weight, allign, reduction="mean").loss)
    with pytest.raises(ValueError):
        o.forward(hidden, weight, np.array([0, 1, 6, 0, 0, 0, 0]), unpadded_vocab=6)


def pin_bf16_round(o):
    """FP32 -> BF16 round-to-nearest-even equals torch's cast, including ties
    (1 + 2^-8 -> 1, 1 + 3*2^-8 -> 1 + 2^-6), overflow to inf, signed zero, NaN."""
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(0.02),
        rng.standard_normal(20000).astype(np.float32) * np.float32(1e4),
        np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 3.0e38, -3.4e38, 0.0, -0.0,
                  1e-40, np.inf, -np.inf], dtype=np.float32)])
    got = o.bf16_round(x)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, want)
    assert got[40000] == 1.0 and got[40001] == 1 + 2**-6 and got[40002] == -1.0
    assert np.signbit(got[40006]) and not np.signbit(got[40005])
    nan = o.bf16_round(np.array([np.nan], dtype=np.float32))
    assert np.isnan(nan[0])
    # an FP32 head is rounded before use: f32 head == its bf16-rounded f64 copy
    hidden, _, labels = _problem(12, 4, 8, 6)
    w32 = (rng.standard_normal((6, 8)) * 0.3).astype(np.float32)
    a = o.forward(hidden, w32, labels).loss
    b = o.forward(hidden, torch.from_numpy(w32).to(torch.bfloat16).double().numpy(), labels).loss
    assert a == b


def pin_brute_force_loops(o):
    """Pure-Python loops (math.fsum) on a tiny case agree with the vectorised oracle."""
    hidden, weight, labels = _problem(13, 4, 3, 5, vp=6, ignore=(2,))
    for c in (0.0, 1.25):
        toks = []
        for i in range(4):
            zs = []
            for j in range(5):
                zz = math.fsum(hidden[i, k] * weight[j, k] for k in range(3))
                zs.append(c * math.tanh(zz / c) if c > 0 else zz)
            lse = math.log(math.fsum(math.exp(t) for t in zs))
            toks.append(0.0 if labels[i] == II else lse - zs[labels[i]])
        r = o.forward(hidden, weight, labels, softcap=c, unpadded_vocab=5)
        assert abs(r.loss - math.fsum(toks)) < 1e-12


def pin_row_sampled_forms(o):
    """forward_rows / dh_rows / dw_rows give the rows of the full forward/backward."""
    hidden, weight, labels = _problem(14, 9, 5, 7, vp=10, ignore=(4,))
    for c in (0.0, 2.0):
        for red, nlt, g in (("sum", 6, 1.5), ("mean", None, 0.7),
                            ("none", None, np.linspace(0.5, 1.5, 9))):
            full = o.forward(hidden, weight, labels, softcap=c, unpadded_vocab=7)
            dh, dw = o.backward(hidden, weight, labels, softcap=c, unpadded_vocab=7,
                                reduction=red, num_label_tokens=nlt, grad_loss=g)
            rows = np.array([8, 0, 4])
            lse, tok = o.forward_rows(hidden, weight, labels, rows, softcap=c, unpadded_vocab=7)
            assert np.allclose(lse, full.lse[rows], atol=1e-14)
            assert np.allclose(tok, full.token_loss[rows], atol=1e-14)
            kw = dict(softcap=c, unpadded_vocab=7, reduction=red, num_label_tokens=nlt,
                      grad_loss=g)
            assert np.allclose(o.dh_rows(hidden, weight, labels, rows, **kw), dh[rows], atol=1e-14)
            vr = np.array([9, 2, 6, 7])
            assert np.allclose(o.dw_rows(hidden, weight, labels, vr, full.lse, **kw),
                               dw[vr], atol=1e-14)


PINS = [pin_zero_weights, pin_permutation_head, pin_two_class_closed_form,
        pin_torch_cross_entropy, pin_torch_autograd, pin_finite_differences,
        pin_ignored_tokens, pin_row_sum, pin_padded_rows, pin_softcap_bound,
        pin_reductions, pin_bf16_round, pin_brute_force_loops, pin_row_sampled_forms]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(O)


# ---------------------------------------------------------------------------
# Planted mistakes: each must make at least one pin fail
# ---------------------------------------------------------------------------

def _mutants():
    orig = {name: getattr(O, name) for name in
            ("project", "apply_softcap", "logsumexp_rows", "token_losses", "reduce_losses",
             "token_scales", "logit_grad", "compute_head", "bf16_round", "backward")}

    def lse_no_shift(zc):
        m = zc.max(axis=1, keepdims=True)
        return np.log(np.exp(zc - m).sum(axis=1))

    def head_all_rows(weight, unpadded_vocab):
        return orig["compute_head"](weight, weight.shape[0])

    def cap_no_scale(z, c):
        return np.tanh(z / c) if c > 0 else z

    def losses_flipped(lse, zc, labels, valid):
        return -orig["token_losses"](lse, zc, labels, valid)

    def grad_no_tanh_factor(z, lse, labels, valid, scale, c):
        zc = orig["apply_softcap"](z, c)
        p = np.exp(zc - lse[:, None])
        idx = np.nonzero(valid)[0]
        p[idx, labels[idx]] -= 1.0
        return p * scale[:, None]

    def grad_tanh_unscaled(z, lse, labels, valid, scale, c):
        zc = orig["apply_softcap"](z, c)
        p = np.exp(zc - lse[:, None])
        idx = np.nonzero(valid)[0]
        p[idx, labels[idx]] -= 1.0
        if c > 0:
            p *= 1.0 - np.tanh(z) ** 2
        return p * scale[:, None]

    def grad_sign(z, lse, labels, valid, scale, c):
        return -orig["logit_grad"](z, lse, labels, valid, scale, c)

    def grad_label_shift(z, lse, labels, valid, scale, c):
        return orig["logit_grad"](z, lse, (labels + 1) % z.shape[1], valid, scale, c)

    def reduce_times(tok, valid, reduction, nlt):
        r = orig["reduce_losses"](tok, valid, reduction, None)
        if nlt is not None:
            r = r * nlt
        return r

    def reduce_mean_over_n(tok, valid, reduction, nlt):
        if reduction == "mean":
            return float(np.sum(tok)) / len(tok)
        return orig["reduce_losses"](tok, valid, reduction, nlt)

    def scales_no_mask(valid, reduction, nlt, g):
        return orig["token_scales"](np.ones_like(valid), reduction, nlt, g)

    def bf16_truncate(x):
        f = np.ascontiguousarray(x, dtype=np.float32)
        u = f.view(np.uint32) & np.uint32(0xFFFF0000)
        return u.view(np.float32).astype(np.float64)

    def project_rows_reversed(hidden, head):
        return orig["project"](hidden, head[::-1])

    def project_f32(hidden, head):
        return (np.asarray(hidden, np.float32) @ np.asarray(head, np.float32).T).astype(np.float64)

    def backward_pad_not_zero(hidden, weight, labels, **kw):
        dh, dw = orig["backward"](hidden, weight, labels, **kw)
        v = kw.get("unpadded_vocab") or weight.shape[0]
        dw[v:] = 1e-3
        return dh, dw

    return {
        "lse drops the max shift": ("logsumexp_rows", lse_no_shift),
        "softmax over padded rows": ("compute_head", head_all_rows),
        "softcap without the c factor": ("apply_softcap", cap_no_scale),
        "token loss sign flipped": ("token_losses", losses_flipped),
        "backward drops 1 - tanh^2": ("logit_grad", grad_no_tanh_factor),
        "backward tanh(z) instead of tanh(z/c)": ("logit_grad", grad_tanh_unscaled),
        "logit gradient sign flipped": ("logit_grad", grad_sign),
        "one-hot at the wrong index": ("logit_grad", grad_label_shift),
        "num_label_tokens multiplies": ("reduce_losses", reduce_times),
        "mean over all tokens": ("reduce_losses", reduce_mean_over_n),
        "ignored tokens keep gradient": ("token_scales", scales_no_mask),
        "bf16 by truncation": ("bf16_round", bf16_truncate),
        "head rows in the wrong order": ("project", project_rows_reversed),
        "projection in fp32": ("project", project_f32),
        "padded rows get gradient": ("backward", backward_pad_not_zero),
    }


@pytest.mark.parametrize("mutant", list(_mutants().keys()))
def test_pins_catch_planted_mistakes(mutant, monkeypatch):
    name, fn = _mutants()[mutant]
    monkeypatch.setattr(O, name, fn)
    caught = []
    for pin in PINS:
        try:
            pin(O)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin detects: {mutant}"


# ---------------------------------------------------------------------------
# Cross entropy on given logits (chunked_ce page)
# ---------------------------------------------------------------------------

def test_ce_oracle_matches_torch_cross_entropy():
    """Forward and logits gradient equal torch's cross_entropy and its autograd
    on FP64 logits, with ignore_index, mask and every reduction."""
    rng = np.random.default_rng(21)
    n, v = 11, 37
    z = rng.standard_normal((n, v)) * 2.0
    labels = rng.integers(0, v, size=n)
    labels[3] = II
    mask = np.ones(n, dtype=np.uint8)
    mask[[0, 7]] = 0
    eff = labels.copy()
    eff[[0, 7]] = II
    g = np.linspace(0.5, 1.5, n)
    for red, nlt, grad in (("sum", None, 1.3), ("sum", 6, 0.7), ("mean", None, 2.0), ("none", None, g)):
        r = O.ce_forward(z, labels, mask=mask, reduction=red, num_label_tokens=nlt)
        zt = torch.tensor(z, requires_grad=True)
        loss = F.cross_entropy(zt, torch.from_numpy(eff), ignore_index=II, reduction=red)
        if nlt is not None:
            loss = loss / nlt
        assert np.allclose(r.loss, loss.detach().numpy(), rtol=1e-13, atol=1e-13)
        loss.backward(torch.as_tensor(grad, dtype=torch.float64).reshape(loss.shape))
        dz = O.ce_backward(z, labels, mask=mask, reduction=red, num_label_tokens=nlt, grad_loss=grad)
        assert np.allclose(dz, zt.grad.numpy(), rtol=1e-12, atol=1e-14)
    assert np.all(O.ce_backward(z, labels, mask=mask)[[0, 3, 7]] == 0.0)


def test_ce_oracle_equals_fused_oracle_with_identity_head():
    """With W = I the fused loss is the cross entropy of the hidden values."""
    rng = np.random.default_rng(22)
    n, v = 6, 9
    h = _bf16_vals(rng, (n, v), 1.7)
    labels = rng.integers(0, v, size=n)
    a = O.ce_forward(h, labels)
    b = O.forward(h, np.eye(v), labels)
    assert abs(a.loss - b.loss) < 1e-12 and np.allclose(a.lse, b.lse, atol=1e-13)
