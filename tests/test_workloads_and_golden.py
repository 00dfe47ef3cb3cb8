"""Seeded input recipe and the oracle's regression fixture (CPU only)."""
import json
import math
import os

import numpy as np
import torch

from lm_head_projection_flce_b200 import workloads as W
from oracle import flce_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def test_recipe_shapes_dtypes_and_ignore_count():
    for w in (W.TINY, W.custom(300, 72, 1000, 1024, w_dtype="f32", ignore_frac=0.2, seed=7),
              W.custom(50, 16, 77, label_dist="zipf", ignore_frac=0.1, seed=8)):
        d = W.generate(w)
        assert d["hidden"].shape == (w.n_tokens, w.hidden) and d["hidden"].dtype == torch.bfloat16
        want_w = torch.float32 if w.w_dtype == "f32" else torch.bfloat16
        assert d["weight"].shape == (w.padded_vocab, w.hidden) and d["weight"].dtype == want_w
        lab = d["labels"]
        k = int(math.floor(w.ignore_frac * w.n_tokens + 0.5))
        assert int((lab == W.IGNORE_INDEX).sum()) == k
        assert d["num_label_tokens"] == w.n_tokens - k
        live = lab[lab != W.IGNORE_INDEX]
        assert int(live.min()) >= 0 and int(live.max()) < w.vocab


def test_recipe_is_deterministic():
    a = W.generate(W.TINY)
    b = W.generate(W.TINY)
    for k in ("hidden", "weight", "labels"):
        assert torch.equal(a[k], b[k])


def test_zipf_inverse_cdf():
    # rank-1 mass under s = 1.1 over V = 1000 and monotone frequencies
    u = np.random.default_rng(0).random(200000)
    ids = W.zipf_inverse_cdf(u, 1000, 1.1)
    p1 = 1.0 / np.sum(np.arange(1, 1001, dtype=np.float64) ** -1.1)
    assert abs(np.mean(ids == 0) - p1) < 0.005
    counts = np.bincount(ids, minlength=1000)
    assert counts[0] > counts[1] > counts[5] > counts[100]
    assert ids.min() >= 0 and ids.max() <= 999


def test_workload_table():
    names = [w.name for w in W.WORKLOAD_ORDER]
    assert len(set(names)) == 5
    c2 = W.LLAMA_HEAD
    assert (c2.n_tokens, c2.hidden, c2.vocab) == (4096, 4096, 128256)
    assert abs(c2.flops_fwd_bwd - 8 * 4096 * 128256 * 4096) < 1


def test_golden_tiny_oracle_regression():
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        g = json.load(f)
    w = W.TINY
    d = W.generate(w)
    hidden = d["hidden"].double().numpy()
    weight = d["weight"].double().numpy()
    labels = d["labels"].numpy()
    kw = dict(ignore_index=W.IGNORE_INDEX, softcap=w.softcap, unpadded_vocab=w.vocab,
              reduction=w.reduction)
    fwd = O.forward(hidden, weight, labels, **kw)
    dh, dw = O.backward(hidden, weight, labels, **kw)
    assert abs(fwd.loss - g["loss"]) < 1e-9 * abs(g["loss"])
    assert np.allclose(fwd.lse[:8], g["lse_first8"], rtol=1e-12, atol=0)
    assert np.allclose(dh[0, :8], g["dh_row0_first8"], rtol=1e-10, atol=1e-15)
    assert abs(float(np.abs(dw).sum()) - g["dw_abs_sum"]) < 1e-9 * g["dw_abs_sum"]
