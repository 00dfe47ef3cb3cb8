"""Seeded synthetic inputs for the fused LM-head projection + cross-entropy.

This module only draws random numbers: it holds no step of the loss or of its
gradient, so the CUDA path and the CPU oracle can both read their inputs from
it without sharing any of the method's arithmetic.

Shapes follow the workloads of the NeMo-AutoModel loss pages
("nemo_automodel.components.loss.linear_ce", FusedLinearCrossEntropy.forward:
hidden states ``[batch, sequence, hidden]`` flattened to ``N = batch*sequence``
tokens, labels ``[batch, sequence]``, head ``[vocab, hidden]``;
"nemo_automodel.components.models.inkling2.loss": a padded head
``[padded_vocab, hidden]`` of which the first ``unpadded_vocab_size`` rows are
used, optionally held in FP32).

Recipe (every draw from one ``torch.Generator`` seeded with ``seed``, in this
order): hidden ``~N(0,1)`` in FP32 rounded to BF16; head ``~N(0, w_sigma)`` in
FP32 (rounded to BF16 unless the head is FP32); labels uniform over
``[0, vocab)`` or Zipf(s) by inverse CDF over ranks ``1..vocab`` (token id =
rank - 1); then exactly ``floor(ignore_frac*N + 0.5)`` positions, chosen by a
seeded permutation, are set to ``ignore_index``.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic problem: sizes, value distributions and loss options."""

    name: str
    n_tokens: int
    hidden: int
    vocab: int                 # unpadded vocabulary: rows that enter the softmax
    padded_vocab: int          # rows of the head tensor
    batch: int = 1
    seq: int = 0
    w_dtype: str = "bf16"      # "bf16" or "f32" (an FP32 head is rounded to BF16 before use)
    w_sigma: float = 0.02
    label_dist: str = "uniform"  # "uniform" or "zipf"
    zipf_s: float = 1.1
    ignore_frac: float = 0.0
    softcap: float = 0.0
    reduction: str = "sum"     # "sum", "mean" or "none"
    normalize_by_label_tokens: bool = False
    seed: int = 0

    @property
    def flops_fwd_bwd(self) -> float:
        """Dense work of one forward + recompute backward: 8*N*V*H (V unpadded)."""
        return 8.0 * self.n_tokens * self.vocab * self.hidden


# The five workloads.  Sizes and distributions follow the configurations this
# library is measured on; each is seeded with 1000 + its position (1-based).
WORKLOADS: dict[str, Workload] = {}


def _register(w: Workload) -> Workload:
    WORKLOADS[w.name] = w
    return w


TINY = _register(Workload(
    name="tiny_n64_h256_v1024", n_tokens=64, hidden=256, vocab=1024,
    padded_vocab=1024, batch=1, seq=64, w_sigma=0.02, ignore_frac=0.10,
    softcap=0.0, reduction="sum", seed=1001))

LLAMA_HEAD = _register(Workload(
    name="n4096_h4096_v128256", n_tokens=4096, hidden=4096, vocab=128256,
    padded_vocab=128256, batch=2, seq=2048, w_sigma=0.02, ignore_frac=0.05,
    softcap=0.0, reduction="sum", normalize_by_label_tokens=True, seed=1002))

SOFTCAP_F32_HEAD = _register(Workload(
    name="n8192_h5376_v256000_vp262144_softcap30_f32head", n_tokens=8192,
    hidden=5376, vocab=256000, padded_vocab=262144, batch=4, seq=2048,
    w_dtype="f32", w_sigma=0.02, ignore_frac=0.05, softcap=30.0,
    reduction="sum", seed=1003))

LONG_SEQ = _register(Workload(
    name="long_n32768_h4096_v151936_zipf", n_tokens=32768, hidden=4096,
    vocab=151936, padded_vocab=151936, batch=1, seq=32768, w_sigma=0.02,
    label_dist="zipf", zipf_s=1.1, ignore_frac=0.20, softcap=0.0,
    reduction="sum", normalize_by_label_tokens=True, seed=1004))

LARGE_HEAD = _register(Workload(
    name="n16384_h8192_v200000_vp202048_softcap30", n_tokens=16384,
    hidden=8192, vocab=200000, padded_vocab=202048, batch=8, seq=2048,
    w_sigma=0.015, ignore_frac=0.10, softcap=30.0, reduction="sum", seed=1005))

# Ordered as listed above.
WORKLOAD_ORDER = [TINY, LLAMA_HEAD, SOFTCAP_F32_HEAD, LONG_SEQ, LARGE_HEAD]

# A reduced case for profiler captures: the head (268 MB) is still larger than
# L2, so DRAM counters mean something, but the whole run holds under 1 GB.
PROFILE_CASE = _register(Workload(
    name="profile_n2048_h4096_v32768", n_tokens=2048, hidden=4096, vocab=32768,
    padded_vocab=32768, batch=1, seq=2048, w_sigma=0.02, ignore_frac=0.05, softcap=0.0,
    reduction="sum", normalize_by_label_tokens=True, seed=2001))


def custom(n_tokens: int, hidden: int, vocab: int, padded_vocab: int | None = None,
           **kw) -> Workload:
    """A workload of arbitrary shape (parity cases with ragged tiles, edge cases)."""
    padded_vocab = vocab if padded_vocab is None else padded_vocab
    name = kw.pop("name", f"custom_n{n_tokens}_h{hidden}_v{vocab}_vp{padded_vocab}")
    return Workload(name=name, n_tokens=n_tokens, hidden=hidden, vocab=vocab,
                    padded_vocab=padded_vocab, batch=1, seq=n_tokens, **kw)


def n_ignored(w: Workload) -> int:
    return int(math.floor(w.ignore_frac * w.n_tokens + 0.5))


def zipf_inverse_cdf(u: np.ndarray, vocab: int, s: float) -> np.ndarray:
    """Token ids (rank - 1) for uniform draws ``u`` under P(rank k) ~ k^-s."""
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    pmf = ranks ** (-s)
    cdf = np.cumsum(pmf)
    cdf /= cdf[-1]
    idx = np.searchsorted(cdf, u, side="right")
    return np.minimum(idx, vocab - 1).astype(np.int64)


def generate(w: Workload, device: str | torch.device = "cpu") -> dict:
    """Draw the inputs of ``w`` on the CPU (bit-reproducible) and move them to ``device``.

    Returns ``hidden`` (bf16 [N,H]), ``weight`` ([Vp,H], bf16 or f32),
    ``labels`` (int64 [N]) and ``num_label_tokens`` (count of non-ignored labels).
    """
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    n, h, v, vp = w.n_tokens, w.hidden, w.vocab, w.padded_vocab
    hidden = torch.randn(n, h, generator=g, dtype=torch.float32).to(torch.bfloat16)
    weight = torch.randn(vp, h, generator=g, dtype=torch.float32)
    weight.mul_(w.w_sigma)
    if w.w_dtype == "bf16":
        weight = weight.to(torch.bfloat16)
    elif w.w_dtype != "f32":
        raise ValueError(f"unknown head dtype {w.w_dtype!r}")
    if w.label_dist == "uniform":
        labels = torch.randint(0, v, (n,), generator=g, dtype=torch.int64)
    elif w.label_dist == "zipf":
        u = torch.rand(n, generator=g, dtype=torch.float64).numpy()
        labels = torch.from_numpy(zipf_inverse_cdf(u, v, w.zipf_s))
    else:
        raise ValueError(f"unknown label distribution {w.label_dist!r}")
    k = n_ignored(w)
    if k > 0:
        perm = torch.randperm(n, generator=g)[:k]
        labels[perm] = IGNORE_INDEX
    num_label_tokens = int((labels != IGNORE_INDEX).sum().item())
    out = {"hidden": hidden, "weight": weight, "labels": labels,
           "num_label_tokens": num_label_tokens}
    if str(device) != "cpu":
        out = {k_: (t.to(device) if isinstance(t, torch.Tensor) else t) for k_, t in out.items()}
    return out


# Cross entropy on given logits (the chunked_ce page's ChunkedCrossEntropy):
# logits [N, V] in BF16 drawn N(0, sigma) with sigma = 1.28, the spread of the
# logits of the 4096 x 4096 x 128256 workload (hidden N(0,1), head N(0, 0.02):
# std = 0.02 * sqrt(4096)); labels uniform, 5% ignored.
@dataclasses.dataclass(frozen=True)
class LogitsWorkload:
    name: str
    n_tokens: int
    vocab: int
    dtype: str = "bf16"
    sigma: float = 1.28
    ignore_frac: float = 0.05
    reduction: str = "sum"
    normalize_by_label_tokens: bool = True
    seed: int = 0


CE_LOGITS = LogitsWorkload(name="ce_logits_n4096_v128256_bf16", n_tokens=4096, vocab=128256,
                           seed=3002)


def generate_logits(w: LogitsWorkload) -> dict:
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    logits = torch.randn(w.n_tokens, w.vocab, generator=g, dtype=torch.float32).mul_(w.sigma)
    logits = logits.to(torch.bfloat16 if w.dtype == "bf16" else torch.float32)
    labels = torch.randint(0, w.vocab, (w.n_tokens,), generator=g, dtype=torch.int64)
    k = int(math.floor(w.ignore_frac * w.n_tokens + 0.5))
    if k > 0:
        labels[torch.randperm(w.n_tokens, generator=g)[:k]] = IGNORE_INDEX
    return {"logits": logits, "labels": labels,
            "num_label_tokens": int((labels != IGNORE_INDEX).sum().item())}
