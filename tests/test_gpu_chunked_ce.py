"""GPU parity of cross entropy on given logits (the chunked_ce page's
ChunkedCrossEntropy) against the FP64 oracle: BF16 and FP32 logits, rows that
do not start on a 16-byte boundary, row strides, masks, every reduction and
the edge cases.  Tolerances as for the fused path: |dlse| <= 2e-3, loss
relative error <= 1e-4, max|d dlogits| <= 1e-2 * max|ref|."""
import math

import numpy as np
import pytest
import torch

from lm_head_projection_flce_b200 import flce
from lm_head_projection_flce_b200 import workloads as W
from oracle import flce_oracle as O

from gpu_common import GRAD_REL, LOSS_REL, LSE_ABS, gpu_device, max_rel

pytestmark = pytest.mark.gpu
II = -100


@pytest.fixture(scope="module")
def dev():
    return gpu_device()


def _case(seed, n, v, dtype, ignore_frac=0.1, scale=2.0, ld=None):
    g = torch.Generator().manual_seed(seed)
    ld = v if ld is None else ld
    full = (torch.randn(n, ld, generator=g) * scale).to(dtype)
    logits = full[:, :v]
    labels = torch.randint(0, v, (n,), generator=g)
    k = int(math.floor(ignore_frac * n + 0.5))
    if k:
        labels[torch.randperm(n, generator=g)[:k]] = II
    return full, logits, labels


def _check(dev, logits, labels, *, mask=None, reduction="sum", nlt=None, grad=None):
    z = logits.to(dev)
    lab = labels.to(dev)
    m = None if mask is None else mask.to(dev)
    loss, lse = flce.ce_forward(z, lab, mask=m, reduction=reduction, num_label_tokens=nlt)
    if grad is None:
        grad = torch.ones(1) if reduction != "none" else torch.ones(labels.shape[0])
    dz = flce.ce_backward(z, lab, lse, grad.to(dev), mask=m, reduction=reduction,
                          num_label_tokens=nlt)
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_OK
    zf = logits.double().numpy()
    mk = None if mask is None else mask.numpy()
    ref = O.ce_forward(zf, labels.numpy(), mask=mk, reduction=reduction, num_label_tokens=nlt)
    rdz = O.ce_backward(zf, labels.numpy(), mask=mk, reduction=reduction, num_label_tokens=nlt,
                        grad_loss=grad.double().numpy())
    assert float(np.max(np.abs(lse.double().cpu().numpy() - ref.lse))) <= LSE_ABS
    lg = np.asarray(loss.double().cpu().numpy()).reshape(-1)
    lr = np.asarray(ref.loss).reshape(-1)
    if lr.size == 1:
        if math.isnan(lr[0]):
            assert math.isnan(lg[0])
        elif lr[0] == 0:
            assert lg[0] == 0
        else:
            assert abs(lg[0] - lr[0]) <= LOSS_REL * abs(lr[0])
    else:
        assert float(np.max(np.abs(lg - lr))) <= LSE_ABS
    assert dz.dtype == logits.dtype and dz.shape == logits.shape
    assert max_rel(dz.double().cpu().numpy(), rdz) <= GRAD_REL
    return dz


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n,v", [(64, 1024), (333, 1000), (129, 12289), (8, 7), (300, 50001)])
def test_ce_parity(dev, dtype, n, v):
    _, logits, labels = _case(n * 31 + v, n, v, dtype)
    _check(dev, logits, labels)


@pytest.mark.parametrize("reduction,nlt", [("mean", None), ("none", None), ("sum", 77)])
def test_ce_reductions_and_mask(dev, reduction, nlt):
    _, logits, labels = _case(5, 257, 3001, torch.bfloat16)
    mask = (torch.arange(257) % 5 != 0).to(torch.uint8)
    grad = torch.linspace(-1, 2, 257) if reduction == "none" else torch.tensor([1.5])
    dz = _check(dev, logits, labels, mask=mask, reduction=reduction, nlt=nlt, grad=grad)
    assert torch.all(dz[::5] == 0)


def test_ce_row_stride_and_unaligned_rows(dev):
    # rows 1001 elements apart: every row starts at a different 16-byte phase
    full, logits, labels = _case(6, 90, 997, torch.bfloat16, ld=1001)
    z = full.to(dev)[:, :997]
    lab = labels.to(dev)
    loss, lse = flce.ce_forward(z, lab)
    dbuf = torch.full((90, 1001), 7.0, dtype=torch.bfloat16, device=dev)
    flce.ce_backward(z, lab, lse, torch.ones(1, device=dev), dlogits=dbuf[:, :997])
    torch.cuda.synchronize(dev)
    ref = O.ce_forward(logits.double().numpy(), labels.numpy())
    rdz = O.ce_backward(logits.double().numpy(), labels.numpy())
    assert float(np.max(np.abs(lse.double().cpu().numpy() - ref.lse))) <= LSE_ABS
    assert max_rel(dbuf[:, :997].double().cpu().numpy(), rdz) <= GRAD_REL
    assert torch.all(dbuf[:, 997:] == 7.0)          # the gap between rows is untouched


def test_ce_edge_cases(dev):
    z = torch.zeros(0, 50, dtype=torch.bfloat16, device=dev)
    lab = torch.zeros(0, dtype=torch.int64, device=dev)
    loss, _ = flce.ce_forward(z, lab)
    mean, _ = flce.ce_forward(z, lab, reduction="mean")
    torch.cuda.synchronize(dev)
    assert float(loss) == 0.0 and math.isnan(float(mean))
    _, logits, labels = _case(8, 40, 300, torch.float32, ignore_frac=1.0)
    dz = _check(dev, logits, labels)
    assert torch.all(dz == 0)
    # a bad label is flagged and contributes nothing
    _, logits, labels = _case(9, 40, 300, torch.bfloat16, ignore_frac=0.0)
    bad = labels.clone()
    bad[4] = 300
    zz = logits.to(dev)
    loss, lse = flce.ce_forward(zz, bad.to(dev))
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_ERR_BAD_LABEL
    fixed = bad.clone()
    fixed[4] = II
    ref = O.ce_forward(logits.double().numpy(), fixed.numpy())
    assert abs(float(loss) - ref.loss) <= LOSS_REL * abs(ref.loss)


def test_ce_matches_fused_path_on_materialised_logits(dev):
    """The fused projection + CE equals CE on the FP32 logits it never writes."""
    g = torch.Generator().manual_seed(10)
    hid = torch.randn(200, 256, generator=g).to(torch.bfloat16).to(dev)
    wt = (torch.randn(3000, 256, generator=g) * 0.05).to(torch.bfloat16).to(dev)
    lab = torch.randint(0, 3000, (200,), generator=g).to(dev)
    l1, lse1 = flce.forward(hid, wt, lab)
    logits = hid.float() @ wt.float().T
    l2, lse2 = flce.ce_forward(logits, lab)
    torch.cuda.synchronize(dev)
    assert torch.allclose(lse1, lse2, atol=1e-3, rtol=0)
    assert abs(float(l1) - float(l2)) <= 1e-4 * abs(float(l2))


@pytest.mark.parametrize("dtype,ld", [(torch.bfloat16, 20013), (torch.float32, 20011)])
def test_ce_multi_segment_rows_unaligned_with_mask(dev, dtype, ld):
    """Rows long enough to be cut into several segments, each row starting at
    a different 16-byte phase, with a mask and a row stride."""
    n, v = 70, 20009
    full, logits, labels = _case(11, n, v, dtype, ld=ld)
    mask = (torch.arange(n) % 7 != 3).to(torch.uint8)
    z = full.to(dev)[:, :v]
    lab = labels.to(dev)
    loss, lse = flce.ce_forward(z, lab, mask=mask.to(dev))
    dbuf = torch.full((n, ld), 7.0, dtype=dtype, device=dev)
    flce.ce_backward(z, lab, lse, torch.ones(1, device=dev), mask=mask.to(dev),
                     dlogits=dbuf[:, :v])
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_OK
    zf = logits.double().numpy()
    ref = O.ce_forward(zf, labels.numpy(), mask=mask.numpy())
    rdz = O.ce_backward(zf, labels.numpy(), mask=mask.numpy())
    assert float(np.max(np.abs(lse.double().cpu().numpy() - ref.lse))) <= LSE_ABS
    assert abs(float(loss) - ref.loss) <= LOSS_REL * abs(ref.loss)
    assert max_rel(dbuf[:, :v].double().cpu().numpy(), rdz) <= GRAD_REL
    assert torch.all(dbuf[:, v:] == 7.0)
    assert torch.all(dbuf[3::7, :v] == 0)


def test_ce_segments_of_only_minus_infinity(dev):
    """A row whose leading segments hold only -inf logits (masked vocabulary
    entries): their partials are empty and must not poison the merge."""
    n, v = 40, 20000
    _, logits, labels = _case(12, n, v, torch.bfloat16, ignore_frac=0.0)
    logits[:10, :12000] = float("-inf")
    labels[:10] = torch.randint(12000, v, (10,), generator=torch.Generator().manual_seed(3))
    dz = _check(dev, logits, labels)
    assert torch.all(dz[:10, :12000] == 0)


def test_ce_full_size_bench_workload(dev):
    """The benchmark's logits [4096, 128256] BF16 in the launch configuration
    bench.py times: lse and the loss for every row, dlogits on sampled rows."""
    w = W.CE_LOGITS
    d = W.generate_logits(w)
    logits, labels, nlt = d["logits"], d["labels"], d["num_label_tokens"]
    z = logits.to(dev)
    lab = labels.to(dev)
    loss, lse = flce.ce_forward(z, lab, reduction=w.reduction, num_label_tokens=nlt)
    dz = flce.ce_backward(z, lab, lse, torch.ones(1, device=dev), reduction=w.reduction,
                          num_label_tokens=nlt)
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_OK
    lse_g = lse.double().cpu().numpy()
    tok = np.zeros(w.n_tokens)
    worst = 0.0
    for r0 in range(0, w.n_tokens, 512):
        blk = logits[r0:r0 + 512].double().numpy()
        ref = O.ce_forward(blk, labels[r0:r0 + 512].numpy(), reduction="none")
        worst = max(worst, float(np.max(np.abs(lse_g[r0:r0 + 512] - ref.lse))))
        tok[r0:r0 + 512] = ref.loss
    assert worst <= LSE_ABS
    ref_total = float(tok.sum()) / nlt
    assert abs(float(loss) - ref_total) <= LOSS_REL * abs(ref_total)
    rows = torch.randperm(w.n_tokens, generator=torch.Generator().manual_seed(5))[:48]
    ignored = torch.nonzero(labels == II)[:4, 0]
    rows = torch.cat([rows, ignored, torch.tensor([0, w.n_tokens - 1])]).unique()
    sub = logits[rows].double().numpy()
    rdz = O.ce_backward(sub, labels[rows].numpy(), reduction=w.reduction, num_label_tokens=nlt)
    assert max_rel(dz[rows.to(dev)].double().cpu().numpy(), rdz) <= GRAD_REL


@pytest.mark.parametrize("n,v", [(300, 50001), (40, 70000)])
def test_ce_replay_in_a_cuda_graph(dev, n, v):
    """After one eager call (per-device set-up and launch shapes), forward +
    backward only enqueue kernels, so they can be captured into a CUDA graph
    and replayed bit for bit; the second shape cuts its rows into segments."""
    _, logits, labels = _case(13, n, v, torch.bfloat16)
    z, lab = logits.to(dev), labels.to(dev)
    ws = torch.empty(int(flce.load_library().flce_ce_workspace_size(n)), dtype=torch.uint8,
                     device=dev)
    loss = torch.empty(1, device=dev)
    lse = torch.empty(n, device=dev)
    dz = torch.empty_like(z)
    grad = torch.ones(1, device=dev)

    def step():
        flce.ce_forward(z, lab, loss=loss, lse=lse, workspace=ws)
        flce.ce_backward(z, lab, lse, grad, dlogits=dz, workspace=ws)

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    eager = [t.clone() for t in (loss, lse, dz)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for _ in range(2):
        for t in (loss, lse, dz):
            t.zero_()
        g.replay()
        torch.cuda.synchronize(dev)
        for a, b in zip(eager, (loss, lse, dz)):
            assert torch.equal(a, b)
    assert flce.get_error(dev) == flce.FLCE_OK
