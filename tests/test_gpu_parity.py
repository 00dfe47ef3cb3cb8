"""GPU parity of the CUDA path (through the C ABI) against the FP64 oracle at
sizes the oracle finishes in seconds: several tiles in every dimension, ragged
tails, multiple backward vocabulary chunks, every reduction and the edge cases."""
import math

import numpy as np
import pytest
import torch

from lm_head_projection_flce_b200 import flce
from lm_head_projection_flce_b200 import workloads as W
from oracle import flce_oracle as O

from gpu_common import (GRAD_REL, LSE_ABS, assert_parity, gpu_device, max_rel, run_gpu,
                        run_oracle, to_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return gpu_device()


# ----------------------------------------------------------- GEMM self-test

@pytest.mark.parametrize("a_mn", [False, True])
@pytest.mark.parametrize("b_mn", [False, True])
@pytest.mark.parametrize("mnk", [(128, 256, 64), (296, 264, 328), (1000, 1024, 520), (8, 8, 8)])
def test_tensor_core_gemm_selftest(dev, a_mn, b_mn, mnk):
    m, n, k = mnk
    g = torch.Generator().manual_seed(m * 7 + n * 3 + k)
    a = torch.randn(m, k, generator=g).to(torch.bfloat16)
    b = torch.randn(n, k, generator=g).to(torch.bfloat16)
    ref = a.float() @ b.float().T
    a_dev = (a.T.contiguous() if a_mn else a).to(dev)
    b_dev = (b.T.contiguous() if b_mn else b).to(dev)
    d = flce.selftest_gemm(a_dev, b_dev, m, n, k, a_mn, b_mn)
    torch.cuda.synchronize(dev)
    assert torch.allclose(d.cpu(), ref, rtol=1e-4, atol=1e-3), float((d.cpu() - ref).abs().max())


# ----------------------------------------------------------- parity cases

CASES = {
    "tiny": W.TINY,
    "ragged_softcap_f32head": W.custom(333, 328, 1000, 1024, w_dtype="f32", softcap=30.0,
                                       ignore_frac=0.1, seed=11),
    "multi_tile": W.custom(1100, 1024, 8269, 8269, ignore_frac=0.05, seed=12),
    "ktail_softcap_padded": W.custom(700, 520, 5000, 5120, softcap=30.0, ignore_frac=0.1,
                                     w_sigma=0.05, seed=13),
    "zipf_labels": W.custom(512, 256, 3000, 3000, label_dist="zipf", ignore_frac=0.2, seed=14),
    # hidden (12 ragged 256-row tiles x 8200 = 49 MB) is too large to stay in L2 whole, so the
    # projection and recompute GEMMs take their tile order from the traffic model; ragged
    # edges in every dimension (3000 tokens, 8200 = 128 x 64 + 8 hidden, 20011 of 20480 rows)
    "fallback_raster_ragged": W.custom(3000, 8200, 20011, 20480, softcap=30.0, ignore_frac=0.05,
                                       w_sigma=0.01, seed=15),
}


@pytest.mark.parametrize("name", list(CASES))
def test_parity(dev, name):
    w = CASES[name]
    d = W.generate(w)
    assert_parity(run_gpu(d, w, dev), run_oracle(d, w))


@pytest.mark.parametrize("reduction,nlt", [("mean", None), ("none", None), ("sum", 977)])
def test_reductions(dev, reduction, nlt):
    w = CASES["ktail_softcap_padded"]
    d = W.generate(w)
    grad = None
    if reduction == "none":
        grad = torch.linspace(-1.0, 2.0, w.n_tokens, dtype=torch.float32)
    else:
        grad = torch.tensor([0.75])
    got = run_gpu(d, w, dev, reduction=reduction, grad=grad, num_label_tokens=nlt)
    ref = run_oracle(d, w, reduction=reduction, grad=grad, num_label_tokens=nlt)
    assert_parity(got, ref)


def test_multi_chunk_backward(dev):
    """A smaller workspace makes the backward stream the vocabulary in narrower
    chunks (down to 256 columns): same result within tolerance."""
    w = CASES["multi_tile"]
    d = W.generate(w)
    ref = run_oracle(d, w)
    lo = flce.workspace_size(w.n_tokens, w.hidden, w.padded_vocab, w.vocab, minimum=True)
    hi = flce.workspace_size(w.n_tokens, w.hidden, w.padded_vocab, w.vocab)
    for ws in (lo, lo + 2 * w.n_tokens * 256 * 3, hi):
        assert_parity(run_gpu(d, w, dev, ws_bytes=ws), ref)


def test_outputs_stay_in_bounds(dev):
    """Sentinels after every output and the workspace survive a ragged case."""
    w = CASES["ragged_softcap_f32head"]
    d = W.generate(w)
    n, h, vp = w.n_tokens, w.hidden, w.padded_vocab
    pad = 4096
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    sent = -12345.0
    loss_b = torch.full((1 + pad,), sent, device=dev)
    lse_b = torch.full((n + pad,), sent, device=dev)
    dh_b = torch.full((n * h + pad,), sent, device=dev, dtype=torch.bfloat16)
    dw_b = torch.full((vp * h + pad,), sent, device=dev, dtype=torch.float32)
    ws_n = flce.workspace_size(n, h, vp, w.vocab, torch.float32)
    ws_b = torch.full((ws_n + pad,), 0xA5, device=dev, dtype=torch.uint8)
    loss, lse = flce.forward(hid, wt, lab, softcap=w.softcap, unpadded_vocab=w.vocab,
                             workspace=ws_b[:ws_n], loss=loss_b[:1], lse=lse_b[:n])
    dh, dw = flce.backward(hid, wt, lab, lse, torch.ones(1, device=dev), softcap=w.softcap,
                           unpadded_vocab=w.vocab, workspace=ws_b[:ws_n],
                           dhidden=dh_b[:n * h].view(n, h), dweight=dw_b[:vp * h].view(vp, h))
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_OK
    assert torch.all(loss_b[1:] == sent) and torch.all(lse_b[n:] == sent)
    assert torch.all(dh_b[n * h:] == sent) and torch.all(dw_b[vp * h:] == sent)
    assert torch.all(ws_b[ws_n:] == 0xA5)
    ref = run_oracle(d, w)
    assert float(np.max(np.abs(lse.double().cpu().numpy() - ref["lse"]))) <= LSE_ABS
    assert max_rel(dh.double().cpu().numpy(), ref["dh"]) <= GRAD_REL
    assert max_rel(dw.double().cpu().numpy(), ref["dw"]) <= GRAD_REL


# ----------------------------------------------------------- edge cases

def test_zero_tokens(dev):
    w = W.custom(0, 64, 300, 320, seed=20)
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    loss, lse = flce.forward(hid, wt, lab, unpadded_vocab=w.vocab, reduction="sum")
    mean, _ = flce.forward(hid, wt, lab, unpadded_vocab=w.vocab, reduction="mean")
    none, _ = flce.forward(hid, wt, lab, unpadded_vocab=w.vocab, reduction="none")
    dw = torch.full_like(wt, 7.0)
    dh, dw = flce.backward(hid, wt, lab, lse, torch.ones(1, device=dev), unpadded_vocab=w.vocab,
                           dweight=dw)
    torch.cuda.synchronize(dev)
    assert float(loss) == 0.0 and math.isnan(float(mean)) and none.numel() == 0
    assert dh.numel() == 0 and torch.all(dw == 0)


def test_all_tokens_ignored(dev):
    w = W.custom(200, 128, 700, 768, ignore_frac=1.0, softcap=5.0, seed=21)
    d = W.generate(w)
    got = run_gpu(d, w, dev)
    ref = run_oracle(d, w)
    assert float(got["loss"].reshape(-1)[0]) == 0.0
    assert np.all(got["dh"] == 0) and np.all(got["dw"] == 0)
    assert float(np.max(np.abs(got["lse"] - ref["lse"]))) <= LSE_ABS
    mean = run_gpu(d, w, dev, reduction="mean")
    assert math.isnan(float(mean["loss"].reshape(-1)[0]))
    assert np.all(mean["dh"] == 0) and np.all(mean["dw"] == 0)


@pytest.mark.parametrize("softcap", [0.0, 3.0])
def test_single_vocabulary_row(dev, softcap):
    w = W.custom(150, 64, 1, 16, softcap=softcap, ignore_frac=0.2, seed=22)
    d = W.generate(w)
    got = run_gpu(d, w, dev)
    ref = run_oracle(d, w)
    assert float(np.max(np.abs(got["lse"] - ref["lse"]))) <= LSE_ABS
    assert abs(float(got["loss"].reshape(-1)[0])) <= 1e-3
    assert np.all(got["dw"][1:] == 0) and np.max(np.abs(got["dh"])) <= 1e-6


def test_bad_labels_are_flagged_and_ignored(dev):
    w = W.custom(300, 128, 900, 1024, softcap=0.0, seed=23)
    d = W.generate(w)
    bad = d["labels"].clone()
    bad[3] = w.vocab + 5          # a padded row: never a valid target
    bad[7] = -7
    bad[100] = 10 ** 9
    d_bad = dict(d, labels=bad)
    got = run_gpu(d_bad, w, dev)
    assert got["status"] == flce.FLCE_ERR_BAD_LABEL
    assert flce.get_error(dev) == flce.FLCE_OK   # the word was cleared
    fixed = bad.clone()
    fixed[[3, 7, 100]] = W.IGNORE_INDEX
    ref = run_oracle(dict(d, labels=fixed), w)
    got["status"] = flce.FLCE_OK
    assert_parity(got, ref)


def test_pipeline_wait_timeout_is_reported(dev):
    flce.selftest_wait_timeout(20000, dev)          # 20 ms wait that nothing satisfies
    assert flce.get_error(dev) == flce.FLCE_ERR_TIMEOUT
    # the context stays usable
    w = W.TINY
    d = W.generate(w)
    assert_parity(run_gpu(d, w, dev), run_oracle(d, w))


def test_no_nv_sized_allocation(dev):
    """The call's own allocations (the workspace) stay far below N*V bytes."""
    n, h, v = 4096, 1024, 128256
    g = torch.Generator(device="cpu").manual_seed(5)
    hid = torch.randn(n, h, generator=g).to(torch.bfloat16).to(dev)
    wt = (torch.randn(v, h, generator=g) * 0.02).to(torch.bfloat16).to(dev)
    lab = torch.randint(0, v, (n,), generator=g).to(dev)
    loss = torch.empty(1, device=dev)
    lse = torch.empty(n, device=dev)
    dh = torch.empty_like(hid)
    dw = torch.empty_like(wt)
    grad = torch.ones(1, device=dev)
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    flce.forward(hid, wt, lab, loss=loss, lse=lse)
    flce.backward(hid, wt, lab, lse, grad, dhidden=dh, dweight=dw)
    torch.cuda.synchronize(dev)
    extra = torch.cuda.max_memory_allocated(dev) - base
    assert extra < n * v, (extra, n * v)
    assert flce.get_error(dev) == flce.FLCE_OK


def test_autograd_wrapper(dev):
    w = CASES["ktail_softcap_padded"]
    d = W.generate(w)
    hid = d["hidden"].to(dev).requires_grad_(True)
    wt = d["weight"].to(dev).requires_grad_(True)
    lab = d["labels"].to(dev)
    loss = flce.fused_linear_cross_entropy(hid, wt, lab, softcap=w.softcap, unpadded_vocab=w.vocab)
    (2.0 * loss).backward()
    torch.cuda.synchronize(dev)
    ref = run_oracle(d, w, grad=torch.tensor([2.0]))
    assert abs(float(loss.detach()) - float(ref["loss"])) <= 1e-4 * abs(float(ref["loss"]))
    assert max_rel(hid.grad.double().cpu().numpy(), ref["dh"]) <= GRAD_REL
    assert max_rel(wt.grad.double().cpu().numpy(), ref["dw"]) <= GRAD_REL


def test_results_are_bitwise_reproducible(dev):
    """Tiles are taken dynamically, but every output element is computed by one
    tile in a fixed contraction order and the loss sums run in a fixed order,
    so repeated calls give identical bits."""
    w = CASES["ktail_softcap_padded"]
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    outs = []
    for _ in range(3):
        loss, lse = flce.forward(hid, wt, lab, softcap=w.softcap, unpadded_vocab=w.vocab)
        dh, dw = flce.backward(hid, wt, lab, lse, torch.ones(1, device=dev), softcap=w.softcap,
                               unpadded_vocab=w.vocab)
        torch.cuda.synchronize(dev)
        outs.append((loss.clone(), lse.clone(), dh.clone(), dw.clone()))
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)


@pytest.mark.parametrize("softcap", [1.0, 30.0])
def test_softcap_saturates_on_huge_logits(dev, softcap):
    """Logits of +-1e3 and beyond: the capped logits sit at +-c, so every lse
    lies in [-c + log V, c + log V], and gradients stay finite and match the oracle."""
    w = W.custom(160, 64, 700, 704, softcap=softcap, ignore_frac=0.1, w_sigma=40.0, seed=24)
    d = W.generate(w)
    got = run_gpu(d, w, dev)
    ref = run_oracle(d, w)
    assert np.all(np.isfinite(got["dh"])) and np.all(np.isfinite(got["dw"]))
    lo, hi = -softcap + np.log(700) - 1e-3, softcap + np.log(700) + 1e-3
    assert np.all(got["lse"] >= lo) and np.all(got["lse"] <= hi)
    assert_parity(got, ref)


def test_forward_backward_replay_in_a_cuda_graph(dev):
    """After one eager call (which does the per-device set-up), forward + backward
    only enqueue kernels on the caller's stream, so the pair can be captured
    into a CUDA graph and replayed; replays match the eager results bit for bit."""
    w = CASES["ktail_softcap_padded"]
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    n, h = hid.shape
    ws = torch.empty(flce.workspace_size(n, h, wt.shape[0], w.vocab), dtype=torch.uint8, device=dev)
    loss = torch.empty(1, device=dev)
    lse = torch.empty(n, device=dev)
    dh = torch.empty_like(hid)
    dw = torch.empty_like(wt)
    grad = torch.ones(1, device=dev)
    kw = dict(softcap=w.softcap, unpadded_vocab=w.vocab, workspace=ws)

    def step():
        flce.forward(hid, wt, lab, loss=loss, lse=lse, **kw)
        flce.backward(hid, wt, lab, lse, grad, dhidden=dh, dweight=dw, **kw)

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        step()                                   # eager warm-up on the capture stream
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    eager = [t.clone() for t in (loss, lse, dh, dw)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for _ in range(3):
        for t in (loss, lse, dh, dw):
            t.zero_()
        g.replay()
        torch.cuda.synchronize(dev)
        for a, b in zip(eager, (loss, lse, dh, dw)):
            assert torch.equal(a, b)
    assert flce.get_error(dev) == flce.FLCE_OK


def test_binding_refuses_mismatched_buffers(dev):
    """Caller-supplied outputs, lse and workspace reach the library as raw
    pointers, so the binding refuses any of the wrong dtype, size or layout
    before a kernel could write past them."""
    w = CASES["ktail_softcap_padded"]
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    n, h = hid.reshape(-1, hid.shape[-1]).shape
    kw = dict(softcap=w.softcap, unpadded_vocab=w.vocab)
    loss, lse = flce.forward(hid, wt, lab, **kw)
    g = torch.ones(1, device=dev)
    bad = [
        lambda: flce.forward(hid, wt, lab, lse=torch.empty(n - 1, device=dev), **kw),
        lambda: flce.forward(hid, wt, lab, loss=torch.empty(2, device=dev), **kw),
        lambda: flce.forward(hid, wt, lab, lse=torch.empty(n, device=dev, dtype=torch.float64),
                             **kw),
        lambda: flce.backward(hid, wt, lab, lse[:-1], g, **kw),
        lambda: flce.backward(hid, wt, lab, lse, torch.ones(2, device=dev), **kw),
        lambda: flce.backward(hid, wt, lab, lse, g, **kw,
                              dhidden=torch.empty(n, h - 8, device=dev, dtype=torch.bfloat16)),
        lambda: flce.backward(hid, wt, lab, lse, g, **kw,
                              dweight=torch.empty_like(wt, dtype=torch.float16)),
        lambda: flce.backward(hid, wt, lab, lse, g, **kw,
                              dweight=torch.empty(wt.shape[1], wt.shape[0], device=dev,
                                                  dtype=wt.dtype).t()),
        lambda: flce.forward(hid, wt, lab, workspace=torch.empty(64, 64, device=dev).t(), **kw),
    ]
    for call in bad:
        with pytest.raises(ValueError):
            call()
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_OK


def test_fp32_head_chunkings_noalloc_and_graph_replay(dev):
    """FP32 head (cast to BF16 inside each call): the same results for every
    backward chunking, flce_forward_noalloc equals flce_forward bit for bit,
    and a captured forward + backward replays bit for bit."""
    w = W.custom(300, 264, 5000, 5120, w_dtype="f32", softcap=30.0, ignore_frac=0.1, seed=21)
    d = W.generate(w)
    ref = run_oracle(d, w)
    lo = flce.workspace_size(w.n_tokens, w.hidden, w.padded_vocab, w.vocab, torch.float32,
                             minimum=True)
    hi = flce.workspace_size(w.n_tokens, w.hidden, w.padded_vocab, w.vocab, torch.float32)
    for ws in (lo, lo + 2 * w.n_tokens * 256 * 4, hi):   # 20, 7 and 5 backward chunks
        assert_parity(run_gpu(d, w, dev, ws_bytes=ws), ref)

    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    kw = dict(softcap=w.softcap, unpadded_vocab=w.vocab)
    loss_a, lse_a = flce.forward(hid, wt, lab, **kw)
    loss_b, lse_b = flce.forward_noalloc(hid, wt, lab, **kw)
    torch.cuda.synchronize(dev)
    assert torch.equal(loss_a, loss_b) and torch.equal(lse_a, lse_b)

    ws = torch.empty(lo + 2 * w.n_tokens * 256 * 4, dtype=torch.uint8, device=dev)
    loss = torch.empty(1, device=dev)
    lse = torch.empty(w.n_tokens, device=dev)
    dh = torch.empty_like(hid)
    dw = torch.empty_like(wt)
    grad = torch.ones(1, device=dev)

    def step():
        flce.forward(hid, wt, lab, loss=loss, lse=lse, workspace=ws, **kw)
        flce.backward(hid, wt, lab, lse, grad, dhidden=dh, dweight=dw, workspace=ws, **kw)

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    eager = [t.clone() for t in (loss, lse, dh, dw)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for _ in range(2):
        for t in (loss, lse, dh, dw):
            t.zero_()
        g.replay()
        torch.cuda.synchronize(dev)
        for a, b in zip(eager, (loss, lse, dh, dw)):
            assert torch.equal(a, b)
    assert flce.get_error(dev) == flce.FLCE_OK


def test_backward_reuses_the_forwards_head_copy(dev):
    """flce_backward_ex with FLCE_BWD_HEAD_COPY_VALID: with an FP32 head the
    backward skips its own cast and reads the BF16 copy the forward left at
    the start of the workspace; dhidden and dW equal the recasting backward
    bit for bit at every chunking, and one launch (the cast) is saved.  A
    CapturedStep with an FP32 head (which uses the flag) and the autograd
    wrapper (which keeps the forward's workspace) agree with them too."""
    w = W.custom(300, 264, 5000, 5120, w_dtype="f32", softcap=30.0, ignore_frac=0.1, seed=23)
    d = W.generate(w)
    ref = run_oracle(d, w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    kw = dict(softcap=w.softcap, unpadded_vocab=w.vocab)
    grad = torch.ones(1, device=dev)
    lo = flce.workspace_size(w.n_tokens, w.hidden, w.padded_vocab, w.vocab, torch.float32,
                             minimum=True)
    hi = flce.workspace_size(w.n_tokens, w.hidden, w.padded_vocab, w.vocab, torch.float32)
    for size in (lo, lo + 2 * w.n_tokens * 256 * 4, hi):
        ws = torch.empty(size, dtype=torch.uint8, device=dev)
        loss, lse = flce.forward(hid, wt, lab, workspace=ws, **kw)
        l0 = flce.launch_count()
        dh_a, dw_a = flce.backward(hid, wt, lab, lse, grad, workspace=ws, **kw)
        l1 = flce.launch_count()
        # clear the workspace: the flagged backward can then only see the
        # copy that the next forward writes
        ws.fill_(0xFF)
        flce.forward(hid, wt, lab, workspace=ws, loss=loss, lse=lse, **kw)
        l2 = flce.launch_count()
        dh_b, dw_b = flce.backward(hid, wt, lab, lse, grad, workspace=ws, reuse_head_copy=True,
                                   **kw)
        l3 = flce.launch_count()
        torch.cuda.synchronize(dev)
        assert torch.equal(dh_a, dh_b) and torch.equal(dw_a, dw_b)
        assert (l3 - l2) == (l1 - l0) - 1
        got = {"loss": loss.double().cpu().numpy(), "lse": lse.double().cpu().numpy(),
               "dh": dh_b.double().cpu().numpy(), "dw": dw_b.double().cpu().numpy(),
               "status": flce.get_error(dev)}
        assert_parity(got, ref)

    step = flce.CapturedStep(hid, wt, lab, **kw)
    loss_c, dh_c, dw_c = (t.clone() for t in step.replay())
    torch.cuda.synchronize(dev)
    assert torch.equal(dh_c, dh_a) and torch.equal(dw_c, dw_a)
    with pytest.raises(ValueError):
        step.set_inputs(hid, lab, num_label_tokens=7)

    h = hid.clone().requires_grad_(True)
    wr = wt.clone().requires_grad_(True)
    flce.fused_linear_cross_entropy(h, wr, lab, **kw).backward()
    torch.cuda.synchronize(dev)
    assert torch.equal(h.grad, dh_a) and torch.equal(wr.grad, dw_a)
    assert flce.get_error(dev) == flce.FLCE_OK

    with pytest.raises(ValueError):   # the flag needs the forward's workspace
        flce.backward(hid, wt, lab, lse, grad, reuse_head_copy=True, **kw)


def test_captured_step_replays_the_eager_step(dev):
    """flce.CapturedStep: a forward + backward captured into a CUDA graph over
    static buffers equals the eager calls bit for bit, also after new token
    data is copied into its input buffers."""
    w = CASES["ktail_softcap_padded"]
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    kw = dict(softcap=w.softcap, unpadded_vocab=w.vocab)

    def eager(h, y):
        loss, lse = flce.forward(h, wt, y, **kw)
        dh, dw = flce.backward(h, wt, y, lse, torch.ones(1, device=dev), **kw)
        return loss, dh, dw

    step = flce.CapturedStep(hid, wt, lab, **kw)
    for h, y in ((hid, lab), (hid.flip(0).contiguous(), lab.roll(7).contiguous())):
        step.set_inputs(h, y)
        got = [t.clone() for t in step.replay()]
        ref = eager(h, y)
        torch.cuda.synchronize(dev)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    assert flce.get_error(dev) == flce.FLCE_OK


@pytest.mark.parametrize("name", ["tiny_n64_h256_v1024", "n4096_h4096_v128256"])
def test_matches_torch_cross_entropy_on_fp32_logits(dev, name):
    """Library cross-check ("matching PyTorch behavior"): with no softcap and
    V = Vp, torch's cross_entropy and autograd on the FP32 logits of the same
    BF16 inputs give the loss, dhidden and dW of the fused kernels, which never
    form those logits.  The 64-token and the benchmark workload (the latter
    in the launch configuration bench.py times)."""
    w = W.WORKLOADS[name]
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    nlt = d["num_label_tokens"] if w.normalize_by_label_tokens else None
    loss, lse = flce.forward(hid, wt, lab, reduction=w.reduction, num_label_tokens=nlt)
    dh, dw = flce.backward(hid, wt, lab, lse, torch.ones(1, device=dev), reduction=w.reduction,
                           num_label_tokens=nlt)
    h32 = hid.float().requires_grad_(True)
    w32 = wt.float().requires_grad_(True)
    z = h32 @ w32.T
    ref = torch.nn.functional.cross_entropy(z, lab, ignore_index=W.IGNORE_INDEX, reduction="sum")
    if nlt:
        ref = ref / nlt
    ref.backward()
    ref_lse = torch.logsumexp(z.detach(), dim=1)
    torch.cuda.synchronize(dev)
    assert flce.get_error(dev) == flce.FLCE_OK
    assert float((lse - ref_lse).abs().max()) <= LSE_ABS
    r = float(ref.detach())
    assert abs(float(loss) - r) <= 1e-4 * abs(r)
    for got, want in ((dh.float(), h32.grad), (dw.float(), w32.grad)):
        scale = float(want.abs().max())
        assert float((got - want).abs().max()) <= GRAD_REL * scale


@pytest.mark.parametrize("w_dtype", ["bf16", "f32"])
def test_buffers_only_16_byte_aligned_take_the_16_byte_stores(dev, w_dtype):
    """The G chunk, dW and dhidden-accumulator epilogues use 32-byte stores
    when their buffer and its rows are 32-byte aligned, else 16-byte ones (the
    ABI only asks for 16).  A workspace and outputs placed 16 bytes past a
    32-byte boundary take the second path; every result equals the first's
    bit for bit."""
    # H = 528: rows are 32-byte multiples, and the last 32 columns of a 256-wide
    # tile run past H (that chunk always takes the 16-byte stores)
    w = W.custom(520, 528, 3000, 3072, w_dtype=w_dtype, softcap=30.0, ignore_frac=0.1, seed=41)
    d = W.generate(w)
    hid, wt, lab = (d[k].to(dev) for k in ("hidden", "weight", "labels"))
    kw = dict(softcap=w.softcap, unpadded_vocab=w.vocab)
    size = flce.workspace_size(w.n_tokens, w.hidden, w.padded_vocab, w.vocab, wt.dtype)
    grad = torch.ones(1, device=dev)

    def run(offset):
        ws = torch.empty(size + 64, dtype=torch.uint8, device=dev)[offset:offset + size]
        dwb = torch.empty(wt.numel() + 16, dtype=wt.dtype, device=dev)
        dw = dwb[16 // wt.element_size() if offset else 0:][:wt.numel()].view(wt.shape)
        assert (ws.data_ptr() % 32 == 0) == (offset == 0)
        assert (dw.data_ptr() % 32 == 0) == (offset == 0)
        loss, lse = flce.forward(hid, wt, lab, workspace=ws, **kw)
        dh, dw = flce.backward(hid, wt, lab, lse, grad, workspace=ws, dweight=dw, **kw)
        torch.cuda.synchronize(dev)
        assert flce.get_error(dev) == flce.FLCE_OK
        return loss.clone(), lse.clone(), dh.clone(), dw.clone()

    for x, y in zip(run(0), run(16)):
        assert torch.equal(x, y)
