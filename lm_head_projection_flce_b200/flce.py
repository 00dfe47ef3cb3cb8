"""Python binding of libflce.so: argument marshalling only.

Every step of the loss and its gradient runs in the library's CUDA kernels;
this module checks tensors, allocates outputs and workspace with PyTorch (the
caller's device memory) and passes raw pointers and the current CUDA stream
through ctypes.  If the library is missing it raises: there is no fallback.

Entry points mirror include/flce.h:
  forward(hidden, weight, labels, ...)            -> (loss, lse)
  backward(hidden, weight, labels, lse, grad, ...) -> (dhidden, dweight)
  fused_linear_cross_entropy(...)                  autograd-aware convenience
with the options of the NeMo-AutoModel loss pages
("nemo_automodel.components.loss.linear_ce", FusedLinearCrossEntropy:
ignore_index=-100, logit_softcapping=0, reduction='sum', num_label_tokens;
"nemo_automodel.components.models.inkling2.loss": unpadded_vocab_size and an
FP32 head rounded to BF16).
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

LIB_PATH = _build.LIB_PATH

FLCE_OK = 0
FLCE_ERR_BAD_LABEL = 5
FLCE_ERR_TIMEOUT = 6
STATUS = {0: "FLCE_OK", 1: "FLCE_ERR_INVALID_ARG", 2: "FLCE_ERR_WORKSPACE",
          3: "FLCE_ERR_UNSUPPORTED", 4: "FLCE_ERR_CUDA", 5: "FLCE_ERR_BAD_LABEL",
          6: "FLCE_ERR_TIMEOUT"}
REDUCTIONS = {"sum": 0, "mean": 1, "none": 2}
FLCE_BWD_HEAD_COPY_VALID = 1
FLCE_FUSED_HEAD_CAST = 2
W_DTYPES = {torch.bfloat16: 0, torch.float32: 1}

_c_i64 = ctypes.c_int64
_c_int = ctypes.c_int
_c_ptr = ctypes.c_void_p
_c_size = ctypes.c_size_t

# name -> (restype, argtypes); the exported C ABI of include/flce.h
SIGNATURES = {
    "flce_workspace_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_int]),
    "flce_workspace_min_size": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_int]),
    "flce_workspace_size_ex": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_int, ctypes.c_uint]),
    "flce_workspace_min_size_ex": (_c_size, [_c_i64, _c_i64, _c_i64, _c_i64, _c_int,
                                             ctypes.c_uint]),
    "flce_forward": (_c_int, [_c_ptr, _c_ptr, _c_int, _c_ptr, _c_i64, _c_i64, _c_i64, _c_i64,
                              _c_i64, ctypes.c_float, _c_int, _c_i64, _c_ptr, _c_ptr, _c_ptr,
                              _c_size, _c_ptr]),
    "flce_forward_ex": (_c_int, [_c_ptr, _c_ptr, _c_int, _c_ptr, _c_i64, _c_i64, _c_i64,
                                 _c_i64, _c_i64, ctypes.c_float, _c_int, _c_i64, _c_ptr, _c_ptr,
                                 _c_ptr, _c_size, ctypes.c_uint, _c_ptr]),
    "flce_backward": (_c_int, [_c_ptr, _c_ptr, _c_int, _c_ptr, _c_i64, _c_i64, _c_i64, _c_i64,
                               _c_i64, ctypes.c_float, _c_int, _c_i64, _c_ptr, _c_ptr, _c_ptr,
                               _c_ptr, _c_ptr, _c_size, _c_ptr]),
    "flce_backward_ex": (_c_int, [_c_ptr, _c_ptr, _c_int, _c_ptr, _c_i64, _c_i64, _c_i64,
                                  _c_i64, _c_i64, ctypes.c_float, _c_int, _c_i64, _c_ptr,
                                  _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_size, ctypes.c_uint,
                                  _c_ptr]),
    "flce_get_error": (_c_int, [_c_ptr]),
    "flce_status_string": (ctypes.c_char_p, [_c_int]),
    "flce_flops_fwd_bwd": (ctypes.c_double, [_c_i64, _c_i64, _c_i64]),
    "flce_selftest_gemm": (_c_int, [_c_ptr, _c_ptr, _c_ptr, _c_i64, _c_i64, _c_i64, _c_int,
                                    _c_int, _c_ptr]),
    "flce_selftest_wait_timeout": (_c_int, [ctypes.c_uint, _c_ptr]),
    "flce_forward_noalloc": (_c_int, [_c_ptr, _c_ptr, _c_int, _c_ptr, _c_i64, _c_i64, _c_i64,
                                      _c_i64, _c_i64, ctypes.c_float, _c_int, _c_i64, _c_ptr,
                                      _c_ptr, _c_ptr]),
    "flce_ce_workspace_size": (_c_size, [_c_i64]),
    "flce_ce_forward": (_c_int, [_c_ptr, _c_int, _c_ptr, _c_ptr, _c_i64, _c_i64, _c_i64, _c_i64,
                                 _c_int, _c_i64, _c_ptr, _c_ptr, _c_ptr, _c_size, _c_ptr]),
    "flce_ce_backward": (_c_int, [_c_ptr, _c_int, _c_ptr, _c_ptr, _c_i64, _c_i64, _c_i64, _c_i64,
                                  _c_int, _c_i64, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_size, _c_ptr]),
    "flce_launch_count": (ctypes.c_ulonglong, []),
    "flce_profile_start": (_c_int, []),
    "flce_profile_stop": (_c_int, [_c_ptr, _c_int, ctypes.POINTER(_c_int)]),
}


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]

_LIB = None


class FlceError(RuntimeError):
    def __init__(self, where: str, status: int):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def load_library() -> ctypes.CDLL:
    """Load libflce.so (built in-tree).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m lm_head_projection_flce_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _check(where: str, status: int) -> None:
    if status != FLCE_OK:
        raise FlceError(where, status)


def _stream_handle(device: torch.device, stream=None):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr() if t is not None and t.numel() > 0 else 0)


def _vocab(weight: torch.Tensor, unpadded_vocab: int | None) -> int:
    return weight.shape[0] if unpadded_vocab is None or unpadded_vocab <= 0 else int(unpadded_vocab)


def workspace_size(n_tokens: int, hidden: int, padded_vocab: int, unpadded_vocab: int | None,
                   w_dtype: torch.dtype = torch.bfloat16, minimum: bool = False,
                   fused_head_cast: bool = False) -> int:
    lib = load_library()
    fn = lib.flce_workspace_min_size_ex if minimum else lib.flce_workspace_size_ex
    return int(fn(n_tokens, hidden, padded_vocab, unpadded_vocab or 0, W_DTYPES[w_dtype],
                  FLCE_FUSED_HEAD_CAST if fused_head_cast else 0))


def _prepare(hidden, weight, labels):
    if hidden.dtype != torch.bfloat16:
        raise TypeError("hidden must be bf16")
    if weight.dtype not in W_DTYPES:
        raise TypeError("weight must be bf16 or fp32")
    if labels.dtype != torch.int64:
        raise TypeError("labels must be int64")
    h = hidden.shape[-1]
    hid = hidden.reshape(-1, h)
    lab = labels.reshape(-1)
    if hid.shape[0] != lab.shape[0]:
        raise ValueError("hidden and labels disagree on the number of tokens")
    if weight.dim() != 2 or weight.shape[1] != h:
        raise ValueError("weight must be [vocab, hidden]")
    for t in (hid, weight, lab):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if t.device != hid.device or t.device.type != "cuda":
            raise ValueError("tensors must be on one CUDA device")
    return hid, lab


def _workspace(ws, need: int, device) -> tuple[torch.Tensor, int]:
    """The workspace tensor and its size in bytes (any dtype; contiguous, on `device`)."""
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    elif ws.device != device or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on the inputs' device")
    return ws, ws.numel() * ws.element_size()


def _buffer(t, numel: int, dtype, device, name: str) -> torch.Tensor:
    """A caller-supplied buffer the library reads or writes through a raw pointer:
    it must have exactly the expected dtype, size and device, and be contiguous."""
    if t.dtype != dtype or t.numel() != numel or t.device != device or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of {numel} elements on "
                         f"{device}")
    return t


def _forward_outputs(loss, lse, n: int, reduction: str, dev):
    loss_n = n if reduction == "none" else 1
    loss = (torch.empty(loss_n, dtype=torch.float32, device=dev) if loss is None
            else _buffer(loss, loss_n, torch.float32, dev, "loss"))
    lse = (torch.empty(n, dtype=torch.float32, device=dev) if lse is None
           else _buffer(lse, n, torch.float32, dev, "lse"))
    return loss, lse


def forward(hidden, weight, labels, *, ignore_index: int = -100, softcap: float = 0.0,
            unpadded_vocab: int | None = None, reduction: str = "sum",
            num_label_tokens: int | None = None, workspace: torch.Tensor | None = None,
            loss: torch.Tensor | None = None, lse: torch.Tensor | None = None,
            fused_head_cast: bool = False, stream=None):
    """Fused projection + cross entropy.  Returns ``(loss, lse)`` (FP32).

    ``fused_head_cast=True`` (flce_forward_ex with FLCE_FUSED_HEAD_CAST): an
    FP32 head is rounded to BF16 inside the GEMM instead of into a V x H BF16
    copy in the workspace; same results, smaller workspace, slower GEMM.
    """
    lib = load_library()
    hid, lab = _prepare(hidden, weight, labels)
    n, h = hid.shape
    vp = weight.shape[0]
    v = _vocab(weight, unpadded_vocab)
    dev = hid.device
    red = REDUCTIONS[reduction]
    loss, lse = _forward_outputs(loss, lse, n, reduction, dev)
    ws, ws_bytes = _workspace(
        workspace, workspace_size(n, h, vp, v, weight.dtype, fused_head_cast=fused_head_cast), dev)
    st = lib.flce_forward_ex(_ptr(hid), _ptr(weight), W_DTYPES[weight.dtype], _ptr(lab), n, h, vp,
                             v, ignore_index, float(softcap), red, int(num_label_tokens or 0),
                             _ptr(loss), _ptr(lse), _ptr(ws), ws_bytes,
                             FLCE_FUSED_HEAD_CAST if fused_head_cast else 0,
                             _stream_handle(dev, stream))
    _check("flce_forward", st)
    return (loss if reduction == "none" else loss.reshape(())), lse


def _grad_loss(grad_loss, n: int, reduction: str, dev) -> torch.Tensor:
    """The upstream gradient as FP32 on the device: [N] for 'none', else one value."""
    grad = torch.as_tensor(grad_loss).reshape(-1).to(device=dev, dtype=torch.float32).contiguous()
    if grad.numel() != (n if reduction == "none" else 1):
        raise ValueError("grad_loss must have one value per token for reduction='none', "
                         "else one value")
    return grad


def backward(hidden, weight, labels, lse, grad_loss, *, ignore_index: int = -100,
             softcap: float = 0.0, unpadded_vocab: int | None = None, reduction: str = "sum",
             num_label_tokens: int | None = None, workspace: torch.Tensor | None = None,
             dhidden: torch.Tensor | None = None, dweight: torch.Tensor | None = None,
             reuse_head_copy: bool = False, fused_head_cast: bool = False, stream=None):
    """Gradients ``(dhidden [.., H] bf16, dweight [Vp, H] in the head's dtype)``.

    ``reuse_head_copy=True`` (flce_backward_ex with FLCE_BWD_HEAD_COPY_VALID):
    for an FP32 head, skip the FP32 -> BF16 cast and use the copy that
    ``forward`` wrote into the same ``workspace`` -- the caller promises that
    the head and that workspace are unchanged since.  Needs ``workspace``;
    ignored for a BF16 head.

    ``fused_head_cast=True`` (FLCE_FUSED_HEAD_CAST): the recompute and
    dhidden GEMMs round an FP32 head to BF16 inside the kernel; no copy is
    read or written.  Not combinable with ``reuse_head_copy``.
    """
    lib = load_library()
    hid, lab = _prepare(hidden, weight, labels)
    n, h = hid.shape
    vp = weight.shape[0]
    v = _vocab(weight, unpadded_vocab)
    dev = hid.device
    red = REDUCTIONS[reduction]
    grad = _grad_loss(grad_loss, n, reduction, dev)
    lse = _buffer(lse, n, torch.float32, dev, "lse")
    dhidden = (torch.empty_like(hid) if dhidden is None
               else _buffer(dhidden, n * h, torch.bfloat16, dev, "dhidden"))
    dweight = (torch.empty_like(weight) if dweight is None
               else _buffer(dweight, weight.numel(), weight.dtype, dev, "dweight"))
    if reuse_head_copy and workspace is None:
        raise ValueError("reuse_head_copy needs the workspace the forward wrote the copy into")
    if reuse_head_copy and fused_head_cast:
        raise ValueError("fused_head_cast writes no head copy to reuse")
    ws, ws_bytes = _workspace(
        workspace, workspace_size(n, h, vp, v, weight.dtype, fused_head_cast=fused_head_cast), dev)
    flags = (FLCE_BWD_HEAD_COPY_VALID if reuse_head_copy else 0) | (
        FLCE_FUSED_HEAD_CAST if fused_head_cast else 0)
    st = lib.flce_backward_ex(_ptr(hid), _ptr(weight), W_DTYPES[weight.dtype], _ptr(lab), n, h,
                              vp, v, ignore_index, float(softcap), red, int(num_label_tokens or 0),
                              _ptr(grad), _ptr(lse), _ptr(dhidden), _ptr(dweight), _ptr(ws),
                              ws_bytes, flags, _stream_handle(dev, stream))
    _check("flce_backward", st)
    return dhidden.reshape(hidden.shape), dweight


def get_error(device=None, stream=None) -> int:
    """Synchronise and read-and-clear the device error word (FLCE_* status)."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(lib.flce_get_error(_stream_handle(dev, stream)))


def selftest_gemm(a, b, m: int, n: int, k: int, a_mn: bool, b_mn: bool) -> torch.Tensor:
    """D = A . B^T through the library's tensor-core GEMM (tests only)."""
    lib = load_library()
    d = torch.empty(m, n, dtype=torch.float32, device=a.device)
    st = lib.flce_selftest_gemm(_ptr(a), _ptr(b), _ptr(d), m, n, k, int(a_mn), int(b_mn),
                                _stream_handle(a.device))
    _check("flce_selftest_gemm", st)
    return d


def selftest_wait_timeout(timeout_us: int, device=None) -> None:
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check("flce_selftest_wait_timeout",
           lib.flce_selftest_wait_timeout(timeout_us, _stream_handle(dev)))


class _FusedLinearCE(torch.autograd.Function):
    @staticmethod
    def forward(ctx, hidden, weight, labels, ignore_index, softcap, unpadded_vocab, reduction,
                num_label_tokens, fused_head_cast):
        # An FP32 head's BF16 copy, made by the forward, is kept (in the
        # workspace) for the backward instead of being cast again; autograd's
        # version check refuses a backward after the head changed in place.
        # With fused_head_cast there is no copy and nothing is kept.
        ws = None
        if weight.dtype == torch.float32 and not fused_head_cast:
            hid = hidden.reshape(-1, hidden.shape[-1])
            need = workspace_size(hid.shape[0], hid.shape[1], weight.shape[0],
                                  _vocab(weight, unpadded_vocab), weight.dtype)
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=hidden.device)
        loss, lse = forward(hidden, weight, labels, ignore_index=ignore_index, softcap=softcap,
                            unpadded_vocab=unpadded_vocab, reduction=reduction,
                            num_label_tokens=num_label_tokens, workspace=ws,
                            fused_head_cast=fused_head_cast)
        ctx.save_for_backward(hidden, weight, labels, lse)
        ctx.workspace = ws
        ctx.opts = (ignore_index, softcap, unpadded_vocab, reduction, num_label_tokens,
                    fused_head_cast)
        return loss

    @staticmethod
    def backward(ctx, grad_out):
        hidden, weight, labels, lse = ctx.saved_tensors
        ii, c, uv, red, nlt, fused = ctx.opts
        ws = ctx.workspace
        ctx.workspace = None
        dh, dw = backward(hidden, weight, labels, lse, grad_out, ignore_index=ii, softcap=c,
                          unpadded_vocab=uv, reduction=red, num_label_tokens=nlt, workspace=ws,
                          reuse_head_copy=ws is not None, fused_head_cast=fused)
        return dh, dw, None, None, None, None, None, None, None


def fused_linear_cross_entropy(hidden, weight, labels, *, ignore_index: int = -100,
                               softcap: float = 0.0, unpadded_vocab: int | None = None,
                               reduction: str = "sum", num_label_tokens: int | None = None,
                               fused_head_cast: bool = False):
    """Autograd-aware loss: gradients flow to ``hidden`` and ``weight``.

    With an FP32 head the forward's workspace (which holds the head's BF16
    copy, V x H x 2 bytes, and the backward's buffers) is kept until the
    backward runs, so the head is cast once per step; a BF16 head keeps
    nothing between the two.  ``fused_head_cast=True`` rounds an FP32 head
    inside the GEMMs instead: no copy exists and nothing is kept (less memory,
    slower GEMMs, the same results).
    """
    return _FusedLinearCE.apply(hidden, weight, labels, ignore_index, softcap, unpadded_vocab,
                                reduction, num_label_tokens, fused_head_cast)


class CapturedStep:
    """Forward + backward of the fused loss captured once into a CUDA graph.

    The inputs are static device tensors owned here (``hidden``, ``labels``,
    and the head ``weight`` the caller passes, which must stay alive and keep
    its storage); a step copies new values into them (``set_inputs``) and
    calls ``replay()``, which reruns all of the step's kernel launches as one
    graph launch.  Outputs (``loss``, ``lse``, ``dhidden``, ``dweight``) are static
    too and are overwritten by each replay.  Worth it where a step is short
    enough for launch overhead to show (small batches); the results equal the
    eager calls bit for bit.

    The options, ``num_label_tokens`` included, are host values baked into
    the graph when it is captured: a replay normalises by the count given at
    construction even if ``set_inputs`` brought labels with another number of
    live tokens.  ``set_inputs(..., num_label_tokens=k)`` refuses a ``k`` that
    differs from the captured one; build a new CapturedStep for it.
    An FP32 head is cast to BF16 once per replay (the backward reuses the
    forward's copy).
    """

    def __init__(self, hidden, weight, labels, *, ignore_index: int = -100, softcap: float = 0.0,
                 unpadded_vocab: int | None = None, reduction: str = "sum",
                 num_label_tokens: int | None = None, grad_loss=None):
        hid, lab = _prepare(hidden, weight, labels)
        dev = hid.device
        n, h = hid.shape
        self.hidden = hid.clone()
        self.labels = lab.clone()
        self.weight = weight
        self.kw = dict(ignore_index=ignore_index, softcap=softcap, unpadded_vocab=unpadded_vocab,
                       reduction=reduction, num_label_tokens=num_label_tokens)
        v = _vocab(weight, unpadded_vocab)
        self.workspace = torch.empty(max(workspace_size(n, h, weight.shape[0], v, weight.dtype), 16),
                                     dtype=torch.uint8, device=dev)
        self.loss = torch.empty(n if reduction == "none" else 1, dtype=torch.float32, device=dev)
        self.lse = torch.empty(n, dtype=torch.float32, device=dev)
        self.dhidden = torch.empty_like(self.hidden)
        self.dweight = torch.empty_like(weight)
        g = torch.ones(()) if grad_loss is None else grad_loss
        self.grad = _grad_loss(g, n, reduction, dev).clone()
        stream = torch.cuda.Stream(dev)
        stream.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(stream):
            self._step()          # eager: per-device set-up and launch shapes, outside capture
        torch.cuda.current_stream(dev).wait_stream(stream)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=stream):
            self._step()

    def _step(self):
        forward(self.hidden, self.weight, self.labels, loss=self.loss, lse=self.lse,
                workspace=self.workspace, **self.kw)
        backward(self.hidden, self.weight, self.labels, self.lse, self.grad,
                 dhidden=self.dhidden, dweight=self.dweight, workspace=self.workspace,
                 reuse_head_copy=self.weight.dtype == torch.float32, **self.kw)

    def set_inputs(self, hidden=None, labels=None, num_label_tokens: int | None = None) -> None:
        """Copy new token data into the captured input buffers (same shapes).

        ``num_label_tokens``, if given, must equal the value captured at
        construction (it is fixed inside the graph); anything else raises.
        """
        if num_label_tokens is not None and num_label_tokens != self.kw["num_label_tokens"]:
            raise ValueError(f"num_label_tokens={num_label_tokens} differs from the captured "
                             f"{self.kw['num_label_tokens']}; it is fixed when the graph is "
                             "captured")
        if hidden is not None:
            self.hidden.copy_(hidden.reshape(self.hidden.shape), non_blocking=True)
        if labels is not None:
            self.labels.copy_(labels.reshape(self.labels.shape), non_blocking=True)

    def replay(self):
        """Run forward + backward; returns (loss, dhidden, dweight), static buffers."""
        self.graph.replay()
        loss = self.loss if self.kw["reduction"] == "none" else self.loss.reshape(())
        return loss, self.dhidden, self.dweight


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(load_library().flce_launch_count())


def profile_start() -> None:
    """Bracket every library kernel launch with CUDA events until profile_stop()."""
    _check("flce_profile_start", load_library().flce_profile_start())


def profile_stop() -> dict:
    """Per kernel family: launches, device ms (CUDA events) and algorithmic work."""
    lib = load_library()
    cap = 32
    arr = (KernelStat * cap)()
    count = _c_int(0)
    _check("flce_profile_stop", lib.flce_profile_stop(ctypes.cast(arr, _c_ptr), cap,
                                                       ctypes.byref(count)))
    out = {}
    for i in range(min(count.value, cap)):
        st = arr[i]
        out[st.name.decode()] = {"launches": int(st.launches), "total_ms": float(st.total_ms),
                                 "flops": float(st.flops), "bytes": float(st.bytes)}
    return out


def forward_noalloc(hidden, weight, labels, *, ignore_index: int = -100, softcap: float = 0.0,
                    unpadded_vocab: int | None = None, reduction: str = "sum",
                    num_label_tokens: int | None = None, loss: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, stream=None):
    """flce_forward_noalloc: the forward with the library's fixed 32 MiB device
    scratch instead of a workspace, for callers that cannot provide scratch
    memory.  Only the outputs are allocated here (when not given)."""
    lib = load_library()
    hid, lab = _prepare(hidden, weight, labels)
    n, h = hid.shape
    vp = weight.shape[0]
    v = _vocab(weight, unpadded_vocab)
    dev = hid.device
    loss, lse = _forward_outputs(loss, lse, n, reduction, dev)
    st = lib.flce_forward_noalloc(_ptr(hid), _ptr(weight), W_DTYPES[weight.dtype], _ptr(lab), n,
                                  h, vp, v, ignore_index, float(softcap), REDUCTIONS[reduction],
                                  int(num_label_tokens or 0), _ptr(loss), _ptr(lse),
                                  _stream_handle(dev, stream))
    _check("flce_forward_noalloc", st)
    return (loss if reduction == "none" else loss.reshape(())), lse


# ---------------------------------------------------------------- cross entropy on given logits

def _prepare_logits(logits, labels, mask):
    if logits.dtype not in W_DTYPES:
        raise TypeError("logits must be bf16 or fp32")
    if labels.dtype != torch.int64:
        raise TypeError("labels must be int64")
    v = logits.shape[-1]
    z = logits.reshape(-1, v)
    lab = labels.reshape(-1)
    if z.shape[0] != lab.shape[0]:
        raise ValueError("logits and labels disagree on the number of tokens")
    if z.stride(-1) != 1 or not lab.is_contiguous():
        raise ValueError("logits rows and labels must be contiguous")
    m = None
    if mask is not None:
        m = mask.reshape(-1).to(torch.uint8).contiguous()
        if m.shape[0] != lab.shape[0]:
            raise ValueError("mask must match labels")
    for t in (z, lab) + ((m,) if m is not None else ()):
        if t.device.type != "cuda" or t.device != z.device:
            raise ValueError("tensors must be on one CUDA device")
    return z, lab, m


def ce_forward(logits, labels, *, mask=None, ignore_index: int = -100, reduction: str = "sum",
               num_label_tokens: int | None = None, workspace=None,
               loss: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Cross entropy of given logits [..., V] (ChunkedCrossEntropy).  Returns (loss, lse)."""
    lib = load_library()
    z, lab, m = _prepare_logits(logits, labels, mask)
    n, v = z.shape
    dev = z.device
    loss, lse = _forward_outputs(loss, lse, n, reduction, dev)
    ws, ws_bytes = _workspace(workspace, int(lib.flce_ce_workspace_size(n)), dev)
    st = lib.flce_ce_forward(_ptr(z), W_DTYPES[z.dtype], _ptr(lab), _ptr(m), n, v, z.stride(0),
                             ignore_index, REDUCTIONS[reduction], int(num_label_tokens or 0),
                             _ptr(loss), _ptr(lse), _ptr(ws), ws_bytes, _stream_handle(dev, stream))
    _check("flce_ce_forward", st)
    return (loss if reduction == "none" else loss.reshape(())), lse


def ce_backward(logits, labels, lse, grad_loss, *, mask=None, ignore_index: int = -100,
                reduction: str = "sum", num_label_tokens: int | None = None, dlogits=None,
                workspace=None, stream=None):
    """Gradient w.r.t. the logits, in the logits' dtype and shape."""
    lib = load_library()
    z, lab, m = _prepare_logits(logits, labels, mask)
    n, v = z.shape
    dev = z.device
    grad = _grad_loss(grad_loss, n, reduction, dev)
    lse = _buffer(lse, n, torch.float32, dev, "lse")
    if dlogits is None:
        # the kernels write dlogits with the logits' row stride
        dlogits = torch.empty(n, z.stride(0), dtype=z.dtype, device=dev)[:, :v]
    out = dlogits.reshape(n, v)
    if out.dtype != z.dtype or out.device != dev:
        raise ValueError("dlogits must have the logits' dtype and device")
    if out.stride(0) != z.stride(0) or out.stride(1) != 1:
        raise ValueError("dlogits must have the logits' row stride")
    ws, ws_bytes = _workspace(workspace, int(lib.flce_ce_workspace_size(n)), dev)
    st = lib.flce_ce_backward(_ptr(z), W_DTYPES[z.dtype], _ptr(lab), _ptr(m), n, v, z.stride(0),
                              ignore_index, REDUCTIONS[reduction], int(num_label_tokens or 0),
                              _ptr(grad), _ptr(lse), _ptr(out), _ptr(ws), ws_bytes,
                              _stream_handle(dev, stream))
    _check("flce_ce_backward", st)
    return out.reshape(logits.shape)
