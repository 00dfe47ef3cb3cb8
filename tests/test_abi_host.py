"""The C ABI on the host (CPU only): the library loads, exports every symbol the
header declares, sizes its workspace, and refuses bad arguments before it
touches the GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from lm_head_projection_flce_b200 import build as B
from lm_head_projection_flce_b200 import flce

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flce.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return flce.load_library()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flce_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = header_functions()
    for want in ("flce_forward", "flce_backward", "flce_workspace_size", "flce_get_error"):
        assert want in names


def test_library_exports_every_header_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (flce_\w+)", out))
    missing = [n for n in header_functions() if n not in exported]
    assert not missing, missing
    for n in header_functions():
        assert hasattr(lib, n)
    assert set(flce.SIGNATURES) == set(header_functions())


def test_library_is_sm100a_only():
    # the build command targets sm_100a and nothing else
    assert B.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_workspace_size_arithmetic(lib):
    ws = flce.workspace_size
    # C2-sized: forward partials (501 tiles x 4096 x 8 B) and backward chunk buffer
    n, h, v = 4096, 4096, 128256
    total = ws(n, h, v, v)
    fwd = 501 * n * 8
    assert total >= fwd
    assert total >= n * h * 4                      # FP32 dhidden accumulator
    assert total < n * v * 2                       # never a [N, V] BF16 buffer
    assert ws(n, h, v, v, minimum=True) < total
    # an FP32 head needs room for its BF16 copy
    assert ws(64, 256, 1024, 1000, w_dtype=__import__("torch").float32) >= 1000 * 256 * 2
    # invalid shapes report 0
    assert lib.flce_workspace_size(10, 7, 100, 100, 0) == 0        # H not a multiple of 8
    assert lib.flce_workspace_size(10, 8, 100, 101, 0) == 0        # V > Vp
    assert lib.flce_workspace_size(-1, 8, 100, 100, 0) == 0
    assert lib.flce_workspace_size(10, 8, 100, 100, 7) == 0        # bad dtype code
    assert lib.flce_workspace_size(0, 8, 100, 0, 0) > 0            # N = 0 is valid


def test_flops_helper(lib):
    assert lib.flce_flops_fwd_bwd(4096, 4096, 128256) == 8.0 * 4096 * 4096 * 128256


def test_status_strings(lib):
    for code in range(7):
        assert lib.flce_status_string(code)
    assert b"unknown" in lib.flce_status_string(99)


FAKE = 1 << 20  # 16-byte-aligned fake device address: never dereferenced on these paths


def _fwd(lib, **kw):
    a = dict(hidden=FAKE, weight=FAKE, w_dtype=0, labels=FAKE, n=64, h=256, vp=1024, v=1024,
             ii=-100, c=0.0, red=0, nlt=0, loss=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 40,
             stream=None)
    a.update(kw)
    return lib.flce_forward(a["hidden"], a["weight"], a["w_dtype"], a["labels"], a["n"], a["h"],
                            a["vp"], a["v"], a["ii"], a["c"], a["red"], a["nlt"], a["loss"],
                            a["lse"], a["ws"], a["ws_bytes"], a["stream"])


def _bwd(lib, **kw):
    a = dict(hidden=FAKE, weight=FAKE, w_dtype=0, labels=FAKE, n=64, h=256, vp=1024, v=1024,
             ii=-100, c=0.0, red=0, nlt=0, grad=FAKE, lse=FAKE, dh=FAKE, dw=FAKE, ws=FAKE,
             ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.flce_backward(a["hidden"], a["weight"], a["w_dtype"], a["labels"], a["n"], a["h"],
                             a["vp"], a["v"], a["ii"], a["c"], a["red"], a["nlt"], a["grad"],
                             a["lse"], a["dh"], a["dw"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("call", [_fwd, _bwd])
def test_bad_arguments_fail_closed_on_the_host(lib, call):
    bad = [
        dict(h=250),                 # H not a multiple of 8
        dict(h=0),
        dict(n=-1),
        dict(v=2000),                # unpadded > padded
        dict(vp=0),
        dict(c=-1.0),                # negative softcap
        dict(c=float("inf")),
        dict(c=float("nan")),
        dict(red=3),
        dict(red=1, nlt=5),          # num_label_tokens only with sum
        dict(red=2, nlt=5),
        dict(w_dtype=2),
        dict(hidden=0),
        dict(labels=0),
        dict(weight=0),
        dict(hidden=FAKE + 8),       # misaligned for the TMA engine
        dict(weight=FAKE + 4),
        dict(labels=FAKE + 4),
    ]
    for kw in bad:
        assert call(lib, **kw) == 1, kw
    assert call(lib, ws=0) == 2
    assert call(lib, ws_bytes=1000) == 2
    assert call(lib, ws=FAKE + 8) == 2


def test_backward_ex_flags(lib):
    def bex(flags, **kw):
        a = dict(hidden=FAKE, weight=FAKE, w_dtype=1, labels=FAKE, n=64, h=256, vp=1024, v=1024,
                 ii=-100, c=0.0, red=0, nlt=0, grad=FAKE, lse=FAKE, dh=FAKE, dw=FAKE, ws=FAKE,
                 ws_bytes=1 << 40, stream=None)
        a.update(kw)
        return lib.flce_backward_ex(a["hidden"], a["weight"], a["w_dtype"], a["labels"], a["n"],
                                    a["h"], a["vp"], a["v"], a["ii"], a["c"], a["red"], a["nlt"],
                                    a["grad"], a["lse"], a["dh"], a["dw"], a["ws"], a["ws_bytes"],
                                    flags, a["stream"])
    assert bex(4) == 1 and bex(0x80000000) == 1                  # unknown bits
    assert bex(3) == 1                          # reuse a copy and write none: contradictory
    assert bex(1, h=250) == 1 and bex(1, ws=0) == 2              # the usual checks stay
    assert bex(2, h=250) == 1 and bex(2, ws=0) == 2
    # the documented flags pass the host checks (then the missing GPU answers)
    import torch
    if not torch.cuda.is_available():
        assert bex(flce.FLCE_BWD_HEAD_COPY_VALID) in (3, 4)
        assert bex(flce.FLCE_FUSED_HEAD_CAST) in (3, 4)
        assert bex(0) in (3, 4)


def test_forward_ex_flags(lib):
    def fex(flags, **kw):
        a = dict(hidden=FAKE, weight=FAKE, w_dtype=1, labels=FAKE, n=64, h=256, vp=1024, v=1024,
                 ii=-100, c=0.0, red=0, nlt=0, loss=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 40,
                 stream=None)
        a.update(kw)
        return lib.flce_forward_ex(a["hidden"], a["weight"], a["w_dtype"], a["labels"], a["n"],
                                   a["h"], a["vp"], a["v"], a["ii"], a["c"], a["red"], a["nlt"],
                                   a["loss"], a["lse"], a["ws"], a["ws_bytes"], flags,
                                   a["stream"])
    assert fex(1) == 1 and fex(4) == 1 and fex(0x80000000) == 1  # only FLCE_FUSED_HEAD_CAST
    assert fex(2, h=250) == 1 and fex(2, ws=0) == 2
    import torch
    if not torch.cuda.is_available():
        assert fex(flce.FLCE_FUSED_HEAD_CAST) in (3, 4)
        assert fex(0) in (3, 4)


def test_workspace_size_without_the_head_copy(lib):
    """FLCE_FUSED_HEAD_CAST drops exactly the FP32 head's BF16 copy (V x H x 2
    bytes, rounded up to 1 KiB) from both sizes; a BF16 head has no copy."""
    f32, bf16 = 1, 0
    for n, h, vp, v in ((4096, 4096, 128256, 128256), (8192, 5376, 262144, 256000),
                        (333, 328, 1024, 1000), (0, 8, 100, 0)):
        vv = v if v > 0 else vp
        copy = -(-vv * h * 2 // 1024) * 1024
        for full in (lib.flce_workspace_size_ex, lib.flce_workspace_min_size_ex):
            assert full(n, h, vp, v, f32, 0) - full(n, h, vp, v, f32, 2) == copy
            assert full(n, h, vp, v, bf16, 0) == full(n, h, vp, v, bf16, 2)
            assert full(n, h, vp, v, f32, 1) == 0 and full(n, h, vp, v, f32, 4) == 0
        assert lib.flce_workspace_size_ex(n, h, vp, v, f32, 0) == \
            lib.flce_workspace_size(n, h, vp, v, f32)
        assert lib.flce_workspace_min_size_ex(n, h, vp, v, f32, 0) == \
            lib.flce_workspace_min_size(n, h, vp, v, f32)


def test_backward_specific_arguments(lib):
    for kw in (dict(grad=0), dict(lse=0), dict(dh=0), dict(dw=0), dict(dh=FAKE + 2),
               dict(dw=FAKE + 8)):
        assert _bwd(lib, **kw) == 1, kw


def test_forward_specific_arguments(lib):
    assert _fwd(lib, loss=0) == 1
    assert _fwd(lib, lse=0) == 1
    assert _fwd(lib, loss=FAKE + 2) == 1


def test_valid_arguments_without_gpu_report_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # all checks pass, then the device query fails: an error status, no crash
    assert _fwd(lib) in (3, 4)
    assert _bwd(lib) in (3, 4)
    assert lib.flce_get_error(None) in (3, 4)
    assert lib.flce_selftest_gemm(FAKE, FAKE, FAKE, 128, 256, 64, 0, 0, None) in (3, 4)
    assert lib.flce_selftest_wait_timeout(0, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    h = torch.zeros(4, 8, dtype=torch.bfloat16)
    w = torch.zeros(16, 8, dtype=torch.bfloat16)
    y = torch.zeros(4, dtype=torch.int64)
    with pytest.raises(ValueError):
        flce.forward(h, w, y)
    with pytest.raises(TypeError):
        flce.forward(h.float(), w, y)


def test_ce_entry_points_fail_closed_on_the_host(lib):
    def fwd(**kw):
        a = dict(z=FAKE, dt=0, lab=FAKE, mask=None, n=64, v=1000, ld=1000, ii=-100, red=0, nlt=0,
                 loss=FAKE, lse=FAKE, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return lib.flce_ce_forward(a["z"], a["dt"], a["lab"], a["mask"], a["n"], a["v"], a["ld"],
                                   a["ii"], a["red"], a["nlt"], a["loss"], a["lse"], a["ws"],
                                   a["wsb"], None)

    def bwd(**kw):
        a = dict(z=FAKE, dt=1, lab=FAKE, mask=None, n=64, v=1000, ld=1000, ii=-100, red=0, nlt=0,
                 g=FAKE, lse=FAKE, dz=FAKE, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return lib.flce_ce_backward(a["z"], a["dt"], a["lab"], a["mask"], a["n"], a["v"], a["ld"],
                                    a["ii"], a["red"], a["nlt"], a["g"], a["lse"], a["dz"], a["ws"],
                                    a["wsb"], None)

    for call in (fwd, bwd):
        for kw in (dict(v=0), dict(ld=999), dict(n=-1), dict(dt=5), dict(red=7),
                   dict(red=1, nlt=3), dict(z=0), dict(lab=0), dict(z=FAKE + 4), dict(lab=FAKE + 2)):
            assert call(**kw) == 1, (call.__name__, kw)
        assert call(ws=0) == 2 and call(wsb=10) == 2
    for kw in (dict(g=0), dict(lse=0), dict(dz=0), dict(dz=FAKE + 8)):
        assert bwd(**kw) == 1, kw
    assert fwd(loss=0) == 1 and fwd(lse=0) == 1
    assert lib.flce_ce_workspace_size(4096) >= 4096 * 20 and lib.flce_ce_workspace_size(-1) == 0
