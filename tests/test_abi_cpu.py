"""The C ABI on a machine without a GPU: libcgl.so loads, exports every function
include/cgl.h declares, and rejects bad arguments on the host before launching
anything (no call here reaches the GPU)."""

import ctypes as C
import os
import re

import pytest
import torch

import combine_get_layout_02_b200 as cgl
from combine_get_layout_02_b200 import build as cbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    cbuild.build()
    return cgl.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "cgl.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(cgl_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("cgl_get_layout", "cgl_dispatch_fp8", "cgl_dispatch_bf16", "cgl_combine",
                 "cgl_layout_workspace_bytes", "cgl_status_string", "cgl_version"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert L.cgl_version() >= 100
    assert L.cgl_status_string(0) == b"ok"
    assert L.cgl_status_string(cgl.ECAPACITY) != L.cgl_status_string(cgl.ERANGE)
    assert L.cgl_status_string(99) == b"unknown status"


def test_workspace_size_rules(L):
    assert L.cgl_layout_workspace_bytes(4096, 8, 256, 64) > 0
    assert L.cgl_layout_workspace_bytes(0, 8, 256, 64) > 0          # empty batch still needs one block
    assert L.cgl_layout_workspace_bytes(4096, 8, 256, 60) == 0      # E % R != 0
    assert L.cgl_layout_workspace_bytes(4096, 33, 256, 64) == 0     # k > 32
    assert L.cgl_layout_workspace_bytes(4096, 8, 2048, 64) == 0     # E > 1024
    assert L.cgl_layout_workspace_bytes(-1, 8, 256, 64) == 0
    assert L.cgl_layout_workspace_bytes(2 ** 28, 8, 256, 64) == 0   # N*k >= 2^31


FAKE = 0x10000  # 64 KiB-aligned, never dereferenced: every call below fails its host checks


def _opts(cap=0, sms=0):
    return C.byref(cgl.Opts(sms, cap))


def test_get_layout_host_errors(L):
    p = FAKE
    ws = L.cgl_layout_workspace_bytes(128, 8, 256, 64)
    args = lambda **kw: dict(dict(idx=p, n=128, k=8, E=256, R=64, opts=_opts(), tpe=p, tpr=p, itr=p,
                                  off=p, mx=p, dst=p, src=p, ws=p, wsb=ws, st=p, stream=None), **kw)

    def call(**kw):
        a = args(**kw)
        return L.cgl_get_layout(a["idx"], a["n"], a["k"], a["E"], a["R"], a["opts"], a["tpe"],
                                a["tpr"], a["itr"], a["off"], a["mx"], a["dst"], a["src"], a["ws"],
                                a["wsb"], a["st"], a["stream"])

    assert call(R=60) == cgl.EINVAL
    assert call(k=0) == cgl.EINVAL
    assert call(wsb=ws - 1) == cgl.EINVAL
    assert call(dst=None) == cgl.EINVAL
    assert call(opts=_opts(cap=-1)) == cgl.EINVAL
    assert call(tpe=None) == cgl.EINVAL
    assert call(dst=p + 2) == cgl.EALIGN
    assert call(itr=p + 4) == cgl.EALIGN
    assert call(ws=p + 8) == cgl.EALIGN


def test_copy_kernels_host_errors(L):
    p = FAKE
    # FP8 dispatch needs H % 128 == 0 and 16-byte aligned rows
    assert L.cgl_dispatch_fp8(p, 16, 7000, 8, p, p, p, 128, None, None, None) == cgl.EINVAL
    assert L.cgl_dispatch_fp8(p, 16, 7168, 0, p, p, p, 128, None, None, None) == cgl.EINVAL
    assert L.cgl_dispatch_fp8(p + 8, 16, 7168, 8, p, p, p, 128, None, None, None) == cgl.EALIGN
    assert L.cgl_dispatch_fp8(p, 16, 7168, 8, p, p + 4, p, 128, None, None, None) == cgl.EALIGN
    assert L.cgl_dispatch_fp8(p, 16, 7168, 8, None, p, p, 128, None, None, None) == cgl.EINVAL
    assert L.cgl_dispatch_fp8(p, 16, 7168, 8, p, p, p, 128, _opts(sms=-1), None, None) == cgl.EINVAL
    # BF16 dispatch: H % 8
    assert L.cgl_dispatch_bf16(p, 16, 7164, 8, p, p, 128, None, None, None) == cgl.EINVAL
    assert L.cgl_dispatch_bf16(p, 16, 7168, 8, p, p + 2, 128, None, None, None) == cgl.EALIGN
    # combine
    assert L.cgl_combine(p, 128, p, p, 16, 7168, 33, p, None, None, None) == cgl.EINVAL
    assert L.cgl_combine(p, -1, p, p, 16, 7168, 8, p, None, None, None) == cgl.EINVAL
    assert L.cgl_combine(p, 128, p, None, 16, 7168, 8, p, None, None, None) == cgl.EINVAL
    assert L.cgl_combine(p, 128, p, p, 16, 7168, 8, p + 8, None, None, None) == cgl.EALIGN
    assert L.cgl_combine(p, 128, p, p + 1, 16, 7168, 8, p, None, None, None) == cgl.EALIGN


def test_binding_refuses_cpu_tensors():
    import torch

    with pytest.raises(TypeError):
        cgl.combine(torch.zeros(8, 8, dtype=torch.bfloat16), torch.zeros(1, 8, dtype=torch.int32),
                    torch.zeros(1, 8))


def test_combine_backward_host_errors(L):
    p = FAKE
    assert L.cgl_combine_backward(p, p, 128, p, p, 16, 7160, 8, p, p, None, None, None) == cgl.EINVAL   # H % 16
    assert L.cgl_combine_backward(p, p, 128, p, p, 16, 16400, 8, p, p, None, None, None) == cgl.EINVAL  # H > 16384
    assert L.cgl_combine_backward(p, p, 128, p, p, 16, 7168, 8, p, None, None, None, None) == cgl.EINVAL
    assert L.cgl_combine_backward(p, p + 8, 128, p, p, 16, 7168, 8, p, p, None, None, None) == cgl.EALIGN
    assert L.cgl_combine_backward(p, p, 128, p, p, 16, 7168, 8, p + 4, p, None, None, None) == cgl.EALIGN


def test_rank_layout_host_errors(L):
    p = FAKE
    ws = L.cgl_layout_workspace_bytes(128, 8, 64, 64)
    call = lambda **kw: L.cgl_get_rank_layout(kw.get("idx", p), 128, 8, 256, kw.get("R", 64), None, p, p, p,
                                              kw.get("dst", p), p, kw.get("ws", p), kw.get("wsb", ws), None, None)
    assert call(R=60) == cgl.EINVAL
    assert call(wsb=ws - 1) == cgl.EINVAL
    assert call(dst=None) == cgl.EINVAL
    assert call(ws=p + 8) == cgl.EALIGN
    assert call(idx=p + 2) == cgl.EALIGN


def test_decode_dispatch_host_errors(L):
    p = FAKE
    o = lambda cap=0, sms=0: C.byref(cgl.Opts(sms, cap))
    args = lambda n=128, k=8, h=7168, x=p, itr=p: (p, n, k, 256, 32, o(), x, h, p, p, itr, p, p, p, p, p, p, None, None)
    assert L.cgl_decode_dispatch_fp8(*args(n=129)) == cgl.EINVAL        # more than one layout block at k = 8
    assert L.cgl_decode_dispatch_fp8(*args(h=7000)) == cgl.EINVAL       # hidden % 128
    assert L.cgl_decode_dispatch_fp8(*args(x=p + 8)) == cgl.EALIGN
    assert L.cgl_decode_dispatch_fp8(*args(itr=p + 4)) == cgl.EALIGN


def test_layout_dispatch_host_errors(L):
    p = FAKE
    ws = L.cgl_layout_dispatch_workspace_bytes(4096, 8, 256, 64)
    assert ws >= L.cgl_layout_workspace_bytes(4096, 8, 256, 64) > 0
    assert L.cgl_layout_dispatch_workspace_bytes(4096, 8, 256, 60) == 0     # E % R != 0
    o = lambda cap=0, sms=0: C.byref(cgl.Opts(sms, cap))

    def args(n=4096, k=8, h=7168, x=p, rs=p, wsb=ws, cap=0, w=p):
        return (p, n, k, 256, 64, o(cap), x, h, p, p, p, p, p, p, p, p, rs, w, wsb, None, None)

    assert L.cgl_layout_dispatch_fp8(*args(h=7000)) == cgl.EINVAL           # hidden % 128
    assert L.cgl_layout_dispatch_fp8(*args(wsb=ws - 1)) == cgl.EINVAL       # workspace too small
    assert L.cgl_layout_dispatch_fp8(*args(k=33)) == cgl.EINVAL
    assert L.cgl_layout_dispatch_fp8(*args(cap=-1)) == cgl.EINVAL
    assert L.cgl_layout_dispatch_fp8(*args(x=p + 8)) == cgl.EALIGN
    assert L.cgl_layout_dispatch_fp8(*args(rs=p + 2)) == cgl.EALIGN
    assert L.cgl_layout_dispatch_fp8(*args(w=p + 8)) == cgl.EALIGN
    assert L.cgl_layout_dispatch_kernel_count(4096, 8, 256, 64, 7000, None) == -1


def test_layout_dispatch_workspace_covers_the_split_path(L):
    # the combined call falls back to cgl_get_layout + cgl_dispatch_fp8, so its
    # workspace must be at least the layout's for every size
    for n in (0, 1, 31, 32, 33, 127, 128, 129, 256, 257, 1000, 4095, 4096, 4097, 8193, 16384, 70000):
        for k, E, R in ((8, 256, 64), (1, 4, 2), (6, 96, 12), (32, 1024, 64)):
            a = L.cgl_layout_dispatch_workspace_bytes(n, k, E, R)
            b = L.cgl_layout_workspace_bytes(n, k, E, R)
            assert a >= b > 0, (n, k, E, R, a, b)


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    # no CPU or PyTorch fallback: a missing libcgl.so is an error at the first call
    monkeypatch.setattr(cgl, "_lib", None)
    monkeypatch.setattr(cgl, "LIB_PATH", str(tmp_path / "libcgl.so"))
    with pytest.raises(RuntimeError, match="not built"):
        cgl.layout_workspace_bytes(4096, 8, 256, 64)


def test_noalloc_limits_at_their_exact_boundaries(L):
    """cgl_get_layout_noalloc refuses exactly the sizes past its two limits.

    A refused size returns CGL_EINVAL before anything else.  An accepted size
    goes on to the scratch lookup (CGL_ECUDA without a device) or, where a
    device exists, to cgl_get_layout's checks, which refuse the misaligned
    is_token_in_rank passed here (CGL_EALIGN): nothing is launched either way."""
    f = L.cgl_get_layout_noalloc
    P, I64, I = C.c_void_p, C.c_int64, C.c_int
    f.argtypes = [P, I64, I, I, I, C.POINTER(cgl.Opts), P, P, P, P, P, P, P, P, P]
    f.restype = I
    p = FAKE

    def call(n, k, E, R):
        return f(p, n, k, E, R, None, p, p, p + 2, p, p, p, p, p, None)

    accepted = (cgl.ECUDA, cgl.EALIGN)
    # scratch: 512 KiB holds the per-block counts of exactly 52,096 tokens at top-8, E=256, R=64
    assert L.cgl_layout_workspace_bytes(52096, 8, 256, 64) == 512 * 1024
    assert L.cgl_layout_workspace_bytes(52097, 8, 256, 64) > 512 * 1024
    assert call(52096, 8, 256, 64) in accepted
    assert call(52097, 8, 256, 64) == cgl.EINVAL
    # shared memory: 12 E + R + T ceil(R / 32) <= 9984 with T = min(256, 1024 / k)
    # (R = 1, k = 1: T = 256, so E <= 810; R = 64: E <= 784, the next multiple of 64 is 832)
    assert call(1000, 1, 810, 1) in accepted
    assert call(1000, 1, 811, 1) == cgl.EINVAL
    assert call(1000, 1, 768, 64) in accepted
    assert call(1000, 1, 832, 64) == cgl.EINVAL
    # k = 8, R = 32: T = 128 tokens per block, 12 E + 32 + 128 <= 9984 -> E <= 818 (800 and 832 are multiples of 32)
    assert call(1000, 8, 800, 32) in accepted
    assert call(1000, 8, 832, 32) == cgl.EINVAL


def test_opts_flags_unknown_bits_refused(L):
    """cgl_opts.flags: CGL_OPT_UE8M0_SCALES is the only defined bit; any other bit is
    refused with CGL_EINVAL before anything is launched (fake pointers never used)."""
    src = open(os.path.join(ROOT, "include", "cgl.h")).read()
    assert "#define CGL_OPT_UE8M0_SCALES 1u" in src and "uint32_t flags;" in src
    assert L.cgl_version() >= 200
    p = FAKE
    bad = C.byref(cgl.Opts(0, 0, 2))
    assert L.cgl_dispatch_fp8(p, 128, 7168, 8, p, p, p, 1024, bad, p, None) == cgl.EINVAL
    assert L.cgl_dispatch_bf16(p, 128, 7168, 8, p, p, 1024, bad, p, None) == cgl.EINVAL
    assert L.cgl_combine(p, 1024, p, p, 128, 7168, 8, p, bad, p, None) == cgl.EINVAL
    ws = L.cgl_layout_workspace_bytes(128, 8, 256, 64)
    assert L.cgl_get_layout(p, 128, 8, 256, 64, bad, p, p, p, p, p, p, p, p, ws, p, None) == cgl.EINVAL
    assert L.cgl_decode_dispatch_fp8(p, 128, 8, 256, 32, bad, p, 7168, p, p, p, p, p, p, p, p, p, p, None) \
        == cgl.EINVAL
    wsd = L.cgl_layout_dispatch_workspace_bytes(4096, 8, 256, 64)
    assert L.cgl_layout_dispatch_fp8(p, 4096, 8, 256, 64, bad, p, 7168, p, p, p, p, p, p, p, p, p, p, wsd, p,
                                     None) == cgl.EINVAL
    # the defined bit passes the flag check (then fails on a misaligned pointer, as without it)
    ok = C.byref(cgl.Opts(0, 0, cgl.OPT_UE8M0_SCALES))
    assert L.cgl_dispatch_fp8(p + 8, 128, 7168, 8, p, p, p, 1024, ok, p, None) == cgl.EALIGN


def test_opts_scratch_alignment_and_layout(L):
    """cgl_opts.scratch (library 0.3.0): a device pointer after flags; the dispatch
    calls refuse one that is not 8-byte aligned before launching anything (fake
    pointers never used); NULL keeps the fixed token order."""
    src = open(os.path.join(ROOT, "include", "cgl.h")).read()
    assert "void *scratch;" in src and L.cgl_version() >= 300
    assert [f[0] for f in cgl.Opts._fields_] == ["num_sms", "capacity", "flags", "scratch"]
    assert C.sizeof(cgl.Opts) == 24 and cgl.Opts.scratch.offset == 16
    p = FAKE
    mis = C.byref(cgl.Opts(0, 0, 0, p + 4))
    assert L.cgl_dispatch_fp8(p, 128, 7168, 8, p, p, p, 1024, mis, p, None) == cgl.EALIGN
    assert L.cgl_dispatch_bf16(p, 128, 7168, 8, p, p, 1024, mis, p, None) == cgl.EALIGN
    with pytest.raises(cgl.CglError):
        cgl._opts(scratch=torch.zeros(2, dtype=torch.int64))          # a host tensor is refused
