"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every function include/fa.h declares, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

import exact_attention_115_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

FAKE = 0x10000  # a 16-byte aligned non-null value; never dereferenced on these paths


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from exact_attention_115_b200 import build
    build.build()
    return fa.lib()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "fa_fwd" in names and "fa_bwd" in names and "fa_decode" in names
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
        assert n in fa.SIGNATURES, f"{n} has no ctypes signature in the binding"


def test_version(lib):
    assert "sm_100a" in fa.version()


def fwd(lib, **kw):
    a = dict(Q=FAKE, K=FAKE, V=FAKE, O=FAKE, L=FAKE, B=1, H=1, Nq=128, Nk=128, d=64, causal=0,
             scale=0.125, dtype=fa.FA_BF16, stream=None)
    a.update(kw)
    return lib.fa_fwd(a["Q"], a["K"], a["V"], a["O"], a["L"], a["B"], a["H"], a["Nq"], a["Nk"],
                      a["d"], a["causal"], a["scale"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(Q=None), fa.FA_ERR_INVALID),
    (dict(L=None), fa.FA_ERR_INVALID),
    (dict(K=FAKE + 2), fa.FA_ERR_INVALID),
    (dict(B=0), fa.FA_ERR_INVALID),
    (dict(Nq=0), fa.FA_ERR_INVALID),
    (dict(Nk=-1), fa.FA_ERR_INVALID),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID),
    (dict(scale=0.0), fa.FA_ERR_INVALID),
    (dict(dtype=7), fa.FA_ERR_INVALID),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
    (dict(dtype=fa.FA_FP32, d=128), fa.FA_ERR_UNSUPPORTED),
    (dict(causal=1, Nq=200, Nk=100), fa.FA_ERR_UNSUPPORTED),
    (dict(H=70000), fa.FA_ERR_UNSUPPORTED),
])
def test_fwd_rejects(lib, kw, code):
    assert fwd(lib, **kw) == code


def test_bwd_workspace_query(lib):
    n = lib.fa_bwd_workspace_bytes(2, 3, 100, 200, 64, fa.FA_BF16)
    # D (fp32 per padded row) + fp32 dQ accumulator (padded rows × d), 256-aligned pieces
    rows = 128
    assert n >= 2 * 3 * rows * 4 + 2 * 3 * rows * 64 * 4
    assert lib.fa_bwd_workspace_bytes(0, 3, 100, 200, 64, fa.FA_BF16) == 0
    assert lib.fa_bwd_workspace_bytes(1, 1, 100, 200, 96, fa.FA_BF16) == 0


def test_bwd_dq_modes_change_workspace(lib):
    prev = lib.fa_set_bwd_dq_mode(2)
    prev_g = lib.fa_set_bwd_dq_groups(3)
    try:
        n2 = lib.fa_bwd_workspace_bytes(1, 1, 1024, 1024, 64, fa.FA_BF16)
        lib.fa_set_bwd_dq_mode(1)
        n1 = lib.fa_bwd_workspace_bytes(1, 1, 1024, 1024, 64, fa.FA_BF16)
        assert lib.fa_set_bwd_dq_mode(3) == 1
        n3 = lib.fa_bwd_workspace_bytes(1, 1, 1024, 1024, 64, fa.FA_BF16)
        acc = 1024 * 64 * 4  # one fp32 dQ buffer
        assert n2 - n1 == 7 * acc  # 8 K/V blocks of partial buffers vs one accumulator
        assert n3 - n1 == 2 * acc  # 3 accumulators vs one
        assert lib.fa_set_bwd_dq_groups(5) == 3
        assert lib.fa_bwd_workspace_bytes(1, 1, 1024, 1024, 64, fa.FA_BF16) - n1 == 4 * acc
        for bad in (0, 17, -1):
            assert lib.fa_set_bwd_dq_groups(bad) == fa.FA_ERR_INVALID
        assert lib.fa_set_bwd_dq_mode(4) == fa.FA_ERR_INVALID
        assert lib.fa_set_bwd_dq_mode(-1) == fa.FA_ERR_INVALID
    finally:
        lib.fa_set_bwd_dq_mode(prev)
        lib.fa_set_bwd_dq_groups(prev_g)


def bwd(lib, ws=FAKE, ws_bytes=1 << 40, **kw):
    a = dict(B=1, H=1, Nq=128, Nk=128, d=64, causal=0, scale=0.125, dtype=fa.FA_BF16)
    a.update(kw)
    return lib.fa_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, a["B"], a["H"],
                      a["Nq"], a["Nk"], a["d"], a["causal"], a["scale"], a["dtype"], ws, ws_bytes,
                      None)


def test_bwd_rejects(lib):
    assert bwd(lib, d=80) == fa.FA_ERR_UNSUPPORTED
    assert bwd(lib, Nq=0) == fa.FA_ERR_INVALID
    assert bwd(lib, causal=1, Nq=256, Nk=128) == fa.FA_ERR_UNSUPPORTED
    assert bwd(lib, ws=None) == fa.FA_ERR_WORKSPACE
    assert bwd(lib, ws=FAKE + 16) == fa.FA_ERR_WORKSPACE  # not 256-aligned
    need = lib.fa_bwd_workspace_bytes(1, 1, 128, 128, 64, fa.FA_BF16)
    assert bwd(lib, ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE


def test_decode_rejects(lib):
    def dec(ws=FAKE, ws_bytes=1 << 40, **kw):
        a = dict(B=2, H=2, Nk=1000, d=128, scale=0.1, dtype=fa.FA_BF16, splits=0)
        a.update(kw)
        return lib.fa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, a["B"], a["H"], a["Nk"], a["d"],
                             a["scale"], a["dtype"], a["splits"], ws, ws_bytes, None)
    assert dec(Nk=0) == fa.FA_ERR_INVALID
    assert dec(d=32) == fa.FA_ERR_UNSUPPORTED
    assert dec(dtype=fa.FA_FP32) == fa.FA_ERR_UNSUPPORTED
    assert dec(splits=-2) == fa.FA_ERR_INVALID
    assert dec(ws=None) == fa.FA_ERR_WORKSPACE
    need = lib.fa_decode_workspace_bytes(2, 2, 1000, 128, 0)
    assert need > 0
    assert dec(ws_bytes=need - 1) == fa.FA_ERR_WORKSPACE
    # explicit split counts are clamped to the number of keys
    assert lib.fa_decode_workspace_bytes(1, 1, 5, 64, 100) <= lib.fa_decode_workspace_bytes(1, 1, 5000, 64, 100)


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward(q, q, q)
    with pytest.raises(ValueError):
        fa.decode(q[:, :, :1], q, q)


def test_selftest_rejects_limits_out_of_range(lib):
    # validated before anything is enqueued, so no GPU is needed
    assert lib.fa_selftest_wait_timeout(0, None) == fa.FA_ERR_INVALID
    assert lib.fa_selftest_wait_timeout(1000001, None) == fa.FA_ERR_INVALID


def test_ex_entry_points_validate_layouts(lib):
    L = fa.Layout
    good, bad = L(2 * 64 * 64, 64 * 64, 64), L(2 * 64 * 64, 64 * 64, 3)  # 3 elements: not 16-byte aligned
    P = 4096  # any 16-byte-aligned non-null address: the call returns before touching memory
    args = (1, 2, 64, 64, 64, 0, 0.125)
    r = ctypes.byref
    assert lib.fa_fwd_ex(P, P, P, P, P, r(bad), r(good), r(good), r(good), *args, fa.FA_BF16,
                         None, None, None, None, None) == fa.FA_ERR_INVALID
    assert lib.fa_fwd_ex(P, P, P, P, P, None, r(good), r(good), r(good), *args, fa.FA_BF16,
                         None, None, None, None, None) == fa.FA_ERR_INVALID
    # fp32 reads contiguous tensors only
    nc = L(2 * 64 * 64, 64, 2 * 64)
    assert lib.fa_fwd_ex(P, P, P, P, P, r(nc), r(good), r(good), r(good), *args, fa.FA_FP32,
                         None, None, None, None, None) == fa.FA_ERR_UNSUPPORTED
    lays = [r(good)] * 8
    assert lib.fa_bwd_ex(P, P, P, P, P, P, P, P, P, r(bad), *lays[1:], *args, fa.FA_BF16, None, None,
                         None, None, P, 1 << 30, None) == fa.FA_ERR_INVALID


@pytest.mark.parametrize("p", [-0.1, 1.0, 1.5, float("nan"), 0.999])
def test_ex_entry_points_reject_bad_dropout(lib, p):
    """A probability outside [0, 1), or one that rounds to keeping nothing
    (T = round((1 - p)·256) = 0), is invalid; checked before any launch."""
    good = fa.Layout(2 * 64 * 64, 64 * 64, 64)
    P = 4096
    args = (1, 2, 64, 64, 64, 0, 0.125)
    r = ctypes.byref
    dr = fa.Dropout(p, 1, 0)
    assert lib.fa_fwd_ex(P, P, P, P, P, *[r(good)] * 4, *args, fa.FA_BF16, r(dr), None, None, None,
                         None) == fa.FA_ERR_INVALID
    assert lib.fa_bwd_ex(P, P, P, P, P, P, P, P, P, *[r(good)] * 8, *args, fa.FA_BF16, r(dr), None,
                         None, None, P, 1 << 30, None) == fa.FA_ERR_INVALID


def test_fp32_has_no_dropout(lib):
    good = fa.Layout(2 * 64 * 64, 64 * 64, 64)
    P = 4096
    args = (1, 2, 64, 64, 64, 0, 0.125)
    r = ctypes.byref
    dr = fa.Dropout(0.1, 1, 0)
    assert lib.fa_fwd_ex(P, P, P, P, P, *[r(good)] * 4, *args, fa.FA_FP32, r(dr), None, None, None,
                         None) == fa.FA_ERR_UNSUPPORTED


def test_key_padding_pointer_checks(lib):
    good = fa.Layout(2 * 64 * 64, 64 * 64, 64)
    P = 4096
    args = (1, 2, 64, 64, 64, 0, 0.125)
    r = ctypes.byref
    lays4, lays8 = [r(good)] * 4, [r(good)] * 8
    # a misaligned length array is invalid; fp32 has no key padding
    assert lib.fa_fwd_ex(P, P, P, P, P, *lays4, *args, fa.FA_BF16, None, P + 2, None, None,
                         None) == fa.FA_ERR_INVALID
    assert lib.fa_bwd_ex(P, P, P, P, P, P, P, P, P, *lays8, *args, fa.FA_BF16, None, P + 2, None,
                         None, P, 1 << 30, None) == fa.FA_ERR_INVALID
    assert lib.fa_fwd_ex(P, P, P, P, P, *lays4, *args, fa.FA_FP32, None, P, None, None,
                         None) == fa.FA_ERR_UNSUPPORTED


def test_bias_pointer_and_layout_checks(lib):
    good = fa.Layout(2 * 64 * 64, 64 * 64, 64)
    P = 4096
    args = (1, 2, 64, 64, 64, 0, 0.125)
    r = ctypes.byref
    lays4 = [r(good)] * 4
    bl_ok, bl_bad = fa.Layout(0, 64 * 64, 64), fa.Layout(0, 64 * 64, 60)  # 60 keys: not 16-byte rows
    assert lib.fa_fwd_ex(P, P, P, P, P, *lays4, *args, fa.FA_BF16, None, None, P + 8, r(bl_ok),
                         None) == fa.FA_ERR_INVALID
    assert lib.fa_fwd_ex(P, P, P, P, P, *lays4, *args, fa.FA_BF16, None, None, P, r(bl_bad),
                         None) == fa.FA_ERR_INVALID
    assert lib.fa_fwd_ex(P, P, P, P, P, *lays4, *args, fa.FA_BF16, None, None, P, None,
                         None) == fa.FA_ERR_INVALID
    assert lib.fa_fwd_ex(P, P, P, P, P, *lays4, *args, fa.FA_FP32, None, None, P, r(bl_ok),
                         None) == fa.FA_ERR_UNSUPPORTED


def test_decode_ex_checks_the_length_pointer(lib):
    P = 4096
    # a misaligned key-length array is invalid (checked before any launch)
    assert lib.fa_decode_ex(P, P, P, P, P, 1, 2, 64, 64, 0.125, fa.FA_BF16, 0, P + 2, P, 1 << 20,
                            None) == fa.FA_ERR_INVALID
    assert lib.fa_decode_ex(P, P, P, P, P, 1, 2, 64, 64, 0.125, fa.FA_FP32, 0, None, P, 1 << 20,
                            None) == fa.FA_ERR_UNSUPPORTED


def test_attention_rejects_a_bias_that_wants_a_gradient():
    """The bias is an input constant; asking autograd for its gradient fails
    loudly instead of silently returning none (checked before any launch)."""
    import torch
    b = torch.zeros(1, 1, 4, 8, requires_grad=True)
    q = torch.zeros(1, 1, 4, 64)
    with pytest.raises(ValueError):
        fa.attention(q, q, q, bias=b)


def test_cuda_failure_is_recorded(lib):
    """Without a GPU, fa_status's stream synchronisation fails: FA_ERR_CUDA,
    and fa_last_cuda_error names the runtime error behind it."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("needs a machine without a usable GPU")
    assert lib.fa_status(None) == fa.FA_ERR_CUDA
    code = lib.fa_last_cuda_error()
    assert 0 < code < 100000
