"""The debug build (libfa_b200_debug.so: every kernel compiled with FA_DEBUG
index checks on its plain global accesses and TMA coordinates) over the
library's call matrix: no check fires (fa_status stays FA_OK, never
FA_ERR_BOUNDS), and the results match the fp64 oracle (small cases) or the
release library (full size).  compute-sanitizer is not available for these
runs; the checks stand in for its memory checker."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._parity import check_fwd, check_grad, f64

pytestmark = pytest.mark.gpu


class Libs:
    """The binding, switchable between the debug and the release library."""

    def __init__(self, fa, debug, release):
        self.fa, self.debug, self.release = fa, debug, release

    def use(self, which):
        self.fa._lib = self.debug if which == "debug" else self.release


@pytest.fixture(scope="module")
def libs():
    import exact_attention_115_b200 as fa
    from exact_attention_115_b200 import build

    path = build.build(debug=True)  # no-op when already built
    release = fa.lib()
    h = ctypes.CDLL(path)
    for name, (res, args) in fa.SIGNATURES.items():
        f = getattr(h, name)
        f.restype = res
        f.argtypes = args
    L = Libs(fa, h, release)
    L.use("debug")
    assert "debug" in fa.version()
    try:
        yield L
    finally:
        L.use("release")


@pytest.fixture
def fa_debug(libs):
    libs.use("debug")
    yield libs.fa
    libs.use("release")


def _ok(fa):
    st = fa.status()
    assert st == fa.FA_OK, (f"{fa.STATUS_NAMES.get(st, st)}; site "
                            f"{fa.lib().fa_last_timeout_site()}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (17, 17), (129, 129), (257, 513), (1000, 1000)])
def test_small_shapes_no_check_fires(fa_debug, d, causal, Nq, Nk):
    fa = fa_debug
    if causal and Nq > Nk:
        pytest.skip("causal requires Nq <= Nk")
    q, k, v, do = W.make_tensors(2, 3, Nq, Nk, d, "bf16", seed=Nq + d, device="cuda")
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa.backward(q, k, v, O, do, L, causal=causal, scale=scale)
    _ok(fa)
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, causal)
    check_fwd(O, L, O_ref, L_ref, "debug build")
    g = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal)
    for got, ref, n in zip((dq, dk, dv), g[:3], ("dQ", "dK", "dV")):
        check_grad(got, ref, n, "debug build")


def test_other_paths_no_check_fires(fa_debug):
    fa = fa_debug
    # fp16 and fp32
    for dt, d in (("fp16", 128), ("fp32", 64)):
        q, k, v, do = W.make_tensors(1, 2, 200, 300, d, dt, seed=5, device="cuda")
        O, L = fa.forward(q, k, v, causal=True)
        fa.backward(q, k, v, O, do, L, causal=True)
        _ok(fa)
    # a [B, N, H, d] layout with dropout, key padding and a head-shared bias
    B, H, N, d = 2, 2, 300, 128
    q, k, v, do = W.make_tensors(B, H, N, N, d, "bf16", seed=6, device="cuda")
    bshd = lambda t: t.transpose(1, 2).contiguous().transpose(1, 2)  # noqa: E731
    kv_len = torch.tensor([300, 170], dtype=torch.int32, device="cuda")
    # bias rows start on 16-byte boundaries: a row stride of 304 elements
    bias = torch.randn(1, H, N, 304, device="cuda").to(torch.bfloat16)[..., :N]
    for kw in (dict(dropout_p=0.2, seed=3, offset=1), dict(kv_len=kv_len), dict(bias=bias)):
        O, L = fa.forward(bshd(q), bshd(k), bshd(v), causal=True, **kw)
        fa.backward(bshd(q), bshd(k), bshd(v), O, bshd(do), L, causal=True, **kw)
        _ok(fa)
    # decode: automatic and explicit part counts, key padding
    q, k, v, _ = W.make_tensors(3, 4, 1, 5000, 128, "bf16", seed=7, device="cuda", with_grad=False)
    for splits in (0, 1, 7):
        fa.decode(q, k, v, num_splits=splits)
        _ok(fa)
    fa.decode(q, k, v, kv_len=torch.tensor([5000, 10, 0], dtype=torch.int32, device="cuda"))
    _ok(fa)


@pytest.mark.parametrize("mode", [1, 2], ids=["dq_reduce_add", "dq_partials"])
def test_full_size_matches_release(libs, mode):
    """B8 H16 N2048 d128 causal through the debug build: no check fires, and
    the outputs equal the release build's within the stated bounds (the
    kernels are the same code plus checks; dQ's reduction order may differ)."""
    fa = libs.fa
    w = W.CAUSAL_2K
    q, k, v, do = W.make_inputs(w, device="cuda")
    out = {}
    try:
        for which in ("debug", "release"):
            libs.use(which)
            prev = fa.set_bwd_dq_mode(mode)
            O, L = fa.forward(q, k, v, causal=True)
            grads = fa.backward(q, k, v, O, do, L, causal=True)
            _ok(fa)
            fa.set_bwd_dq_mode(prev)
            out[which] = (O, L, *grads)
    finally:
        libs.use("release")
    O, L, dq, dk, dv = out["debug"]
    O_r, L_r, dq_r, dk_r, dv_r = out["release"]
    assert torch.equal(O, O_r) and torch.equal(L, L_r)
    for got, ref, n in ((dq, dq_r, "dQ"), (dk, dk_r, "dK"), (dv, dv_r, "dV")):
        check_grad(got, f64(ref), n, "debug vs release build")
