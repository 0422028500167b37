"""Full-size parity of the three large workloads against the fp64 oracle,
every output element compared (call path: Python binding -> C ABI ->
sm_100a kernels).

* B8 H16 N2048 d128 causal: O and L of all 128 heads; dQ, dK, dV of all
  128 heads, with each dQ strategy (one fp32 accumulator, per-K/V-block
  partials).
* B1 H32 N16384 d128 causal, Q×3: O and L of all 32 heads; dQ, dK, dV of
  the whole heads 0, 13 and 31 (every query and key row), in the same call
  that computes all 32.
* decode B32 H32 Nk32768 d128: O and L of all 1024 heads.

Every output buffer is filled with NaN before the call, so an element a
kernel never wrote fails the finiteness check.  The bounds are the stated
ones (``tests/_parity.py``): the mean-abs bound on O is taken over the whole
tensor, and each gradient bound is relative to the largest reference value
of the whole compared tensor.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._parity import check_fwd, check_grad, f64, nan_like, oracle_map

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import exact_attention_115_b200 as fa
    fa.lib()
    return fa


def _forward_canary(fa, q, k, v, w):
    B, H, Nq, d = q.shape
    out = torch.full((B, H, Nq, d), float("nan"), dtype=q.dtype, device=q.device)
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=q.device)
    O, L = fa.forward(q, k, v, causal=w.causal, scale=w.scale, out=out, lse=lse)
    assert fa.status() == fa.FA_OK
    assert torch.isfinite(O.float()).all(), "O has unwritten (NaN) or non-finite elements"
    assert torch.isfinite(L).all(), "L has unwritten (NaN) or non-finite elements"
    return O, L


def _backward_canary(fa, q, k, v, O, do, L, w):
    dq, dk, dv = nan_like(q), nan_like(k), nan_like(v)
    fa.backward(q, k, v, O, do, L, causal=w.causal, scale=w.scale, dq=dq, dk=dk, dv=dv)
    assert fa.status() == fa.FA_OK
    for name, g in (("dQ", dq), ("dK", dk), ("dV", dv)):
        assert torch.isfinite(g.float()).all(), f"{name} has unwritten (NaN) or non-finite elements"
    return dq, dk, dv


# ---------------------------------------------------------------- B8 H16 N2048 d128 causal
@pytest.fixture(scope="module")
def causal_2k(fa):
    """Inputs on the GPU and the oracle's O, L, dQ, dK, dV for every head."""
    w = W.CAUSAL_2K
    q, k, v, do = W.make_inputs(w, device="cuda")
    hq, hk, hv, hdo = (f64(x) for x in (q, k, v, do))

    def head(bh):
        b, h = bh
        O, L = oracle.head_forward(hq[b, h], hk[b, h], hv[b, h], w.scale, True)
        dq, dk, dv, _ = oracle.head_backward(hq[b, h], hk[b, h], hv[b, h], hdo[b, h], w.scale,
                                             True)
        return O, L, dq, dk, dv

    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    res = oracle_map(head, heads)
    ref = [np.stack([r[i] for r in res]).reshape((w.B, w.H) + res[0][i].shape) for i in range(5)]
    return w, (q, k, v, do), ref


def test_causal_2k_forward_every_element(fa, causal_2k):
    w, (q, k, v, _), (O_ref, L_ref, *_) = causal_2k
    O, L = _forward_canary(fa, q, k, v, w)
    check_fwd(O, L, O_ref, L_ref, f"{w.name}, all 128 heads")


@pytest.mark.parametrize("mode", [1, 2, 3], ids=["dq_reduce_add", "dq_partials", "dq_grouped4"])
def test_causal_2k_backward_every_element(fa, causal_2k, mode):
    w, (q, k, v, do), (_, _, dq_ref, dk_ref, dv_ref) = causal_2k
    prev = fa.set_bwd_dq_mode(mode)
    prev_g = fa.set_bwd_dq_groups(4)
    try:
        O, L = _forward_canary(fa, q, k, v, w)
        dq, dk, dv = _backward_canary(fa, q, k, v, O, do, L, w)
    finally:
        fa.set_bwd_dq_mode(prev)
        fa.set_bwd_dq_groups(prev_g)
    what = f"{w.name}, all 128 heads, dq mode {mode}"
    for g, r, n in ((dq, dq_ref, "dQ"), (dk, dk_ref, "dK"), (dv, dv_ref, "dV")):
        check_grad(g, r, n, what)


# ---------------------------------------------------------------- B1 H32 N16384 d128 causal, Q×3
LONG_BWD_HEADS = (0, 13, 31)


def test_long_16k_every_element(fa):
    """O and L of all 32 heads; the gradients of whole heads 0, 13 and 31."""
    w = W.LONG_16K
    q, k, v, do = W.make_inputs(w, device="cuda")
    O, L = _forward_canary(fa, q, k, v, w)
    dq, dk, dv = _backward_canary(fa, q, k, v, O, do, L, w)
    hq, hk, hv, hdo = (f64(x[0]) for x in (q, k, v, do))

    fwd = oracle_map(lambda h: oracle.head_forward(hq[h], hk[h], hv[h], w.scale, True),
                     list(range(w.H)))
    O_ref = np.stack([r[0] for r in fwd])[None]
    L_ref = np.stack([r[1] for r in fwd])[None]
    check_fwd(O, L, O_ref, L_ref, f"{w.name}, all 32 heads")

    bwd = oracle_map(lambda h: oracle.head_backward(hq[h], hk[h], hv[h], hdo[h], w.scale, True),
                     list(LONG_BWD_HEADS))
    for h, (dq_ref, dk_ref, dv_ref, _) in zip(LONG_BWD_HEADS, bwd):
        what = f"{w.name}, head {h}, every row"
        check_grad(dq[0, h], dq_ref, "dQ", what)
        check_grad(dk[0, h], dk_ref, "dK", what)
        check_grad(dv[0, h], dv_ref, "dV", what)

    # the grouped dQ strategy (8 accumulators) on the same inputs
    prev, prev_g = fa.set_bwd_dq_mode(3), fa.set_bwd_dq_groups(8)
    try:
        dq, dk, dv = _backward_canary(fa, q, k, v, O, do, L, w)
    finally:
        fa.set_bwd_dq_mode(prev)
        fa.set_bwd_dq_groups(prev_g)
    for h, (dq_ref, dk_ref, dv_ref, _) in zip(LONG_BWD_HEADS, bwd):
        what = f"{w.name}, head {h}, every row, dq mode 3 (G = 8)"
        check_grad(dq[0, h], dq_ref, "dQ", what)
        check_grad(dk[0, h], dk_ref, "dK", what)
        check_grad(dv[0, h], dv_ref, "dV", what)


# ---------------------------------------------------------------- decode B32 H32 Nk32768 d128
def test_decode_every_head(fa):
    w = W.DECODE_32K
    q, k, v, _ = W.make_inputs(w, device="cuda", with_grad=False)
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.H, 1), float("nan"), dtype=torch.float32, device="cuda")
    O, L = fa.decode(q, k, v, scale=w.scale, out=out, lse=lse)
    assert fa.status() == fa.FA_OK
    assert torch.isfinite(O.float()).all() and torch.isfinite(L).all()
    O_ref = np.empty((w.B, w.H, 1, w.d))
    L_ref = np.empty((w.B, w.H, 1))
    hq = f64(q)
    for b in range(w.B):  # one batch element of K and V on the host at a time
        hk, hv = f64(k[b]), f64(v[b])
        res = oracle_map(lambda h: oracle.head_forward(hq[b, h], hk[h], hv[h], w.scale, False),
                         list(range(w.H)))
        for h, (o, l) in enumerate(res):
            O_ref[b, h], L_ref[b, h] = o, l
    check_fwd(O, L, O_ref, L_ref, f"{w.name}, all 1024 heads")
