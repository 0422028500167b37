"""GPU parity for tensors with arbitrary strides (fa_fwd_ex / fa_bwd_ex
through the Python binding): [B, N, H, d] ("sequence before
head"), slices of a fused [B, N, 3, H, d] QKV projection, rows padded past
d (heads and batches still merge into one tensor-map index, but the plain
accesses need the strides) and a mix of these in one call.  The
kernels read and write the same elements as for contiguous tensors, so the
forward results and dK / dV are bit-identical to the contiguous run; dQ (whose
fp32 reduction order varies between runs) and everything else are checked
against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._parity import check_fwd, check_grad, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import exact_attention_115_b200 as fa
    fa.lib()
    return fa


def bshd(t):
    """The same values laid out [B, N, H, d], viewed back as [B, H, N, d]."""
    return t.transpose(1, 2).contiguous().transpose(1, 2)


def padded(t, pad=64):
    """The same values in a [B, H, N, d + pad] buffer, sliced back to d."""
    buf = torch.zeros(*t.shape[:3], t.shape[3] + pad, dtype=t.dtype, device=t.device)
    buf[..., : t.shape[3]] = t
    return buf[..., : t.shape[3]]


LAYOUTS = {"bshd": bshd, "padded": padded}


def fused_qkv(q, k, v):
    """Q, K, V as slices of one [B, N, 3, H, d] buffer (Nq == Nk)."""
    buf = torch.stack([x.transpose(1, 2) for x in (q, k, v)], dim=2).contiguous()
    return tuple(buf[:, :, i].transpose(1, 2) for i in range(3))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [200, 385])
@pytest.mark.parametrize("how", ["bshd", "fused", "padded", "mixed"])
def test_strided_forward(fa, how, N, causal, d):
    B, H = 2, 3
    q, k, v, _ = W.make_tensors(B, H, N, N, d, "bf16", seed=7, device="cuda", with_grad=False)
    scale = 1 / math.sqrt(d)
    O0, L0 = fa.forward(q, k, v, causal=causal, scale=scale)
    if how == "fused":
        qs, ks, vs = fused_qkv(q, k, v)
    elif how == "mixed":
        qs, ks, vs = bshd(q), padded(k), v
    else:
        qs, ks, vs = (LAYOUTS[how](t) for t in (q, k, v))
    assert not qs.is_contiguous() or not ks.is_contiguous()
    # O written straight into a [B, N, H, d] (or row-padded) buffer
    out = padded(torch.empty_like(q)) if how == "padded" else bshd(torch.empty_like(q))
    O1, L1 = fa.forward(qs, ks, vs, causal=causal, scale=scale, out=out)
    assert fa.status() == fa.FA_OK
    assert O1.data_ptr() == out.data_ptr()
    assert torch.equal(O1, O0) and torch.equal(L1, L0)
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, causal)
    check_fwd(O1, L1, O_ref, L_ref, f"{how} N{N} d{d} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(200, 200), (130, 300)])
@pytest.mark.parametrize("how", ["bshd", "padded"])
def test_strided_backward(fa, how, Nq, Nk, causal, d):
    B, H = 2, 3
    q, k, v, do = W.make_tensors(B, H, Nq, Nk, d, "bf16", seed=11, device="cuda", with_grad=True)
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(q, k, v, causal=causal, scale=scale)
    dq0, dk0, dv0 = fa.backward(q, k, v, O, do, L, causal=causal, scale=scale)
    lay = LAYOUTS[how]
    ins = [lay(t) for t in (q, k, v, O, do)]
    outs = [lay(torch.empty_like(t)) for t in (q, k, v)]
    dq1, dk1, dv1 = fa.backward(*ins, L, causal=causal, scale=scale, dq=outs[0], dk=outs[1],
                                dv=outs[2])
    assert fa.status() == fa.FA_OK
    assert torch.equal(dk1, dk0) and torch.equal(dv1, dv0)
    dQ_ref, dK_ref, dV_ref, _ = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal)
    what = f"{how} Nq{Nq} Nk{Nk} d{d} causal={causal}"
    check_grad(dq1, dQ_ref, "dQ", what)
    check_grad(dk1, dK_ref, "dK", what)
    check_grad(dv1, dV_ref, "dV", what)
    # dQ agrees with the contiguous run up to the reduction order
    assert float((dq1.float() - dq0.float()).abs().max()) <= 1e-2 * float(dq0.float().abs().max()) + 1e-6
