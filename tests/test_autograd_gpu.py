"""The autograd wrapper (exact_attention_115_b200.attention) against the
direct forward/backward calls and the fp64 oracle."""
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


@pytest.mark.parametrize("causal", [False, True])
def test_autograd_matches_direct_calls(fa, causal):
    q, k, v, do = W.make_tensors(2, 3, 200, 200, 128, "bf16", seed=61, device="cuda")
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    O = fa.attention(qa, ka, va, causal=causal)
    O.backward(do)
    O0, L0 = fa.forward(q, k, v, causal=causal)
    dq0, dk0, dv0 = fa.backward(q, k, v, O0, do, L0, causal=causal)
    assert fa.status() == fa.FA_OK
    assert torch.equal(O.detach(), O0)
    assert torch.equal(ka.grad, dk0) and torch.equal(va.grad, dv0)
    # dQ's fp32 reduction order may differ between runs
    assert float((qa.grad.float() - dq0.float()).abs().max()) <= 1e-2 * float(dq0.float().abs().max())


def test_autograd_dropout_padding_in_a_graph(fa):
    """attention() inside a small graph (a loss of O) with dropout and key
    padding: the gradients equal the oracle's for the same mask."""
    B, H, N, d = 2, 2, 160, 64
    q, k, v, _ = W.make_tensors(B, H, N, N, d, "bf16", seed=62, device="cuda", with_grad=False)
    w = torch.randn(B, H, N, d, device="cuda", dtype=torch.float32)
    kvl = torch.tensor([160, 90], dtype=torch.int32, device="cuda")
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    O = fa.attention(qa, ka, va, causal=True, dropout_p=0.1, seed=77, offset=2, kv_len=kvl)
    loss = (O.float() * w).sum()
    loss.backward()
    assert fa.status() == fa.FA_OK
    scale = 1 / math.sqrt(d)
    dr = (0.1, 77, 2)
    O_ref, _ = oracle.attention_forward(f64(q), f64(k), f64(v), scale, True, dropout=dr, kv_len=[160, 90])
    assert np.abs(f64(O) - O_ref).max() <= 1e-2 + 2.0 ** -8 * np.abs(O_ref).max()
    dO = w.to(torch.bfloat16)  # the upstream gradient the kernel received, as bf16
    g = oracle.attention_backward(f64(q), f64(k), f64(v), f64(dO), scale, True, dropout=dr,
                                  kv_len=[160, 90])
    for got, ref, n in zip((qa.grad, ka.grad, va.grad), g[:3], ("dQ", "dK", "dV")):
        check_grad(got, ref, n, "autograd dropout + padding")
