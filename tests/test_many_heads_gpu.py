"""More than 65535 heads (B·H = 70000, a grid's second dimension holds at
most 65535 blocks): forward, backward and decode against the fp64 oracle on
heads on both sides of that boundary and at the ends."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _parity import check_fwd, check_grad, f64

pytestmark = pytest.mark.gpu

B, H, d = 2, 35000, 64
SAMPLE = [0, 1, 34999, 35000, 65534, 65535, 65536, 69999]  # flattened b·H + h


def _heads(t, idx):
    """[1, len(idx), N, d] float64 copy of the sampled heads of a [B, H, N, d] tensor."""
    flat = t.reshape(B * H, *t.shape[2:])
    return f64(flat[idx]).reshape(1, len(idx), *t.shape[2:])


def test_forward_backward_many_heads():
    import exact_attention_115_b200 as fa

    N = 100
    q, k, v, do = W.make_tensors(B, H, N, N, d, "bf16", seed=21, device="cuda")
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(q, k, v, causal=True, scale=scale)
    dq, dk, dv = fa.backward(q, k, v, O, do, L, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.status() == fa.FA_OK
    idx = torch.tensor(SAMPLE, device="cuda")
    qs, ks, vs, dos = (_heads(t, idx) for t in (q, k, v, do))
    O_ref, L_ref = oracle.attention_forward(qs, ks, vs, scale, causal=True)
    Ls = f64(L.reshape(B * H, N)[idx]).reshape(1, len(SAMPLE), N)
    check_fwd(_heads(O, idx), Ls, O_ref, L_ref, "B·H = 70000 forward")
    g_ref = oracle.attention_backward(qs, ks, vs, dos, scale, causal=True)
    for name, G, R in zip(("dQ", "dK", "dV"), (dq, dk, dv), g_ref[:3]):
        check_grad(_heads(G, idx), R, name, "B·H = 70000 backward")
    # every head was written (the outputs start as uninitialised memory)
    for t in (O, dq, dk, dv):
        assert bool(torch.isfinite(t).all())


@pytest.mark.parametrize("splits", [0, 3])
def test_decode_many_heads(splits):
    import exact_attention_115_b200 as fa

    Nk = 300
    q, k, v, _ = W.make_tensors(B, H, 1, Nk, d, "bf16", seed=22, device="cuda", with_grad=False)
    scale = 1 / math.sqrt(d)
    O, L = fa.decode(q, k, v, scale=scale, num_splits=splits)
    torch.cuda.synchronize()
    assert fa.status() == fa.FA_OK
    idx = torch.tensor(SAMPLE, device="cuda")
    O_ref, L_ref = oracle.attention_decode(_heads(q, idx), _heads(k, idx), _heads(v, idx), scale)
    Ls = f64(L.reshape(B * H, 1)[idx]).reshape(1, len(SAMPLE), 1)
    check_fwd(_heads(O, idx), Ls, O_ref, L_ref, f"B·H = 70000 decode, splits {splits}")
    assert bool(torch.isfinite(O).all()) and bool(torch.isfinite(L).all())
    assert np.isfinite(f64(L)).all()
