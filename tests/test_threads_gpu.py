"""Calls from a host thread that has made no CUDA runtime call of its own
(as autograd's worker threads may not have): such a thread has no current
context, and the library's tensor-map encoding (a driver call) must not
depend on one being there.  Every buffer is allocated on the main thread,
so the library's calls are the thread's first CUDA work."""
import math
import threading

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def test_forward_backward_from_a_fresh_thread():
    import exact_attention_115_b200 as fa

    B, H, N, d = 1, 3, 300, 128
    q, k, v, do = W.make_tensors(B, H, N, N, d, "bf16", seed=4, device="cuda")
    scale = 1 / math.sqrt(d)
    O1, L1 = fa.forward(q, k, v, causal=True, scale=scale)
    dq1, dk1, dv1 = fa.backward(q, k, v, O1, do, L1, causal=True, scale=scale)
    O, L = torch.empty_like(O1), torch.empty_like(L1)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, N, d), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    errors = []

    def run():
        try:
            fa.forward(q, k, v, causal=True, scale=scale, out=O, lse=L)
            fa.backward(q, k, v, O, do, L, causal=True, scale=scale, dq=dq, dk=dk, dv=dv,
                        workspace=ws)
        except Exception as e:  # noqa: BLE001 - reported below
            errors.append(e)

    t = threading.Thread(target=run)
    t.start()
    t.join(timeout=120)
    assert not t.is_alive()
    assert not errors, errors[0]
    torch.cuda.synchronize()
    assert fa.status() == fa.FA_OK
    assert torch.equal(O, O1) and torch.equal(L, L1)
    assert torch.equal(dk, dk1) and torch.equal(dv, dv1)
    gmax = dq1.float().abs().max().item()
    assert (dq.float() - dq1.float()).abs().max().item() <= 2e-2 * gmax
