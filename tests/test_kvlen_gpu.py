"""GPU parity of the key-padding mask (kv_len: batch element b sees keys
j < kv_len[b]) in fa_fwd_ex / fa_bwd_ex against the fp64 oracle.

Lengths cover the full length, a single key, tile edges ± 1, lengths past
Nk and below zero (clamped to [0, Nk]) and zero (every row of that batch element sees no key:
O = 0, L = -inf, zero gradients, and every K/V block of it is a work item
with no query steps)."""
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


def _check(fa, q, k, v, do, kv_len, causal, what, dropout=None, layout=None):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    scale = 1 / math.sqrt(d)
    kvl = torch.tensor(kv_len, dtype=torch.int32, device=q.device)
    eff = [min(max(n, 0), Nk) for n in kv_len]
    kw = {} if dropout is None else dict(dropout_p=dropout[0], seed=dropout[1], offset=dropout[2])
    lay = (lambda t: t) if layout is None else layout
    O, L = fa.forward(lay(q), lay(k), lay(v), causal=causal, scale=scale, kv_len=kvl, **kw)
    dq, dk, dv = fa.backward(lay(q), lay(k), lay(v), O, lay(do), L, causal=causal, scale=scale,
                             kv_len=kvl, **kw)
    assert fa.status() == fa.FA_OK
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, causal, dropout=dropout,
                                            kv_len=eff)
    g_ref = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal,
                                      dropout=dropout, kv_len=eff)
    On, Ln = f64(O), f64(L)
    live = [b for b in range(B) if eff[b] > 0]
    for b in range(B):
        if eff[b] == 0:
            assert np.all(On[b] == 0), f"{what}: O of an empty batch element"
            assert np.all(np.isneginf(Ln[b])), f"{what}: L of an empty batch element"
    check_fwd(O[live], L[live], O_ref[live], L_ref[live], what)
    for g, r, n in zip((dq, dk, dv), g_ref[:3], ("dQ", "dK", "dV")):
        check_grad(g, r, n, what)
    gk, gv = f64(dk), f64(dv)
    for b in range(B):  # keys past the length: exactly zero
        assert np.all(gk[b, :, eff[b]:] == 0) and np.all(gv[b, :, eff[b]:] == 0), what


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_key_padding(fa, d, causal):
    N = 300
    kv_len = [N, 1, 129, 0, 127, 1000, -5]  # past Nk and negative: clamped
    q, k, v, do = W.make_tensors(len(kv_len), 2, N, N, d, "bf16", seed=31 + d, device="cuda")
    _check(fa, q, k, v, do, kv_len, causal, f"kv_len d{d} causal={causal}")


def test_key_padding_rectangular_causal(fa):
    kv_len = [300, 200, 90]
    q, k, v, do = W.make_tensors(3, 2, 130, 300, 128, "bf16", seed=40, device="cuda")
    _check(fa, q, k, v, do, kv_len, True, "kv_len Nq130 Nk300 causal")


def test_key_padding_with_dropout_fp16_strided(fa):
    kv_len = [256, 70, 0]
    q, k, v, do = W.make_tensors(3, 2, 256, 256, 64, "fp16", seed=41, device="cuda")
    bshd = lambda t: t.transpose(1, 2).contiguous().transpose(1, 2)  # noqa: E731
    _check(fa, q, k, v, do, kv_len, False, "kv_len + dropout fp16 bshd", dropout=(0.2, 5, 1),
           layout=bshd)


def test_key_padding_longer(fa):
    kv_len = [1024, 700, 333]
    q, k, v, do = W.make_tensors(3, 4, 1024, 1024, 128, "bf16", seed=42, device="cuda")
    _check(fa, q, k, v, do, kv_len, True, "kv_len N1024 causal")


def test_full_length_equals_no_mask(fa):
    q, k, v, do = W.make_tensors(2, 2, 256, 256, 128, "bf16", seed=43, device="cuda")
    O0, L0 = fa.forward(q, k, v, causal=True)
    kvl = torch.tensor([256, 256], dtype=torch.int32, device="cuda")
    O1, L1 = fa.forward(q, k, v, causal=True, kv_len=kvl)
    assert torch.equal(O0, O1) and torch.equal(L0, L1)
