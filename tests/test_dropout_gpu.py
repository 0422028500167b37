"""GPU parity of attention dropout (fa_fwd_ex / fa_bwd_ex with an fa_dropout)
against the fp64 oracle and its own Philox4x32-10 keep mask.

The mask itself is checked bit for bit: with K = 0 every visible weight is
1/Nk, and with V_j = e_(j mod d) · 2^(j div d) each output element
O_ic · Nk · T/256 is the integer Σ_t Z(i, c + d·t) 2^t, exact in the 16-bit
output when 256/T is a power of two (p = 0.5, 0.75), so it spells out eight
keep bits of row i.  The backward is read out
the same way through dV with dO_i = e_(i mod d) · 2^(i div d).  Random-input
cases then compare O, L, dQ, dK, dV with the oracle under the same mask."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import philox
from tests._parity import check_fwd, check_grad, f64

pytestmark = pytest.mark.gpu

TORCH = {"bf16": torch.bfloat16, "fp16": torch.float16}


@pytest.fixture(scope="module")
def fa():
    import exact_attention_115_b200 as fa
    fa.lib()
    return fa


def _powers(n, d, dtype):
    """[n, d] rows e_(j mod d) · 2^(j div d)."""
    x = torch.zeros(n, d, dtype=torch.float32)
    j = torch.arange(n)
    x[j, j % d] = 2.0 ** (j // d).float()
    return x.to(dtype)


def _bits(Z, d):
    """Σ_t Z[..., c + d·t] 2^t over the last axis (length 8d) → [..., d]."""
    t = Z.shape[-1] // d
    Zr = Z.reshape(*Z.shape[:-1], t, d).astype(np.int64)
    return (Zr * (1 << np.arange(t))[:, None]).sum(-2)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("p", [0.5, 0.75])  # 256/T a power of two: exact readout
def test_forward_mask_bits_exact(fa, d, dtype, p):
    B, H, Nq, Nk = 2, 2, 300, 8 * d
    dev = "cuda"
    q = torch.randn(B, H, Nq, d, device=dev).to(TORCH[dtype])
    k = torch.zeros(B, H, Nk, d, device=dev, dtype=TORCH[dtype])
    v = _powers(Nk, d, TORCH[dtype]).to(dev).expand(B, H, Nk, d).contiguous()
    seed, off = 0x0123456789ABCDEF, 5
    O, L = fa.forward(q, k, v, scale=0.125, dropout_p=p, seed=seed, offset=off)
    assert fa.status() == fa.FA_OK
    t = philox.dropout_threshold(p)
    got = f64(O) * Nk * t / 256
    assert np.array_equal(got, np.round(got)), "readout not integral"
    for b in range(B):
        for h in range(H):
            Z = philox.keep_mask(b * H + h, np.arange(Nq), np.arange(Nk), p, seed, off)
            want = _bits(Z, d)
            bad = np.argwhere(got[b, h].astype(np.int64) != want)
            assert bad.size == 0, f"b{b} h{h}: {len(bad)} mismatches, first at {bad[0]}"
    assert np.allclose(f64(L), math.log(Nk), atol=1e-5)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("p", [0.5, 0.75])  # 256/T a power of two: exact readout
def test_backward_mask_bits_exact(fa, d, p):
    B, H, N = 1, 2, 8 * d
    dev = "cuda"
    dt = torch.bfloat16
    q = torch.randn(B, H, N, d, device=dev).to(dt)
    k = torch.zeros(B, H, N, d, device=dev, dtype=dt)
    v = torch.randn(B, H, N, d, device=dev).to(dt)
    do = _powers(N, d, dt).to(dev).expand(B, H, N, d).contiguous()
    seed, off = 987654321, 17
    O, L = fa.forward(q, k, v, scale=0.125, dropout_p=p, seed=seed, offset=off)
    dq, dk, dv = fa.backward(q, k, v, O, do, L, scale=0.125, dropout_p=p, seed=seed, offset=off)
    assert fa.status() == fa.FA_OK
    t = philox.dropout_threshold(p)
    got = f64(dv) * N * t / 256  # dV_jc · N · T/256 = Σ_t Z(c + d·t, j) 2^t
    assert np.array_equal(got, np.round(got)), "readout not integral"
    for h in range(H):
        Z = philox.keep_mask(h, np.arange(N), np.arange(N), p, seed, off)  # [query, key]
        want = _bits(Z.T, d)  # per key j, over queries
        bad = np.argwhere(got[0, h].astype(np.int64) != want)
        assert bad.size == 0, f"h{h}: {len(bad)} mismatches, first at {bad[0]}"


CASES = [  # B, H, Nq, Nk, d, causal
    (2, 3, 200, 200, 64, False),
    (2, 3, 200, 200, 128, True),
    (1, 2, 130, 300, 128, False),
    (1, 2, 130, 300, 64, True),
    (1, 2, 384, 384, 128, True),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", CASES)
@pytest.mark.parametrize("p", [0.1, 0.5])
def test_dropout_matches_oracle(fa, B, H, Nq, Nk, d, causal, p):
    q, k, v, do = W.make_tensors(B, H, Nq, Nk, d, "bf16", seed=21, device="cuda")
    scale = 1 / math.sqrt(d)
    seed, off = 1234 + Nq, 3
    O, L = fa.forward(q, k, v, causal=causal, scale=scale, dropout_p=p, seed=seed, offset=off)
    dq, dk, dv = fa.backward(q, k, v, O, do, L, causal=causal, scale=scale, dropout_p=p, seed=seed,
                             offset=off)
    assert fa.status() == fa.FA_OK
    dr = (p, seed, off)
    what = f"B{B} H{H} Nq{Nq} Nk{Nk} d{d} causal={causal} p={p}"
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, causal, dropout=dr)
    check_fwd(O, L, O_ref, L_ref, what)
    # the backward consumes the kernel's own O (through D); the oracle's
    # gradient uses its own O, which agrees within the forward tolerance
    dQ, dK, dV, _ = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal,
                                              dropout=dr)
    check_grad(dq, dQ, "dQ", what)
    check_grad(dk, dK, "dK", what)
    check_grad(dv, dV, "dV", what)


def test_dropout_fp16_and_strided(fa):
    """fp16 inputs in a [B, N, H, d] layout (the general-layout kernels)."""
    B, H, N, d, p = 2, 2, 256, 128, 0.2
    q, k, v, do = W.make_tensors(B, H, N, N, d, "fp16", seed=5, device="cuda")
    qs, ks, vs, dos = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v, do))
    scale, seed, off = 1 / math.sqrt(d), 42, 0
    O, L = fa.forward(qs, ks, vs, causal=True, scale=scale, dropout_p=p, seed=seed, offset=off)
    dq, dk, dv = fa.backward(qs, ks, vs, O, dos, L, causal=True, scale=scale, dropout_p=p,
                             seed=seed, offset=off)
    assert fa.status() == fa.FA_OK
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, True, dropout=(p, seed, off))
    check_fwd(O, L, O_ref, L_ref, "fp16 strided dropout")
    dQ, dK, dV, _ = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, True,
                                              dropout=(p, seed, off))
    for g, r, n in ((dq, dQ, "dQ"), (dk, dK, "dK"), (dv, dV, "dV")):
        check_grad(g, r, n, "fp16 strided dropout")


def test_same_seed_same_result_other_offset_differs(fa):
    q, k, v, _ = W.make_tensors(1, 2, 256, 256, 64, "bf16", seed=8, device="cuda", with_grad=False)
    O1, _ = fa.forward(q, k, v, dropout_p=0.3, seed=9, offset=1)
    O2, _ = fa.forward(q, k, v, dropout_p=0.3, seed=9, offset=1)
    O3, _ = fa.forward(q, k, v, dropout_p=0.3, seed=9, offset=2)
    O0, _ = fa.forward(q, k, v)
    assert torch.equal(O1, O2)
    assert not torch.equal(O1, O3)
    assert not torch.equal(O1, O0)
    # p = 0 is no dropout at all
    Oz, _ = fa.forward(q, k, v, dropout_p=0.0, seed=9, offset=1)
    assert torch.equal(Oz, O0)
