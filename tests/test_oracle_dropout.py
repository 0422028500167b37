"""Pins for the oracle's dropout: its Philox4x32-10 generator, the keep mask
built from it, and attention with a keep mask.

* the generator against published known-answer vectors (tests/golden);
* the mask's layout against a per-element restatement, and its keep rate
  against the binomial distribution;
* attention with dropout against brute force on tiny inputs, against torch
  float64 autograd through an explicit mask, against central finite
  differences with the mask held fixed, and (statistically) against the
  undropped result it must equal on average.
"""
import math
import pathlib

import numpy as np
import pytest
import torch

import oracle
from oracle import philox

GOLDEN = pathlib.Path(__file__).parent / "golden" / "philox4x32_10_kat.txt"


def _kat():
    for line in GOLDEN.read_text().splitlines():
        if line.startswith("#") or not line.strip():
            continue
        words = [int(x, 16) for x in line.split()]
        yield words[:4], words[4:6], words[6:10]


def test_philox_known_answers():
    cases = list(_kat())
    assert len(cases) >= 2
    for ctr, key, want in cases:
        got = philox.philox4x32_10(ctr, key)
        assert [int(x) for x in got] == want


def test_philox_broadcasts_over_counters():
    ctr = np.array([[0, 0, 0, 0], [0xFFFFFFFF] * 4], dtype=np.uint64)
    key = np.array([[0, 0], [0xFFFFFFFF] * 2], dtype=np.uint64)
    got = philox.philox4x32_10(ctr, key)
    want = [w for _, _, w in _kat()][:2]
    assert got.tolist() == want


def test_threshold_and_scale():
    assert philox.dropout_threshold(0.0) == 256
    assert philox.dropout_threshold(0.5) == 128
    assert philox.dropout_threshold(0.25) == 192
    assert philox.dropout_threshold(0.1) == 230  # (1 - 0.1f)·256 = 230.4
    assert philox.keep_scale(0.5) == 2.0
    for bad in (-0.1, 1.0, 0.999):
        with pytest.raises(ValueError):
            philox.dropout_threshold(bad)


def test_keep_mask_layout_per_element():
    """Every element from its own generator call: block (i//4, j//4),
    counter (j//4, i//4, bh, offset), word i%4, byte j%4."""
    bh, p, seed, offset = 5, 0.3, 0x1234_5678_9ABC_DEF0, 77
    rows = np.array([0, 1, 3, 4, 9, 130])
    cols = np.array([0, 2, 3, 4, 7, 127, 128, 301])
    got = philox.keep_mask(bh, rows, cols, p, seed, offset)
    t = philox.dropout_threshold(p)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for a, i in enumerate(rows):
        for b, j in enumerate(cols):
            w = int(philox.philox4x32_10([j // 4, i // 4, bh, offset], key)[i % 4])
            assert got[a, b] == (((w >> (8 * (j % 4))) & 0xFF) < t)


def test_keep_rate_is_binomial():
    p = 0.25
    m = philox.keep_mask(3, np.arange(256), np.arange(1024), p, seed=99, offset=0)
    n = m.size
    q = philox.dropout_threshold(p) / 256
    assert abs(m.mean() - q) <= 5 * math.sqrt(q * (1 - q) / n)
    # different heads, offsets and seeds give different masks
    m2 = philox.keep_mask(4, np.arange(256), np.arange(1024), p, seed=99, offset=0)
    m3 = philox.keep_mask(3, np.arange(256), np.arange(1024), p, seed=99, offset=1)
    m4 = philox.keep_mask(3, np.arange(256), np.arange(1024), p, seed=100, offset=0)
    for other in (m2, m3, m4):
        agree = (m == other).mean()
        assert abs(agree - (q * q + (1 - q) * (1 - q))) < 0.01


def test_no_dropout_is_identity():
    rng = np.random.default_rng(1)
    Q, K, V = (rng.standard_normal((1, 2, 9, 4)) for _ in range(3))
    O0, L0 = oracle.attention_forward(Q, K, V, 0.5, True)
    O1, L1 = oracle.attention_forward(Q, K, V, 0.5, True, dropout=(0.0, 7, 3))
    assert np.array_equal(O0, O1) and np.array_equal(L0, L1)


def test_dropout_forward_brute_force():
    rng = np.random.default_rng(2)
    B, H, Nq, Nk, d = 1, 2, 6, 9, 3
    Q, K, V = rng.standard_normal((B, H, Nq, d)), rng.standard_normal((B, H, Nk, d)), \
        rng.standard_normal((B, H, Nk, d))
    p, seed, off, scale = 0.4, 12345, 6, 0.8
    for causal in (False, True):
        O, L = oracle.attention_forward(Q, K, V, scale, causal, dropout=(p, seed, off))
        t = philox.dropout_threshold(p)
        for h in range(H):
            for i in range(Nq):
                vis = [j for j in range(Nk) if not causal or j <= i + Nk - Nq]
                s = {j: scale * sum(Q[0, h, i, c] * K[0, h, j, c] for c in range(d)) for j in vis}
                mx = max(s.values())
                den = sum(math.exp(x - mx) for x in s.values())
                want = [0.0] * d
                for j in vis:
                    w = int(philox.philox4x32_10([j // 4, i // 4, h, off],
                                                 [seed & 0xFFFFFFFF, seed >> 32])[i % 4])
                    if ((w >> (8 * (j % 4))) & 0xFF) < t:
                        for c in range(d):
                            want[c] += math.exp(s[j] - mx) / den * (256 / t) * V[0, h, j, c]
                assert np.max(np.abs(O[0, h, i] - want)) <= 1e-12
                assert abs(L[0, h, i] - (mx + math.log(den))) <= 1e-12


def _torch_dropout_attention(Q, K, V, dO, scale, causal, Z, ks):
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    s = scale * q @ k.transpose(-1, -2)
    if causal:
        nq, nk = s.shape[-2:]
        vis = torch.arange(nk)[None, :] <= torch.arange(nq)[:, None] + (nk - nq)
        s = s.masked_fill(~vis, float("-inf"))
    o = (torch.softmax(s, dim=-1) * torch.tensor(Z, dtype=torch.float64) * ks) @ v
    o.backward(torch.tensor(dO, dtype=torch.float64))
    return o.detach().numpy(), q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_backward_matches_torch_autograd(causal):
    rng = np.random.default_rng(3)
    B, H, Nq, Nk, d = 2, 2, 37, 53, 16
    Q, dO = rng.standard_normal((B, H, Nq, d)), rng.standard_normal((B, H, Nq, d))
    K, V = rng.standard_normal((B, H, Nk, d)), rng.standard_normal((B, H, Nk, d))
    p, seed, off, scale = 0.3, 2024, 1, 0.25
    Z = np.stack([np.stack([philox.keep_mask(b * H + h, np.arange(Nq), np.arange(Nk), p, seed, off)
                            for h in range(H)]) for b in range(B)])
    O, L = oracle.attention_forward(Q, K, V, scale, causal, dropout=(p, seed, off))
    dQ, dK, dV, D = oracle.attention_backward(Q, K, V, dO, scale, causal, dropout=(p, seed, off))
    # the factor written out, independent of the oracle: p = 0.3 keeps a
    # weight iff its byte is below T = round(0.7 · 256) = 179, scaled by 256/179
    assert philox.dropout_threshold(p) == 179
    tO, tq, tk, tv = _torch_dropout_attention(Q, K, V, dO, scale, causal, Z, 256 / 179)
    assert np.max(np.abs(O - tO)) <= 1e-12
    for got, want in ((dQ, tq), (dK, tk), (dV, tv)):
        assert np.max(np.abs(got - want)) <= 1e-10
    assert np.max(np.abs(D - (dO * O).sum(-1))) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_backward_matches_finite_differences(causal):
    rng = np.random.default_rng(4)
    n, d, scale, p, seed, off = 6, 3, 0.7, 0.5, 77, 2
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    fn = lambda r, c: philox.keep_mask(0, r, c, p, seed, off)  # noqa: E731
    ks = philox.keep_scale(p)
    dq, dk, dv, _ = oracle.head_backward(q, k, v, do, scale, causal, keep_fn=fn, kscale=ks)

    def f(qq, kk, vv):
        O, _ = oracle.head_forward(qq, kk, vv, scale, causal, keep_fn=fn, kscale=ks)
        return float(np.sum(do * O))

    h = 1e-6
    for which, got in enumerate((dq, dk, dv)):
        args = [q, k, v]
        for idx in np.ndindex(*got.shape):
            ap = [x.copy() for x in args]
            am = [x.copy() for x in args]
            ap[which][idx] += h
            am[which][idx] -= h
            want = (f(*ap) - f(*am)) / (2 * h)
            assert abs(got[idx] - want) <= 1e-7 * max(1.0, abs(want))


def test_dropout_is_unbiased_on_average():
    """E[O with dropout] = O: the mean over many independent masks (offsets)
    converges to the undropped output."""
    rng = np.random.default_rng(5)
    Q, K, V = (rng.standard_normal((1, 1, 4, 3)) for _ in range(3))
    O0, _ = oracle.attention_forward(Q, K, V, 0.6, False)
    n = 3000
    acc = np.zeros_like(O0)
    sq = np.zeros_like(O0)
    for off in range(n):
        O, _ = oracle.attention_forward(Q, K, V, 0.6, False, dropout=(0.5, 31337, off))
        acc += O
        sq += O * O
    mean = acc / n
    sd = np.sqrt(np.maximum(sq / n - mean * mean, 1e-30) / n)
    assert np.all(np.abs(mean - O0) <= 5 * sd + 1e-12)


def test_dropout_backward_rows_equal_full():
    rng = np.random.default_rng(6)
    q, k, v, do = (rng.standard_normal((70, 8)) for _ in range(4))
    fn = lambda r, c: philox.keep_mask(2, r, c, 0.2, 5, 9)  # noqa: E731
    ks = philox.keep_scale(0.2)
    dq, dk, dv, D = oracle.head_backward(q, k, v, do, 0.3, True, keep_fn=fn, kscale=ks)
    qr, kr = np.array([0, 5, 44, 69]), np.array([1, 17, 60, 69])
    rq, rk, rv, rD = oracle.head_backward_rows(q, k, v, do, 0.3, True, qr, kr, keep_fn=fn, kscale=ks)
    for got, want in ((rq, dq[qr]), (rk, dk[kr]), (rv, dv[kr]), (rD, D[qr])):
        assert np.max(np.abs(got - want)) <= 1e-13
