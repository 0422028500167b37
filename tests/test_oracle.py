"""Pins for the fp64 oracle against things other than itself.

Each test ties the oracle to the pages' worked example, a closed form, an
invariant, brute force on tiny inputs, finite differences, or a library
routine (torch's scaled_dot_product_attention in float64 on the CPU).  Each
is chosen so that a plausible slip in the oracle (a dropped scale, a missing
transpose, a sign, an off-by-one in the causal mask, a wrong logsumexp)
fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _sdpa(Q, K, V, scale, causal, dO=None):
    """torch SDPA in float64 on the CPU (+ autograd when dO is given)."""
    q = torch.tensor(Q, dtype=torch.float64, requires_grad=dO is not None)
    k = torch.tensor(K, dtype=torch.float64, requires_grad=dO is not None)
    v = torch.tensor(V, dtype=torch.float64, requires_grad=dO is not None)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=scale)
    if dO is None:
        return o.detach().numpy(), None
    o.backward(torch.tensor(dO, dtype=torch.float64))
    return o.detach().numpy(), (q.grad.numpy(), k.grad.numpy(), v.grad.numpy())


# ---------------------------------------------------------------- page 1 example
@pytest.mark.parametrize("n,d", [(4, 2), (257, 7)])
def test_worked_example_equals_softmax_times_v(n, d):
    """FlashAttention1 post (CSDN), section "例子说明": the token-by-token
    online softmax must equal softmax(S) V.  The page draws S and V unseeded
    and its printed output was an image, so the draw here is seeded."""
    rng = _rng(0)
    S = rng.random((1, n))
    V = rng.random((n, d))
    got = oracle.tiled_softmax_then_matmul(S, V)
    e = np.exp(S - S.max())
    want = (e / e.sum()) @ V
    assert np.max(np.abs(got - want)) <= 1e-12


def test_worked_example_extreme_scores():
    """Scores far apart (±700) must not overflow the running sum."""
    s = np.array([[-700.0, 700.0, 0.0, 699.0]])
    V = np.arange(8, dtype=np.float64).reshape(4, 2)
    got = oracle.tiled_softmax_then_matmul(s, V)
    e = np.exp(s - 700.0)
    want = (e / e.sum()) @ V
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want)) <= 1e-12


# ---------------------------------------------------------------- forward vs SDPA
@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 1, 128, 64, False), (1, 1, 128, 64, True), (2, 3, 33, 16, True), (1, 2, 200, 8, False)])
def test_forward_matches_torch_sdpa(B, H, N, d, causal):
    rng = _rng(1)
    Q, K, V = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    scale = 1 / math.sqrt(d)
    O, L = oracle.attention_forward(Q, K, V, scale, causal)
    want, _ = _sdpa(Q, K, V, scale, causal)
    assert np.max(np.abs(O - want)) <= 1e-12


def test_forward_rectangular_matches_sdpa():
    rng = _rng(2)
    Q = rng.standard_normal((1, 2, 17, 8))
    K = rng.standard_normal((1, 2, 45, 8))
    V = rng.standard_normal((1, 2, 45, 8))
    O, _ = oracle.attention_forward(Q, K, V, 0.3, False)
    want, _ = _sdpa(Q, K, V, 0.3, False)
    assert np.max(np.abs(O - want)) <= 1e-12


# ---------------------------------------------------------------- closed forms
def test_zero_keys_give_mean_of_values_and_log_n():
    rng = _rng(3)
    nk = 37
    Q = rng.standard_normal((1, 1, 11, 8))
    K = np.zeros((1, 1, nk, 8))
    V = rng.standard_normal((1, 1, nk, 8))
    O, L = oracle.attention_forward(Q, K, V, 0.5, False)
    assert np.max(np.abs(O[0, 0] - V[0, 0].mean(axis=0))) <= 1e-14
    assert np.max(np.abs(L - math.log(nk))) <= 1e-14


def test_causal_first_row_sees_only_first_key():
    rng = _rng(4)
    Q, K, V = (rng.standard_normal((1, 1, 19, 8)) for _ in range(3))
    scale = 0.37
    O, L = oracle.attention_forward(Q, K, V, scale, True)
    assert np.max(np.abs(O[0, 0, 0] - V[0, 0, 0])) <= 1e-15
    assert abs(L[0, 0, 0] - scale * Q[0, 0, 0] @ K[0, 0, 0]) <= 1e-13


def test_ones_values_give_ones():
    rng = _rng(5)
    Q, K = (rng.standard_normal((1, 2, 23, 8)) for _ in range(2))
    V = np.ones((1, 2, 23, 8))
    for causal in (False, True):
        O, _ = oracle.attention_forward(Q, K, V, 0.4, causal)
        assert np.max(np.abs(O - 1.0)) <= 1e-14


def test_prob_rows_sum_to_one_and_respect_mask():
    rng = _rng(6)
    q, k = rng.standard_normal((20, 8)), rng.standard_normal((30, 8))
    P, _ = oracle.head_probs(q, k, 0.3, True, np.arange(20), 20)
    assert np.max(np.abs(P.sum(axis=1) - 1.0)) <= 1e-15
    # bottom-right alignment: query i sees keys 0..i+10
    for i in range(20):
        assert np.all(P[i, i + 11:] == 0.0)
        assert np.all(P[i, : i + 11] > 0.0)


def test_logsumexp_brute_force():
    """L against a Python-float brute force (math.fsum of math.exp) on tiny
    inputs, causal and not."""
    rng = _rng(7)
    q, k, v = rng.standard_normal((6, 3)), rng.standard_normal((9, 3)), rng.standard_normal((9, 3))
    scale = 0.8
    for causal in (False, True):
        _, L = oracle.head_forward(q, k, v, scale, causal)
        for i in range(6):
            terms = []
            for j in range(9):
                if causal and j > i + 3:
                    continue
                s = scale * sum(float(q[i, c]) * float(k[j, c]) for c in range(3))
                terms.append(math.exp(s))
            assert abs(L[i] - math.log(math.fsum(terms))) <= 1e-13


def test_key_shift_invariance():
    """Adding k0 to every key row leaves O unchanged and shifts L_i by
    scale·q_i·k0 (softmax is shift invariant per row)."""
    rng = _rng(8)
    Q, K, V = (rng.standard_normal((1, 1, 40, 8)) for _ in range(3))
    k0 = rng.standard_normal(8) * 5
    scale = 0.35
    for causal in (False, True):
        O1, L1 = oracle.attention_forward(Q, K, V, scale, causal)
        O2, L2 = oracle.attention_forward(Q, K + k0, V, scale, causal)
        assert np.max(np.abs(O1 - O2)) <= 1e-12
        assert np.max(np.abs(L2 - L1 - scale * (Q[0, 0] @ k0))) <= 1e-11


def test_key_permutation_invariance():
    rng = _rng(9)
    Q, K, V = (rng.standard_normal((1, 1, 31, 8)) for _ in range(3))
    perm = rng.permutation(31)
    O1, L1 = oracle.attention_forward(Q, K, V, 0.3, False)
    O2, L2 = oracle.attention_forward(Q, K[:, :, perm], V[:, :, perm], 0.3, False)
    assert np.max(np.abs(O1 - O2)) <= 1e-13
    assert np.max(np.abs(L1 - L2)) <= 1e-13


def test_huge_scores_stay_finite():
    """scale·S of order ±1000: a naive exp would overflow; the oracle must be
    finite and still satisfy the shift invariance."""
    rng = _rng(10)
    Q = 40 * rng.standard_normal((1, 1, 16, 8))
    K = 40 * rng.standard_normal((1, 1, 16, 8))
    V = rng.standard_normal((1, 1, 16, 8))
    scale = 1 / math.sqrt(8)
    O, L = oracle.attention_forward(Q, K, V, scale, False)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L))
    assert np.max(np.abs(L)) > 500
    k0 = np.full(8, 3.0)
    O2, _ = oracle.attention_forward(Q, K + k0, V, scale, False)
    assert np.max(np.abs(O - O2)) <= 1e-9


def test_causal_rectangular_is_tail_of_square():
    """Bottom-right causal alignment with Nq < Nk equals the last Nq rows of
    the square causal problem whose first Nk−Nq queries are arbitrary."""
    rng = _rng(11)
    nq, nk, d = 7, 19, 8
    Qfull = rng.standard_normal((1, 1, nk, d))
    K, V = (rng.standard_normal((1, 1, nk, d)) for _ in range(2))
    Osq, Lsq = oracle.attention_forward(Qfull, K, V, 0.4, True)
    Ort, Lrt = oracle.attention_forward(Qfull[:, :, nk - nq:], K, V, 0.4, True)
    assert np.max(np.abs(Ort - Osq[:, :, nk - nq:])) <= 1e-14
    assert np.max(np.abs(Lrt - Lsq[:, :, nk - nq:])) <= 1e-14


def test_row_subset_forward_equals_full():
    rng = _rng(12)
    q, k, v = (rng.standard_normal((50, 8)) for _ in range(3))
    O, L = oracle.head_forward(q, k, v, 0.3, True)
    rows = np.array([0, 7, 31, 49])
    Or, Lr = oracle.head_forward(q[rows], k, v, 0.3, True, rows=rows, nq_total=50)
    assert np.max(np.abs(Or - O[rows])) <= 1e-15
    assert np.max(np.abs(Lr - L[rows])) <= 1e-15


def test_chunked_rows_equal_unchunked(monkeypatch):
    import oracle.attention as oa
    rng = _rng(13)
    q, k, v, do = (rng.standard_normal((70, 8)) for _ in range(4))
    O1, L1 = oa.head_forward(q, k, v, 0.3, True)
    g1 = oa.head_backward(q, k, v, do, 0.3, True)
    monkeypatch.setattr(oa, "_ROW_CHUNK", 16)
    O2, L2 = oa.head_forward(q, k, v, 0.3, True)
    g2 = oa.head_backward(q, k, v, do, 0.3, True)
    assert np.max(np.abs(O1 - O2)) <= 1e-15 and np.max(np.abs(L1 - L2)) <= 1e-15
    for a, b in zip(g1, g2):
        assert np.max(np.abs(a - b)) <= 1e-13


# ---------------------------------------------------------------- backward
def _fd_grads(q, k, v, do, scale, causal, h=1e-6):
    """Central finite differences of f = Σ dO ∘ O(q, k, v)."""
    def f(qq, kk, vv):
        O, _ = oracle.head_forward(qq, kk, vv, scale, causal)
        return float(np.sum(do * O))

    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        for idx in np.ndindex(*g.shape):
            a_p = [x.copy() for x in args]
            a_m = [x.copy() for x in args]
            a_p[which][idx] += h
            a_m[which][idx] -= h
            g[idx] = (f(*a_p) - f(*a_m)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("n", [3, 5])
@pytest.mark.parametrize("d", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(n, d, causal):
    rng = _rng(100 + n * 10 + d + causal)
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    scale = 0.7
    dq, dk, dv, _ = oracle.head_backward(q, k, v, do, scale, causal)
    fq, fk, fv = _fd_grads(q, k, v, do, scale, causal)
    for got, want in ((dq, fq), (dk, fk), (dv, fv)):
        assert np.max(np.abs(got - want)) <= 1e-7 * max(1.0, np.max(np.abs(want)))


def test_backward_rectangular_matches_finite_differences():
    rng = _rng(150)
    q, do = rng.standard_normal((3, 4)), rng.standard_normal((3, 4))
    k, v = rng.standard_normal((6, 4)), rng.standard_normal((6, 4))
    for causal in (False, True):
        dq, dk, dv, _ = oracle.head_backward(q, k, v, do, 0.6, causal)
        fq, fk, fv = _fd_grads(q, k, v, do, 0.6, causal)
        for got, want in ((dq, fq), (dk, fk), (dv, fv)):
            assert np.max(np.abs(got - want)) <= 1e-7 * max(1.0, np.max(np.abs(want)))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd(causal):
    rng = _rng(200)
    B, H, N, d = 1, 2, 128, 64
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    scale = 1 / math.sqrt(d)
    dQ, dK, dV, D = oracle.attention_backward(Q, K, V, dO, scale, causal)
    O, grads = _sdpa(Q, K, V, scale, causal, dO)
    for got, want in zip((dQ, dK, dV), grads):
        assert np.max(np.abs(got - want)) <= 1e-10
    assert np.max(np.abs(D - (dO * O).sum(-1))) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sum_invariants(causal):
    """Σ_j dS_ij = 0 makes the key-row sum of dK vanish; rows of P summing to
    one make Σ_j dV_j = Σ_i dO_i."""
    rng = _rng(300)
    q, k, v, do = (rng.standard_normal((64, 16)) for _ in range(4))
    dq, dk, dv, _ = oracle.head_backward(q, k, v, do, 0.25, causal)
    assert np.max(np.abs(dk.sum(axis=0))) <= 1e-11
    assert np.max(np.abs(dv.sum(axis=0) - do.sum(axis=0))) <= 1e-11


def test_backward_rows_equal_full():
    rng = _rng(400)
    q, k, v, do = (rng.standard_normal((90, 8)) for _ in range(4))
    dq, dk, dv, D = oracle.head_backward(q, k, v, do, 0.3, True)
    qr = np.array([0, 5, 44, 89])
    kr = np.array([1, 17, 60, 89])
    rq, rk, rv, rD = oracle.head_backward_rows(q, k, v, do, 0.3, True, qr, kr)
    assert np.max(np.abs(rq - dq[qr])) <= 1e-13
    assert np.max(np.abs(rk - dk[kr])) <= 1e-13
    assert np.max(np.abs(rv - dv[kr])) <= 1e-13
    assert np.max(np.abs(rD - D[qr])) <= 1e-13


# ---------------------------------------------------------------- decode
@pytest.mark.parametrize("splits", [1, 7, 64])
def test_decode_split_combine_equals_unsplit(splits):
    rng = _rng(500)
    q = rng.standard_normal(32)
    k, v = rng.standard_normal((1000, 32)), rng.standard_normal((1000, 32))
    O, L = oracle.decode_split_combine(q, k, v, 0.2, splits)
    Ow, Lw = oracle.head_forward(q[None], k, v, 0.2, False)
    assert np.max(np.abs(O - Ow[0])) <= 1e-12
    assert abs(L - Lw[0]) <= 1e-12


def test_decode_split_with_empty_parts():
    rng = _rng(501)
    q = rng.standard_normal(8)
    k, v = rng.standard_normal((5, 8)), rng.standard_normal((5, 8))
    O, L = oracle.decode_split_combine(q, k, v, 0.5, 8)  # 3 of 8 parts empty
    Ow, Lw = oracle.head_forward(q[None], k, v, 0.5, False)
    assert np.max(np.abs(O - Ow[0])) <= 1e-13
    assert abs(L - Lw[0]) <= 1e-13


def test_decode_matches_sdpa():
    rng = _rng(502)
    Q = rng.standard_normal((2, 3, 1, 16))
    K, V = rng.standard_normal((2, 3, 300, 16)), rng.standard_normal((2, 3, 300, 16))
    O, L = oracle.attention_decode(Q, K, V, 0.25)
    want, _ = _sdpa(Q, K, V, 0.25, False)
    assert np.max(np.abs(O - want)) <= 1e-13


# --------------------------------------------------------------------------
# Key padding (kv_len): pinned by the truncated problem it must equal.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_key_padding_matches_torch_autograd(causal):
    """Hiding keys j >= kv_len[b] against torch float64 SDPA with the same
    boolean mask (padding AND bottom-right causal with the full Nk), forward
    and autograd gradients; the hidden keys get zero dK and dV."""
    rng = _rng(500)
    B, H, Nq, Nk, d = 3, 2, 7, 11, 4
    Q, dO = rng.standard_normal((B, H, Nq, d)), rng.standard_normal((B, H, Nq, d))
    K, V = rng.standard_normal((B, H, Nk, d)), rng.standard_normal((B, H, Nk, d))
    kv_len = [11, 9, 6]
    O, L = oracle.attention_forward(Q, K, V, 0.5, causal, kv_len=kv_len)
    dQ, dK, dV, _ = oracle.attention_backward(Q, K, V, dO, 0.5, causal, kv_len=kv_len)
    j = np.arange(Nk)[None, None, None, :]
    vis = j < np.array(kv_len)[:, None, None, None]
    if causal:
        vis = vis & (j <= np.arange(Nq)[None, None, :, None] + (Nk - Nq))
    q, k, v = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.tensor(vis),
                                                         scale=0.5)
    o.backward(torch.tensor(dO))
    assert np.max(np.abs(O - o.detach().numpy())) <= 1e-12
    for got, want in ((dQ, q.grad), (dK, k.grad), (dV, v.grad)):
        assert np.max(np.abs(got - want.numpy())) <= 1e-11
    for b, n in enumerate(kv_len):
        assert np.all(dK[b, :, n:] == 0) and np.all(dV[b, :, n:] == 0)


def test_key_padding_full_length_is_no_mask_and_zero_length_is_empty():
    rng = _rng(501)
    Q, K, V, dO = (rng.standard_normal((2, 1, 5, 3)) for _ in range(4))
    O0, L0 = oracle.attention_forward(Q, K, V, 0.4, False)
    O1, L1 = oracle.attention_forward(Q, K, V, 0.4, False, kv_len=[5, 5])
    assert np.array_equal(O0, O1) and np.array_equal(L0, L1)
    O2, L2 = oracle.attention_forward(Q, K, V, 0.4, False, kv_len=[0, 5])
    assert np.all(O2[0] == 0) and np.all(np.isneginf(L2[0]))
    assert np.array_equal(O2[1], O0[1])
    g = oracle.attention_backward(Q, K, V, dO, 0.4, False, kv_len=[0, 5])
    for x in g[:3]:
        assert np.all(x[0] == 0)


def test_key_padding_matches_torch_sdpa_bool_mask():
    rng = _rng(502)
    B, H, N, d = 2, 2, 33, 8
    Q, K, V = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    kv_len = [20, 33]
    mask = torch.tensor(np.arange(N)[None, None, None, :] < np.array(kv_len)[:, None, None, None])
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(Q), torch.tensor(K), torch.tensor(V), attn_mask=mask, scale=0.3)
    O, _ = oracle.attention_forward(Q, K, V, 0.3, False, kv_len=kv_len)
    assert np.max(np.abs(O - o.numpy())) <= 1e-12


def test_decode_key_padding_matches_sdpa():
    rng = _rng(503)
    B, H, Nk, d = 3, 2, 50, 8
    Q = rng.standard_normal((B, H, 1, d))
    K, V = rng.standard_normal((B, H, Nk, d)), rng.standard_normal((B, H, Nk, d))
    kv_len = [50, 17, 1]
    mask = torch.tensor(np.arange(Nk)[None, None, None, :] < np.array(kv_len)[:, None, None, None])
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(Q), torch.tensor(K), torch.tensor(V), attn_mask=mask, scale=0.35)
    O, L = oracle.attention_decode(Q, K, V, 0.35, kv_len=kv_len)
    assert np.max(np.abs(O - o.numpy())) <= 1e-12
    s = 0.35 * np.einsum("bhqd,bhkd->bhqk", Q, K)
    for b, n in enumerate(kv_len):
        ref = np.log(np.exp(s[b, :, :, :n]).sum(-1))
        assert np.max(np.abs(L[b] - ref)) <= 1e-12


# --------------------------------------------------------------------------
# Additive bias: pinned by torch SDPA with the same float mask.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_bias_matches_torch_autograd(causal):
    rng = _rng(504)
    B, H, Nq, Nk, d = 2, 3, 9, 13, 4
    Q, dO = rng.standard_normal((B, H, Nq, d)), rng.standard_normal((B, H, Nq, d))
    K, V = rng.standard_normal((B, H, Nk, d)), rng.standard_normal((B, H, Nk, d))
    bias = rng.standard_normal((1, H, Nq, Nk))  # broadcast over the batch
    bias[0, 1, 2, :5] = -np.inf                 # some hidden keys
    O, L = oracle.attention_forward(Q, K, V, 0.6, causal, bias=bias)
    dQ, dK, dV, _ = oracle.attention_backward(Q, K, V, dO, 0.6, causal, bias=bias)
    m = np.broadcast_to(bias, (B, H, Nq, Nk)).copy()
    if causal:
        vis = np.arange(Nk)[None, :] <= np.arange(Nq)[:, None] + (Nk - Nq)
        m = np.where(vis, m, -np.inf)
    q, k, v = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.tensor(m), scale=0.6)
    o.backward(torch.tensor(dO))
    assert np.max(np.abs(O - o.detach().numpy())) <= 1e-12
    for got, want in ((dQ, q.grad), (dK, k.grad), (dV, v.grad)):
        assert np.max(np.abs(got - want.numpy())) <= 1e-11
    s = 0.6 * np.einsum("bhqd,bhkd->bhqk", Q, K) + m
    ref_L = np.log(np.exp(s - s.max(-1, keepdims=True)).sum(-1)) + s.max(-1)
    assert np.max(np.abs(L - ref_L)) <= 1e-12


def test_bias_constant_per_row_changes_nothing_but_L():
    """softmax is invariant to a per-row constant: O unchanged, L shifted."""
    rng = _rng(505)
    Q, K, V = (rng.standard_normal((1, 2, 6, 4)) for _ in range(3))
    c = rng.standard_normal((1, 2, 6, 1))
    O0, L0 = oracle.attention_forward(Q, K, V, 0.5, False)
    O1, L1 = oracle.attention_forward(Q, K, V, 0.5, False, bias=np.broadcast_to(c, (1, 2, 6, 6)))
    assert np.max(np.abs(O1 - O0)) <= 1e-12
    assert np.max(np.abs(L1 - L0 - c[..., 0])) <= 1e-12
