"""Plain fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The library itself never calls it; there is no CPU fallback.

What it computes is the plain definition that FlashAttention reaches exactly
(up to rounding order), written out with a library matmul as the only
primitive:

* FlashAttention1 post (CSDN), section "具体算法":  S = Q Kᵀ, P = softmax(S),
  O = P V, here with the usual ``scale`` on S and an optional causal mask.
* FlashAttention V1/V2 study notes (51CTO), section "算法的改进": the backward
  pass needs only the row logsumexp L, not the running max, so L is an output.
* Same notes, section "Warp Level 并行": the backward products dV = Pᵀ dO,
  dS = P ∘ dP, dQ = dS K, dK = dSᵀ Q.  The page omits transposes, the scale
  and the −D term of the softmax Jacobian; this file writes the exact gradient
  of O = softmax(scale·Q Kᵀ) V (D = rowsum(dO ∘ O)).
* Same notes, section "算法的改进": the note under the V1/V2 forward and
  backward figures says the V1 algorithm also carries mask and dropout steps.
  The figures did not survive, so where dropout acts is a reading: on the
  normalised weights P, so the product uses P ∘ Z · s instead of P, where Z is
  a 0/1 keep mask and s = 1 / (keep probability); L stays the logsumexp of
  the undropped scores.  The backward is the exact gradient for that fixed Z:
  dP = (dO Vᵀ) ∘ Z · s and D = rowsum(dO ∘ O) with the dropped O.  The mask
  is an input here (``keep_fn``); ``oracle/philox.py`` draws it.
* Same notes, section "Sequence Parallel" (last paragraph, Flash-Decoding):
  split K/V along the sequence, compute each part's softmax, then a reduction
  rescales and adds the parts.  ``decode_split_combine`` restates that.

Readings where the pages are silent (each also listed in the design notes):

* causal masking is bottom-right aligned: key j is visible to query i iff
  j <= i + (Nk - Nq).  For Nq == Nk this is the plain lower triangle.
* L is the natural-log logsumexp of the scaled, masked scores of a row.
* a row with no visible key (a split of the decode, or a key-padding mask
  that hides every key) has O = 0 and L = -inf.
* key padding (``kv_len``): batch element b sees only keys j < kv_len[b]
  (an additive 0 / -inf mask over keys, ANDed with the causal mask, whose
  alignment still uses the full Nq and Nk).  The FlashAttention1 post
  (CSDN), section "引言/动机", lists the fused chain as matmul, scale, mask,
  softmax, so a mask acts on the scaled scores before the softmax; the
  51CTO notes' background list names custom masks as a reason to write
  one's own kernel.  Which masks is not fixed; this one is the padding of
  batched sequences of different lengths.
* additive bias (``bias``): the 51CTO background list names adding a bias as
  the first modification one writes one's own kernel for.  Reading: a
  constant added to the scaled scores, S' = scale·Q Kᵀ + bias (natural-log
  units, -inf allowed), before the masks and the softmax; L is the
  logsumexp of S'.  The bias gets no gradient (it is an input constant).

Everything is float64.  Inputs are whatever the caller passes (normally the
storage-dtype values the GPU sees, upcast exactly).  Rows are processed in
chunks so that long sequences do not materialise more than ``_ROW_CHUNK`` rows
of S at a time; chunking rows does not change any result because rows are
independent.
"""
from __future__ import annotations

import numpy as np

# Rows of S held at a time.  Rows are independent, so the chunk size changes
# no result; a small one keeps each temporary (128 × Nk floats) in the
# allocator's heap instead of a fresh mapping per chunk, whose page faults
# otherwise dominate the run time at long sequence lengths.
_ROW_CHUNK = 128


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def causal_visible(nq: int, nk: int, rows: np.ndarray | None = None) -> np.ndarray:
    """Boolean [len(rows), nk] mask of visible keys under bottom-right causal
    alignment (key j visible to query i iff j <= i + nk - nq)."""
    if rows is None:
        rows = np.arange(nq)
    rows = np.asarray(rows)
    return np.arange(nk)[None, :] <= (rows[:, None] + (nk - nq))


# --------------------------------------------------------------------------
# Page 1 worked example, restated: one query row, keys visited one at a time.
# --------------------------------------------------------------------------
def tiled_softmax_then_matmul(s_row, V) -> np.ndarray:
    """Online softmax followed by the product with V, one key at a time.

    FlashAttention1 post (CSDN), section "例子说明": walk the scores of one
    query row left to right, keeping the running maximum and the running sum
    of exponentials relative to it; each new key's probability is its
    exponential over the new running sum, the accumulated output is first
    rescaled by old_sum / new_sum (after moving the old sum onto the new
    maximum), and then the new key's probability times its V row is added.
    The accumulator is normalised after every step, as on the page.
    Returns a [1, d] array equal to softmax(s_row) @ V.
    """
    s = _f64(s_row).reshape(-1)
    V = _f64(V)
    n, d = V.shape
    assert s.shape[0] == n
    acc = np.zeros((1, d))
    run_max = -np.inf
    run_sum = 0.0
    for j in range(n):
        new_max = max(run_max, s[j])
        # the old sum was taken relative to run_max; move it onto new_max
        old_sum_on_new_max = run_sum * np.exp(run_max - new_max)
        new_sum = old_sum_on_new_max + np.exp(s[j] - new_max)
        prob_j = np.exp(s[j] - new_max) / new_sum
        acc *= old_sum_on_new_max / new_sum
        acc += prob_j * V[j][None, :]
        run_max, run_sum = new_max, new_sum
    return acc


# --------------------------------------------------------------------------
# Forward: the plain definition, per (batch, head), rows in chunks.
# --------------------------------------------------------------------------
def head_probs(q, k, scale: float, causal: bool, rows=None, nq_total=None, nk_valid=None,
               bias=None):
    """P (softmax rows) and L for the given query rows of one head.

    q: [r, d] the query rows, k: [Nk, d].  ``rows`` are the absolute indices
    of those query rows (needed for the causal mask) and ``nq_total`` the
    head's full query length; keys j >= ``nk_valid`` are masked (key
    padding); ``bias`` [r, Nk] is added to the scaled scores of these rows.
    Returns (P [r, Nk], L [r]).
    """
    q = _f64(q)
    k = _f64(k)
    r = q.shape[0]
    nk = k.shape[0]
    if rows is None:
        rows = np.arange(r)
    if nq_total is None:
        nq_total = r
    s = scale * (q @ k.T)
    if bias is not None:
        s = s + _f64(bias)
    if causal:
        s = np.where(causal_visible(nq_total, nk, rows), s, -np.inf)
    if nk_valid is not None:
        s = np.where(np.arange(nk)[None, :] < nk_valid, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    empty = ~np.isfinite(m)  # row with no visible key
    m = np.where(empty, 0.0, m)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(empty, 0.0, e / l)
        L = np.where(empty[:, 0], -np.inf, m[:, 0] + np.log(l[:, 0]))
    return p, L


def head_forward(q, k, v, scale: float, causal: bool, rows=None, nq_total=None, keep_fn=None,
                 kscale: float = 1.0, nk_valid=None, bias=None):
    """O [r, d] and L [r] for query rows of one head (see ``head_probs``).

    With dropout, ``keep_fn(rows, cols)`` gives the boolean keep mask at
    absolute query rows / key columns and ``kscale`` the factor on kept
    weights: O = (P ∘ Z · kscale) V."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    r = q.shape[0]
    if rows is None:
        rows = np.arange(r)
    rows = np.asarray(rows)
    if nq_total is None:
        nq_total = r
    O = np.empty((r, v.shape[1]))
    L = np.empty(r)
    for c0 in range(0, r, _ROW_CHUNK):
        c1 = min(r, c0 + _ROW_CHUNK)
        p, l = head_probs(q[c0:c1], k, scale, causal, rows[c0:c1], nq_total, nk_valid,
                          None if bias is None else bias[c0:c1])
        if keep_fn is not None:
            p = p * keep_fn(rows[c0:c1], np.arange(k.shape[0])) * kscale
        O[c0:c1] = p @ v
        L[c0:c1] = l
    return O, L


def _dropout_fn(dropout, bh):
    """(keep_fn, kscale) of head index bh for dropout = (p, seed, offset)."""
    if dropout is None:
        return None, 1.0
    from . import philox

    p, seed, offset = dropout
    return (lambda r, c: philox.keep_mask(bh, r, c, p, seed, offset)), philox.keep_scale(p)


def attention_forward(Q, K, V, scale: float, causal: bool = False, dropout=None, kv_len=None,
                      bias=None):
    """O [B,H,Nq,d] and L [B,H,Nq] (float64) for [B,H,N,d] inputs.
    ``dropout`` = (p, seed, offset) applies the Philox keep mask of
    ``oracle/philox.py`` to head index b·H + h; ``kv_len`` (B integers)
    hides keys j >= kv_len[b] of batch element b; ``bias`` (broadcastable to
    [B, H, Nq, Nk]) is added to the scaled scores."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, Nq, d = Q.shape
    if bias is not None:
        bias = np.broadcast_to(_f64(bias), (B, H, Nq, K.shape[2]))
    O = np.empty((B, H, Nq, V.shape[3]))
    L = np.empty((B, H, Nq))
    for b in range(B):
        for h in range(H):
            fn, ks = _dropout_fn(dropout, b * H + h)
            O[b, h], L[b, h] = head_forward(Q[b, h], K[b, h], V[b, h], scale, causal,
                                            keep_fn=fn, kscale=ks,
                                            nk_valid=None if kv_len is None else int(kv_len[b]),
                                            bias=None if bias is None else bias[b, h])
    return O, L


# --------------------------------------------------------------------------
# Backward: the exact gradient of O = softmax(scale Q Kᵀ [masked]) V.
# --------------------------------------------------------------------------
def head_backward(q, k, v, do, scale: float, causal: bool, keep_fn=None, kscale: float = 1.0,
                  nk_valid=None, bias=None):
    """dQ, dK, dV, D for one head (all query rows), float64.

    D_i = Σ_c dO_ic O_ic; dP = dO Vᵀ; dS = P ∘ (dP − D); dV = Pᵀ dO;
    dQ = scale · dS K; dK = scale · dSᵀ Q.  With dropout (``keep_fn``, see
    ``head_forward``) the products that see P ∘ Z · kscale are O and dV, and
    dP = (dO Vᵀ) ∘ Z · kscale.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    nq = q.shape[0]
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    D = np.empty(nq)
    rows_all = np.arange(nq)
    for c0 in range(0, nq, _ROW_CHUNK):
        c1 = min(nq, c0 + _ROW_CHUNK)
        p, _ = head_probs(q[c0:c1], k, scale, causal, rows_all[c0:c1], nq, nk_valid,
                          None if bias is None else bias[c0:c1])
        z = 1.0 if keep_fn is None else keep_fn(rows_all[c0:c1], np.arange(k.shape[0])) * kscale
        pz = p * z
        o = pz @ v
        Di = (do[c0:c1] * o).sum(axis=1)
        dp = (do[c0:c1] @ v.T) * z
        ds = p * (dp - Di[:, None])
        dv += pz.T @ do[c0:c1]
        dk += scale * (ds.T @ q[c0:c1])
        dq[c0:c1] = scale * (ds @ k)
        D[c0:c1] = Di
    return dq, dk, dv, D


def attention_backward(Q, K, V, dO, scale: float, causal: bool = False, dropout=None,
                       kv_len=None, bias=None):
    """dQ, dK, dV ([B,H,N,d]) and D ([B,H,Nq]) in float64 (``dropout`` and
    ``kv_len`` and ``bias`` as in ``attention_forward``; no gradient for
    the bias)."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    B, H = Q.shape[:2]
    if bias is not None:
        bias = np.broadcast_to(_f64(bias), (B, H, Q.shape[2], K.shape[2]))
    dQ = np.empty_like(Q)
    dK = np.empty_like(K)
    dV = np.empty_like(V)
    D = np.empty(Q.shape[:3])
    for b in range(B):
        for h in range(H):
            fn, ks = _dropout_fn(dropout, b * H + h)
            dQ[b, h], dK[b, h], dV[b, h], D[b, h] = head_backward(
                Q[b, h], K[b, h], V[b, h], dO[b, h], scale, causal, keep_fn=fn, kscale=ks,
                nk_valid=None if kv_len is None else int(kv_len[b]),
                bias=None if bias is None else bias[b, h])
    return dQ, dK, dV, D


def head_backward_rows(q, k, v, do, scale: float, causal: bool, q_rows, k_rows, keep_fn=None,
                       kscale: float = 1.0, nk_valid=None):
    """The same gradient as ``head_backward`` at selected rows only.

    Returns (dQ[q_rows], dK[k_rows], dV[k_rows], D[q_rows]).  dK/dV of a key
    row need P and dS of that key's column for every query row, hence the
    loop over all query chunks; dQ of a query row needs only that row.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    nq = q.shape[0]
    q_rows = np.asarray(q_rows)
    k_rows = np.asarray(k_rows)
    dk = np.zeros((len(k_rows), k.shape[1]))
    dv = np.zeros((len(k_rows), v.shape[1]))
    rows_all = np.arange(nq)
    for c0 in range(0, nq, _ROW_CHUNK):
        c1 = min(nq, c0 + _ROW_CHUNK)
        p, _ = head_probs(q[c0:c1], k, scale, causal, rows_all[c0:c1], nq, nk_valid)
        z = 1.0 if keep_fn is None else keep_fn(rows_all[c0:c1], np.arange(k.shape[0])) * kscale
        o = (p * z) @ v
        Di = (do[c0:c1] * o).sum(axis=1)
        zc = 1.0 if keep_fn is None else z[:, k_rows]
        pc = p[:, k_rows]
        dpc = (do[c0:c1] @ v[k_rows].T) * zc
        dsc = pc * (dpc - Di[:, None])
        dv += (pc * zc).T @ do[c0:c1]
        dk += scale * (dsc.T @ q[c0:c1])
    p, _ = head_probs(q[q_rows], k, scale, causal, q_rows, nq, nk_valid)
    z = 1.0 if keep_fn is None else keep_fn(q_rows, np.arange(k.shape[0])) * kscale
    o = (p * z) @ v
    Dq = (do[q_rows] * o).sum(axis=1)
    dp = (do[q_rows] @ v.T) * z
    ds = p * (dp - Dq[:, None])
    dq = scale * (ds @ k)
    return dq, dk, dv, Dq


# --------------------------------------------------------------------------
# Decode: Nq = 1; and the split-KV + logsumexp combine restated.
# --------------------------------------------------------------------------
def decode_split_combine(q, k, v, scale: float, num_splits: int):
    """Split-KV decode for one head, then the rescaling reduction.

    FlashAttention V1/V2 study notes (51CTO), section "Sequence Parallel",
    Flash-Decoding paragraph: cut K/V along the sequence into parts, run the
    softmax forward on each part, then reduce: each part's normalised output
    O_s is weighted by exp(L_s − L) where L = log Σ_s exp(L_s).  A part with
    no keys has L_s = −inf and weight 0.  q: [d] or [1, d]; returns (O [d], L).
    """
    q = _f64(q).reshape(1, -1)
    k, v = _f64(k), _f64(v)
    nk = k.shape[0]
    bounds = np.linspace(0, nk, num_splits + 1).round().astype(int)
    Os, Ls = [], []
    for s in range(num_splits):
        a, b = bounds[s], bounds[s + 1]
        if b <= a:
            Os.append(np.zeros(v.shape[1]))
            Ls.append(-np.inf)
            continue
        o, l = head_forward(q, k[a:b], v[a:b], scale, False)
        Os.append(o[0])
        Ls.append(l[0])
    Ls = np.array(Ls)
    Os = np.array(Os)
    mx = Ls.max()
    if not np.isfinite(mx):
        return np.zeros(v.shape[1]), -np.inf
    w = np.exp(Ls - mx)
    L = mx + np.log(w.sum())
    O = (np.exp(Ls - L)[:, None] * Os).sum(axis=0)
    return O, L


def attention_decode(Q, K, V, scale: float, kv_len=None):
    """Decode forward (Nq = 1, no causal mask; ``kv_len`` as in
    ``attention_forward``): O [B,H,1,d], L [B,H,1]."""
    return attention_forward(Q, K, V, scale, causal=False, kv_len=kv_len)
