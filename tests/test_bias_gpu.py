"""GPU parity of the additive bias (fa_fwd_ex / fa_bwd_ex with a bias on the
scaled scores) against the fp64 oracle: full and broadcast biases, rows
padded to a multiple of 8 keys, -inf entries and fully hidden rows, and the
bias together with dropout, key padding and strided inputs."""
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


def _bias(shape, Nk, dtype, seed, ninf=0.0):
    """A bias of `shape` [b, h, Nq, Nk] in rows padded to a multiple of 8
    keys (sliced back to Nk), N(0, 1) values, a share `ninf` of them -inf."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    pad = (Nk + 7) // 8 * 8
    x = torch.randn(*shape[:3], pad, generator=g)
    if ninf:
        x[torch.rand(x.shape, generator=g) < ninf] = -math.inf
    return x.to(dtype).cuda()[..., :Nk]


def _run(fa, q, k, v, do, bias, causal, what, **kw):
    d = q.shape[-1]
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(q, k, v, causal=causal, scale=scale, bias=bias, **kw)
    dq, dk, dv = fa.backward(q, k, v, O, do, L, causal=causal, scale=scale, bias=bias, **kw)
    assert fa.status() == fa.FA_OK
    okw = {}
    if "dropout_p" in kw:
        okw["dropout"] = (kw["dropout_p"], kw["seed"], kw["offset"])
    if "kv_len" in kw:
        okw["kv_len"] = [int(x) for x in kw["kv_len"].cpu()]
    bf = f64(bias)
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, causal, bias=bf, **okw)
    g = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal, bias=bf, **okw)
    _check_rows(O, L, O_ref, L_ref, what)
    for got, ref, n in zip((dq, dk, dv), g[:3], ("dQ", "dK", "dV")):
        check_grad(got, ref, n, what)


def _check_rows(O, L, O_ref, L_ref, what):
    """Rows that see no key (every visible score hidden by a -inf bias, as
    happens to the first causal rows) must give O = 0 and L = -inf; the
    others are held to the forward tolerance in their own dtype."""
    live = np.isfinite(L_ref)
    dead = torch.from_numpy(~live).to(O.device)
    assert torch.all(O[dead] == 0) and torch.all(torch.isneginf(L[dead])), f"{what}: empty rows"
    keep = torch.from_numpy(live).to(O.device)
    check_fwd(O[keep], L[keep], O_ref[live], L_ref[live], what)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bshape", ["full", "batch_bcast", "head_bcast", "query_bcast", "keys_only"])
def test_bias(fa, d, causal, bshape):
    """Broadcast forms: over batches, heads, query rows ([B, H, 1, Nk]: one
    row per step staged for every query in the backward), or all three."""
    B, H, N = 2, 3, 300
    q, k, v, do = W.make_tensors(B, H, N, N, d, "bf16", seed=81 + d, device="cuda")
    shape = {"full": (B, H, N), "batch_bcast": (1, H, N), "head_bcast": (B, 1, N),
             "query_bcast": (B, H, 1), "keys_only": (1, 1, 1)}[bshape]
    bias = _bias(shape + (N,), N, torch.bfloat16, seed=7, ninf=0.05)
    _run(fa, q, k, v, do, bias, causal, f"bias {bshape} d{d} causal={causal}")


def test_bias_rectangular_causal(fa):
    q, k, v, do = W.make_tensors(1, 2, 130, 300, 128, "bf16", seed=90, device="cuda")
    bias = _bias((1, 2, 130, 300), 300, torch.bfloat16, seed=8)
    _run(fa, q, k, v, do, bias, True, "bias Nq130 Nk300 causal")


@pytest.mark.parametrize("bshape", ["full", "query_bcast"])
def test_bias_long_rows(fa, bshape):
    """Rows of 3100 keys at d = 128: without a bias such rows take the
    two-tile forward; with one they stay on the one-tile kernel and its
    64-key bias tiles, here over 49 K/V steps (the ring wraps many times)."""
    B, H, Nq, Nk = 1, 2, 200, 3100
    q, k, v, do = W.make_tensors(B, H, Nq, Nk, 128, "bf16", seed=94, device="cuda")
    shape = (B, H, Nq) if bshape == "full" else (B, H, 1)
    bias = _bias(shape + (Nk,), Nk, torch.bfloat16, seed=12, ninf=0.05)
    _run(fa, q, k, v, do, bias, False, f"bias {bshape} Nq{Nq} Nk{Nk}")


def test_bias_with_dropout_padding_fp16_strided(fa):
    B, H, N, d = 2, 2, 256, 64
    q, k, v, do = W.make_tensors(B, H, N, N, d, "fp16", seed=91, device="cuda")
    bshd = lambda t: t.transpose(1, 2).contiguous().transpose(1, 2)  # noqa: E731
    bias = _bias((B, H, N, N), N, torch.float16, seed=9, ninf=0.02)
    kvl = torch.tensor([256, 180], dtype=torch.int32, device="cuda")
    d_ = dict(dropout_p=0.15, seed=3, offset=4, kv_len=kvl)
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(bshd(q), bshd(k), bshd(v), scale=scale, bias=bias, **d_)
    dq, dk, dv = fa.backward(bshd(q), bshd(k), bshd(v), O, bshd(do), L, scale=scale, bias=bias, **d_)
    assert fa.status() == fa.FA_OK
    okw = dict(dropout=(0.15, 3, 4), kv_len=[256, 180], bias=f64(bias))
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, False, **okw)
    g = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, False, **okw)
    check_fwd(O, L, O_ref, L_ref, "bias + dropout + kv_len fp16 bshd")
    for got, ref, n in zip((dq, dk, dv), g[:3], ("dQ", "dK", "dV")):
        check_grad(got, ref, n, "bias + dropout + kv_len fp16 bshd")


def test_bias_hiding_whole_rows(fa):
    """Rows whose bias is -inf everywhere see no key: O = 0, L = -inf, and
    they contribute nothing to any gradient (their dQ is zero)."""
    B, H, N, d = 1, 2, 200, 128
    q, k, v, do = W.make_tensors(B, H, N, N, d, "bf16", seed=92, device="cuda")
    bias = _bias((B, H, N, N), N, torch.bfloat16, seed=10)
    hidden = [0, 77, 199]
    bias[:, :, hidden, :] = -math.inf
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(q, k, v, scale=scale, bias=bias)
    dq, dk, dv = fa.backward(q, k, v, O, do, L, scale=scale, bias=bias)
    assert fa.status() == fa.FA_OK
    assert torch.all(O[:, :, hidden] == 0) and torch.all(torch.isneginf(L[:, :, hidden]))
    assert torch.all(dq[:, :, hidden] == 0)
    live = [i for i in range(N) if i not in hidden]
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, False, bias=f64(bias))
    check_fwd(O[:, :, live], L[:, :, live], O_ref[:, :, live], L_ref[:, :, live], "hidden rows")
    g = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, False, bias=f64(bias))
    for got, ref, n in zip((dq, dk, dv), g[:3], ("dQ", "dK", "dV")):
        check_grad(got, ref, n, "hidden rows")


def test_bias_autograd(fa):
    q, k, v, do = W.make_tensors(2, 2, 160, 160, 64, "bf16", seed=93, device="cuda")
    bias = _bias((1, 2, 160, 160), 160, torch.bfloat16, seed=11)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    O = fa.attention(qa, ka, va, causal=True, bias=bias)
    O.backward(do)
    O0, L0 = fa.forward(q, k, v, causal=True, bias=bias)
    _, dk0, dv0 = fa.backward(q, k, v, O0, do, L0, causal=True, bias=bias)
    assert fa.status() == fa.FA_OK
    assert torch.equal(O.detach(), O0)
    assert torch.equal(ka.grad, dk0) and torch.equal(va.grad, dv0)


def test_bias_repeatable(fa):
    """The same call gives the same bits every time: O and L of the forward,
    dK and dV of the backward (dQ is summed by atomics, in no fixed order).
    The staged bias tile is refilled by TMA right after the softmax threads
    read it; a missing proxy fence there showed as rows of L and O that
    changed from run to run, most often on long rows (here 46 steps of 64
    keys per query tile, one-tile kernel)."""
    B, H, N, d = 4, 16, 2944, 128
    q, k, v, do = W.make_tensors(B, H, N, N, d, "bf16", seed=95, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(13)
    bias = torch.randn(1, H, N, N, generator=g, device="cuda").to(torch.bfloat16)
    outs = [fa.forward(q, k, v, bias=bias) for _ in range(20)]
    torch.cuda.synchronize()
    assert fa.status() == fa.FA_OK
    O0, L0 = outs[0]
    differ = [i for i, (O, L) in enumerate(outs) if not (torch.equal(O, O0) and torch.equal(L, L0))]
    assert not differ, f"forward runs {differ} differ from the first"
    del outs
    grads = [fa.backward(q, k, v, O0, do, L0, bias=bias)[1:] for _ in range(4)]
    torch.cuda.synchronize()
    assert fa.status() == fa.FA_OK
    for i, (dk, dv) in enumerate(grads[1:], 1):
        assert torch.equal(dk, grads[0][0]) and torch.equal(dv, grads[0][1]), f"backward run {i} differs"
