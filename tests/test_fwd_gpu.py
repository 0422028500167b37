"""GPU parity of the forward kernel against the fp64 oracle (call path:
Python binding -> fa_fwd C ABI -> sm_100a kernel)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._parity import check_fwd, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import exact_attention_115_b200 as fa
    fa.lib()
    return fa


def run_full(fa, B, H, Nq, Nk, d, causal, dtype="bf16", seed=0, q_mult=1.0):
    q, k, v, _ = W.make_tensors(B, H, Nq, Nk, d, dtype, seed=seed, q_mult=q_mult,
                                device="cuda", with_grad=False)
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(q, k, v, causal=causal, scale=scale)
    assert fa.status() == fa.FA_OK
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, causal)
    return check_fwd(O, L, O_ref, L_ref, f"B{B} H{H} Nq{Nq} Nk{Nk} d{d} {dtype} causal={causal}")


@pytest.mark.parametrize("w", [W.TINY_BF16, W.TINY_FP32], ids=lambda w: w.name)
def test_tiny_workloads(fa, w):
    run_full(fa, w.B, w.H, w.Nq, w.Nk, w.d, w.causal, w.dtype)


def test_medium_workload(fa):
    w = W.MEDIUM
    run_full(fa, w.B, w.H, w.Nq, w.Nk, w.d, w.causal, w.dtype)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 127, 128, 129, 255, 256, 257, 1000])
def test_odd_lengths(fa, N, d, causal):
    run_full(fa, 2, 3, N, N, d, causal, seed=N)


@pytest.mark.parametrize("Nq,Nk", [(1, 300), (100, 1000), (257, 513), (700, 129)])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular(fa, Nq, Nk, causal):
    if causal and Nq > Nk:
        pytest.skip("causal requires Nq <= Nk")
    run_full(fa, 1, 2, Nq, Nk, 128, causal, seed=Nq + Nk)


@pytest.mark.parametrize("Nq,Nk,causal,dtype", [
    (3100, 3100, False, "bf16"),   # 25 K/V tiles per query tile; the last CTA holds 28 rows
    (300, 6500, True, "bf16"),     # bottom-right causal, ~50 K/V tiles on average, ragged ends
    (1000, 7000, True, "fp16"),    # bottom-right causal with Nk − Nq = 6000
    (129, 3200, False, "bf16"),    # two Q tiles, the second with one row
])
def test_two_tile_d128_kernel(fa, Nq, Nk, causal, dtype):
    """Shapes whose query tiles see 24 or more 128-key K/V tiles on average
    (48 or more with the causal mask) run the 16-bit d = 128 forward with two
    Q tiles per CTA; the shorter ones (every other test here at d = 128) run
    one Q tile over 64-key K/V tiles."""
    run_full(fa, 1, 2, Nq, Nk, 128, causal, dtype, seed=Nq + 3 * Nk)


def test_two_tile_d128_kernel_strided_with_padding(fa):
    """The two-tile d = 128 forward on a [B, N, H, d] layout with key padding."""
    B, H, N, d = 2, 2, 3200, 128
    q, k, v, _ = W.make_tensors(B, H, N, N, d, "bf16", seed=8, device="cuda", with_grad=False)
    bshd = lambda t: t.transpose(1, 2).contiguous().transpose(1, 2)  # noqa: E731
    kv_len = torch.tensor([3200, 900], dtype=torch.int32, device="cuda")
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(bshd(q), bshd(k), bshd(v), causal=False, scale=scale, kv_len=kv_len)
    assert fa.status() == fa.FA_OK
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, False,
                                            kv_len=kv_len.cpu().numpy())
    check_fwd(O, L, O_ref, L_ref, "two-tile d128, [B, N, H, d], kv_len")


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_fp16_and_bf16(fa, dtype):
    run_full(fa, 2, 4, 384, 384, 128, True, dtype)
    run_full(fa, 2, 4, 384, 512, 64, False, dtype)


def test_fp32_tf32(fa):
    run_full(fa, 1, 2, 300, 300, 64, True, "fp32")


def test_peaky_rescaling(fa):
    """Q scaled ×6: row maxima grow across many K/V tiles, exercising the
    correction of the O accumulator, under the standard bounds."""
    run_full(fa, 1, 4, 1024, 1024, 128, False, q_mult=6.0, seed=3)
    run_full(fa, 1, 4, 1024, 1024, 128, True, q_mult=6.0, seed=4)


def test_very_peaky_rescaling_sanity(fa):
    """Q scaled ×8: the softmax is dominated by one or two keys per row, so
    the bf16 rounding of P and of O alone approach the 1e-2 bound (about
    1.8e-2 at |O| ~ 3.3 is observed); a wrong rescale would give errors of
    order |V|.  Checked with a 5e-2 element bound and the stated L bound."""
    for causal, seed in ((False, 3), (True, 4)):
        q, k, v, _ = W.make_tensors(1, 4, 1024, 1024, 128, "bf16", seed=seed, q_mult=8.0,
                                    device="cuda", with_grad=False)
        O, L = fa.forward(q, k, v, causal=causal)
        O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), 1 / math.sqrt(128), causal)
        assert np.abs(f64(O) - O_ref).max() <= 5e-2
        assert np.abs(f64(O) - O_ref).mean() <= 1e-3
        assert np.abs(f64(L) - L_ref).max() <= 1e-3


def test_keys_sorted_ascending_force_rescales(fa):
    """Scores that grow along the key axis: every tile raises the maximum."""
    B, H, N, d = 1, 1, 1024, 64
    q = torch.ones(B, H, N, d, device="cuda", dtype=torch.bfloat16)
    ramp = torch.linspace(-4, 4, N, device="cuda").view(1, 1, N, 1)
    k = (ramp * torch.ones(1, 1, 1, d, device="cuda")).to(torch.bfloat16).contiguous()
    v = torch.randn(B, H, N, d, device="cuda", generator=torch.Generator("cuda").manual_seed(1)).to(torch.bfloat16)
    O, L = fa.forward(q, k, v, causal=False, scale=1.0)
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), 1.0, False)
    check_fwd(O, L, O_ref, L_ref, "ascending scores")
