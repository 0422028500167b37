"""GPU parity of the backward path (fa_bwd: D preprocessing, the tcgen05
backward kernel, dQ reduction and finalisation) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._parity import check_grad, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import exact_attention_115_b200 as fa
    fa.lib()
    return fa


@pytest.fixture(params=[1, 2, 3], ids=["dq_reduce_add", "dq_partials", "dq_grouped3"])
def dq_mode(request, fa):
    """Every dQ strategy; the grouped one with G = 3 buffers, so that K/V
    block counts not divisible by G leave groups of unequal sizes."""
    prev = fa.set_bwd_dq_mode(request.param)
    prev_g = fa.set_bwd_dq_groups(3)
    yield request.param
    fa.set_bwd_dq_mode(prev)
    fa.set_bwd_dq_groups(prev_g)


def run_bwd(fa, B, H, Nq, Nk, d, causal, dtype="bf16", seed=0, q_mult=1.0):
    q, k, v, do = W.make_tensors(B, H, Nq, Nk, d, dtype, seed=seed, q_mult=q_mult, device="cuda")
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa.backward(q, k, v, O, do, L, causal=causal, scale=scale)
    assert fa.status() == fa.FA_OK
    ref = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal)
    what = f"B{B} H{H} Nq{Nq} Nk{Nk} d{d} {dtype} causal={causal}"
    return [check_grad(g, r, n, what) for g, r, n in zip((dq, dk, dv), ref[:3], ("dQ", "dK", "dV"))]


@pytest.mark.parametrize("w", [W.TINY_BF16, W.TINY_FP32], ids=lambda w: w.name)
def test_tiny_workloads(fa, w, dq_mode):
    run_bwd(fa, w.B, w.H, w.Nq, w.Nk, w.d, w.causal, w.dtype)


def test_medium_workload(fa, dq_mode):
    w = W.MEDIUM
    run_bwd(fa, w.B, w.H, w.Nq, w.Nk, w.d, w.causal, w.dtype)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 127, 128, 129, 200, 257, 1000])
def test_odd_lengths(fa, N, d, causal):
    run_bwd(fa, 2, 3, N, N, d, causal, seed=N)


@pytest.mark.parametrize("Nq,Nk", [(1, 300), (100, 1000), (257, 513), (700, 129)])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular(fa, Nq, Nk, causal, dq_mode):
    if causal and Nq > Nk:
        pytest.skip("causal requires Nq <= Nk")
    run_bwd(fa, 1, 2, Nq, Nk, 128, causal, seed=Nq + Nk)
    run_bwd(fa, 1, 2, Nq, Nk, 64, causal, seed=Nq + Nk + 1)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_fp16_and_bf16(fa, dtype):
    run_bwd(fa, 2, 4, 384, 384, 128, True, dtype)
    run_bwd(fa, 2, 4, 384, 512, 64, False, dtype)


def test_fp32_rectangular(fa):
    run_bwd(fa, 1, 2, 100, 300, 64, True, "fp32")
    run_bwd(fa, 1, 2, 300, 200, 64, False, "fp32")


def test_peaky(fa):
    run_bwd(fa, 1, 4, 1024, 1024, 128, True, q_mult=3.0, seed=7)


def test_gradient_sum_invariants(fa):
    """Σ_j dK_j = 0 (rows of dS sum to zero) and Σ_j dV_j = Σ_i dO_i, at a
    size too large for a full oracle comparison."""
    w = W.CAUSAL_2K
    q, k, v, do = W.make_inputs(w, device="cuda")
    O, L = fa.forward(q, k, v, causal=True, scale=w.scale)
    dq, dk, dv = fa.backward(q, k, v, O, do, L, causal=True, scale=w.scale)
    sdk = dk.double().sum(dim=2)
    sdv = dv.double().sum(dim=2)
    sdo = do.double().sum(dim=2)
    assert (sdk.abs().max() / dk.double().abs().amax()).item() < 0.05
    assert ((sdv - sdo).abs().max() / sdo.abs().max()).item() < 0.02
