"""GPU parity of split-KV decode + combine against the fp64 oracle."""
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


@pytest.mark.parametrize("Nk", [1, 7, 64, 255, 1000, 4097])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("splits", [0, 1, 3, 16])
def test_decode_small(fa, Nk, d, splits):
    q, k, v, _ = W.make_tensors(2, 3, 1, Nk, d, "bf16", seed=Nk + d, device="cuda", with_grad=False)
    scale = 1 / math.sqrt(d)
    O, L = fa.decode(q, k, v, scale=scale, num_splits=splits)
    assert fa.status() == fa.FA_OK
    O_ref, L_ref = oracle.attention_decode(f64(q), f64(k), f64(v), scale)
    check_fwd(O, L, O_ref, L_ref, f"decode Nk{Nk} d{d} splits{splits}")


def test_decode_fp16(fa):
    q, k, v, _ = W.make_tensors(3, 2, 1, 3000, 128, "fp16", seed=5, device="cuda", with_grad=False)
    O, L = fa.decode(q, k, v)
    O_ref, L_ref = oracle.attention_decode(f64(q), f64(k), f64(v), 1 / math.sqrt(128))
    check_fwd(O, L, O_ref, L_ref, "decode fp16")


def test_decode_matches_forward_kernel(fa):
    """Decode and the tiled forward compute the same thing for Nq = 1."""
    q, k, v, _ = W.make_tensors(2, 4, 1, 2000, 128, "bf16", seed=9, device="cuda", with_grad=False)
    O1, L1 = fa.decode(q, k, v, num_splits=7)
    O2, L2 = fa.forward(q, k, v)
    assert (O1.float() - O2.float()).abs().max().item() <= 1e-2
    assert (L1 - L2).abs().max().item() <= 1e-3
