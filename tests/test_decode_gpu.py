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


def test_decode_full_size_sampled(fa):
    w = W.DECODE_32K
    q, k, v, _ = W.make_inputs(w, device="cuda", with_grad=False)
    O, L = fa.decode(q, k, v, scale=w.scale)
    assert fa.status() == fa.FA_OK
    assert torch.isfinite(O.float()).all() and torch.isfinite(L).all()
    rng = np.random.default_rng(0)
    pairs = [(0, 0), (31, 31)] + [tuple(x) for x in rng.integers(0, 32, (6, 2))]
    for b, h in pairs:
        O_ref, L_ref = oracle.head_forward(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), w.scale, False)
        check_fwd(O[b, h], L[b, h], O_ref, L_ref, f"decode head ({b},{h})")
    del q, k, v
    torch.cuda.empty_cache()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("splits", [0, 1, 5, 64])
def test_decode_key_padding(fa, d, splits):
    """Per-sequence lengths of a KV cache padded to Nk (fa_decode_ex): parts
    past a length are empty; a zero length gives O = 0, L = -inf."""
    Nk = 3000
    kv_len = [Nk, 1, 0, 1537, 64, 5000]
    B = len(kv_len)
    q, k, v, _ = W.make_tensors(B, 2, 1, Nk, d, "bf16", seed=70 + d, device="cuda", with_grad=False)
    scale = 1 / math.sqrt(d)
    kvl = torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    O, L = fa.decode(q, k, v, scale=scale, num_splits=splits, kv_len=kvl)
    assert fa.status() == fa.FA_OK
    eff = [min(n, Nk) for n in kv_len]
    O_ref, L_ref = oracle.attention_decode(f64(q), f64(k), f64(v), scale, kv_len=eff)
    live = [b for b in range(B) if eff[b] > 0]
    check_fwd(O[live], L[live], O_ref[live], L_ref[live], f"decode kv_len d{d} splits{splits}")
    assert torch.all(O[2] == 0) and torch.all(torch.isneginf(L[2]))
    # full lengths equal the unpadded call bit for bit
    full = torch.full((B,), Nk, dtype=torch.int32, device="cuda")
    O1, L1 = fa.decode(q, k, v, scale=scale, num_splits=splits, kv_len=full)
    O0, L0 = fa.decode(q, k, v, scale=scale, num_splits=splits)
    assert torch.equal(O1, O0) and torch.equal(L1, L0)
