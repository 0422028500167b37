"""fa_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a runtime or plugin that owns all device memory
and hands the library only its input and output buffers, or a service whose
device memory is fixed after start-up).  It uses the library's own device
scratch array instead of a caller-provided workspace.

Checked through the C ABI against the existing entry point, fa_decode, on
two calls in a row (the second call reuses the scratch the first one left),
and against the fp64 oracle, with the tolerances used throughout (O 1e-2
plus half an ulp of the output dtype, L 1e-3), plus the rejection of sizes
beyond the built-in scratch.  This file is named to be collected last."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._parity import check_fwd, f64

pytestmark = pytest.mark.gpu


def _noalloc(fa, q, k, v, num_splits):
    B, H, _, d = q.shape
    Nk = k.shape[2]
    O = torch.empty_like(q)
    L = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    rc = fa.lib().fa_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), O.data_ptr(),
                                    L.data_ptr(), B, H, Nk, d, 1.0 / math.sqrt(d),
                                    fa.FA_BF16 if q.dtype == torch.bfloat16 else fa.FA_FP16,
                                    num_splits, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, O, L


@pytest.mark.parametrize("num_splits", [0, 5])
def test_noalloc_matches_decode_on_two_calls(num_splits):
    import exact_attention_115_b200 as fa
    shapes = [(4, 8, 3000, 128, "bf16", 11), (2, 16, 777, 64, "fp16", 12)]
    for call, (B, H, Nk, d, dt, seed) in enumerate(shapes):
        q, k, v, _ = W.make_tensors(B, H, 1, Nk, d, dt, seed=seed, device="cuda", with_grad=False)
        rc, O, L = _noalloc(fa, q, k, v, num_splits)
        assert rc == fa.FA_OK, f"call {call}: {fa.STATUS_NAMES.get(rc, rc)}"
        assert fa.status() == fa.FA_OK
        O_ref, L_ref = fa.decode(q, k, v, num_splits=num_splits)
        assert fa.status() == fa.FA_OK
        check_fwd(O, L, f64(O_ref), f64(L_ref), f"no-alloc decode call {call} vs fa_decode")
        O_o, L_o = oracle.attention_decode(f64(q), f64(k), f64(v), 1.0 / math.sqrt(d))
        check_fwd(O, L, O_o, L_o, f"no-alloc decode call {call} vs the oracle")


def test_noalloc_full_size_workload_matches_decode():
    import exact_attention_115_b200 as fa
    w = W.DECODE_32K
    q, k, v, _ = W.make_inputs(w, device="cuda", with_grad=False)
    O, L = fa.decode_noalloc(q, k, v)
    assert fa.status() == fa.FA_OK
    O_ref, L_ref = fa.decode(q, k, v)
    check_fwd(O, L, f64(O_ref), f64(L_ref), "no-alloc decode, B32 H32 Nk32768")
    # batch element 0 (32 heads) against the oracle as well
    hq, hk, hv = f64(q[0]), f64(k[0]), f64(v[0])
    for h in range(w.H):
        O_o, L_o = oracle.head_forward(hq[h], hk[h], hv[h], w.scale, False)
        check_fwd(O[0, h], L[0, h], O_o, L_o, f"no-alloc decode head (0,{h}) vs the oracle")
    del q, k, v
    torch.cuda.empty_cache()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import exact_attention_115_b200 as fa
    lib = fa.lib()
    fake = 0x10000  # rejected before anything is enqueued; never dereferenced
    # an explicit split count whose partials exceed the 8 MiB
    rc = lib.fa_decode_noalloc(fake, fake, fake, fake, fake, 64, 32, 32768, 128, 0.1, fa.FA_BF16,
                               64, None)
    assert rc == fa.FA_ERR_WORKSPACE
    # even one part per (batch, head) does not fit: B*H*(d+1)*4 > 8 MiB
    rc = lib.fa_decode_noalloc(fake, fake, fake, fake, fake, 512, 64, 4096, 128, 0.1, fa.FA_BF16,
                               0, None)
    assert rc == fa.FA_ERR_WORKSPACE
    assert fa.FA_DECODE_NOALLOC_SCRATCH_BYTES == 8 << 20
