"""Shared helpers for the GPU parity tests: tolerance checks against the
fp64 oracle.  Tolerances (bf16/fp16 inputs, fp32 accumulation):
O max-abs <= 1e-2 and mean-abs <= 1e-3; L max-abs <= 1e-3;
dQ/dK/dV max-abs <= 2e-2 * max|grad_ref| (each).

O is stored in the input dtype, and the final cast alone moves a value by
up to half a unit in the last place of that dtype (0.0156 for bf16 values in
[4, 8)), more than 1e-2 for any |O| > 2.56.  The element-wise O bound is
therefore 1e-2 plus half an ulp of the output dtype at the reference value;
the mean-abs bound and the L bound are applied as stated.  ``check_fwd``
also returns the plain max-abs error so callers can report it."""
import ctypes
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

O_MAX, O_MEAN, L_MAX, G_REL = 1e-2, 1e-3, 1e-3, 2e-2


def f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


MANTISSA_BITS = {torch.bfloat16: 7, torch.float16: 10, torch.float32: 23}


def half_ulp(x, dtype):
    """Half a unit in the last place of ``dtype`` at |x| (normal range)."""
    mb = MANTISSA_BITS[dtype]
    ax = np.maximum(np.abs(x), 2.0 ** -14)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(int) - mb - 1)


def check_fwd(O, L, O_ref, L_ref, what=""):
    dtype = O.dtype if isinstance(O, torch.Tensor) else torch.float32
    O, L = f64(O), f64(L)
    assert np.all(np.isfinite(O)), f"{what}: non-finite O"
    assert np.all(np.isfinite(L)), f"{what}: non-finite L"
    e = np.abs(O - O_ref)
    el = np.abs(L - L_ref)
    bound = O_MAX + half_ulp(O_ref, dtype)
    worst = np.argmax(e - bound)
    assert np.all(e <= bound), (f"{what}: O error {e.flat[worst]:.3e} at ref {O_ref.flat[worst]:.4f} "
                                f"exceeds 1e-2 + half-ulp; plain max-abs {e.max():.3e}")
    assert e.mean() <= O_MEAN, f"{what}: O mean-abs {e.mean():.3e}"
    assert el.max() <= L_MAX, f"{what}: L max-abs {el.max():.3e}"
    return e.max(), e.mean(), el.max()


# When the exact gradient is identically zero (e.g. a single visible key:
# the softmax is constant, so dS = 0), the relative bound is 0; fp32 rounding
# then leaves ~1e-7, so an absolute floor applies.
G_ABS_FLOOR = 1e-5


def check_grad(G, G_ref, name, what="", scale_ref=None):
    G = f64(G)
    assert np.all(np.isfinite(G)), f"{what}: non-finite {name}"
    ref_max = np.abs(G_ref).max() if scale_ref is None else scale_ref
    e = np.abs(G - G_ref).max()
    bound = max(G_REL * ref_max, G_ABS_FLOOR)
    assert e <= bound, f"{what}: {name} max-abs {e:.3e} > {bound:.3e} (max|ref| {ref_max:.3e})"
    return e / max(ref_max, 1e-30)


def _keep_freed_memory_in_heap():
    """The oracle's temporaries at long sequence lengths are tens of MB each;
    glibc maps and unmaps every such block, and the page faults then dominate
    the oracle's run time.  Raising the trim and mmap thresholds keeps freed
    blocks in the heap for reuse.  This affects only the test process."""
    try:
        libc = ctypes.CDLL("libc.so.6")
        libc.mallopt(-1, 1 << 30)   # M_TRIM_THRESHOLD
        libc.mallopt(-3, 32 << 20)  # M_MMAP_THRESHOLD (its largest allowed value)
    except (OSError, AttributeError):
        pass


_keep_freed_memory_in_heap()


def host_cores() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def oracle_map(fn, items):
    """[fn(x) for x in items] on all host cores, in threads (numpy releases
    the GIL in its matrix products and element-wise loops, so the calls run
    in parallel), the cores' BLAS threads shared out between the calls."""
    from threadpoolctl import threadpool_limits

    workers = min(host_cores(), max(1, len(items)))
    with threadpool_limits(max(1, host_cores() // workers)):
        with ThreadPoolExecutor(workers) as ex:
            return list(ex.map(fn, items))


def nan_like(t):
    """A NaN-filled buffer shaped like ``t``: passed as an output, it shows any
    element a kernel failed to write (the check then finds a non-finite value)."""
    return torch.full_like(t, float("nan"))
