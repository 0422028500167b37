"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies runs out, the library reports it through fa_status and names the
wait, and the context keeps computing correct results afterwards."""
import math

import pytest

import oracle
import workloads as W
from tests._parity import check_fwd, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import exact_attention_115_b200 as fa
    fa.lib()
    return fa


def test_wait_timeout_is_reported_and_context_survives(fa):
    assert fa.status() == fa.FA_OK  # start clean
    assert fa.selftest_wait_timeout(20000) == fa.FA_OK  # a 20 ms wait that runs out
    assert fa.status() == fa.FA_ERR_TIMEOUT
    site = fa.lib().fa_last_timeout_site()
    assert 30000 < site < 40000, site  # the wait in the decode file's self-test kernel
    assert fa.status() == fa.FA_OK  # reading the status cleared it

    # the context is intact: a forward pass still matches the oracle
    B, H, N, d = 1, 2, 300, 64
    q, k, v, _ = W.make_tensors(B, H, N, N, d, "bf16", seed=3, device="cuda", with_grad=False)
    scale = 1 / math.sqrt(d)
    O, L = fa.forward(q, k, v, causal=True, scale=scale)
    assert fa.status() == fa.FA_OK
    O_ref, L_ref = oracle.attention_forward(f64(q), f64(k), f64(v), scale, True)
    check_fwd(O, L, O_ref, L_ref, "after a reported timeout")


def test_two_timeouts_report_once_each(fa):
    for _ in range(2):
        assert fa.selftest_wait_timeout(5000) == fa.FA_OK
        assert fa.status() == fa.FA_ERR_TIMEOUT
    assert fa.status() == fa.FA_OK
