"""The head-sharded call on the GPU kernels: two ranks (processes on the
one visible GPU, gloo for the gathers; no kernel of one rank waits on the
other) each run the forward and backward kernels on half of the heads.  The
gathered results must equal the unsharded call: O, L, dK and dV bit for
bit (each head's arithmetic is the same, whichever launch computes it), and
dQ within the oracle tolerance (its fp32 reduce-adds may sum in another
order)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, shape, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import exact_attention_115_b200 as fa
    import workloads as W
    from exact_attention_115_b200 import sharded

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        B, H, N, d = shape
        q, k, v, do = W.make_tensors(B, H, N, N, d, "bf16", seed=11, device="cuda")
        O, L = sharded.forward(q, k, v, causal=causal)
        dq, dk, dv = sharded.backward(q, k, v, O, do, L, causal=causal)
        qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
        Oa = sharded.attention(qa, ka, va, causal=causal)
        Oa.backward(do)
        torch.cuda.synchronize()
        st = fa.status()
        O1, L1 = fa.forward(q, k, v, causal=causal)
        dq1, dk1, dv1 = fa.backward(q, k, v, O1, do, L1, causal=causal)
        torch.cuda.synchronize()
        gmax = dq1.float().abs().max().item()
        rel = lambda a, b: (a.float() - b.float()).abs().max().item() / gmax  # noqa: E731
        out[rank] = dict(
            status=st,
            exact=[torch.equal(a, b) for a, b in
                   ((O, O1), (L, L1), (dk, dk1), (dv, dv1), (Oa.detach(), O1),
                    (ka.grad, dk1), (va.grad, dv1))],
            dq_rel=max(rel(dq, dq1), rel(qa.grad, dq1)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shape,causal", [((2, 3, 300, 128), True), ((1, 5, 257, 64), False)])
def test_two_ranks_match_the_unsharded_call(shape, causal):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shape, causal, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    for r in range(world):
        res = out[r]
        assert res["status"] == 0
        assert all(res["exact"]), res["exact"]
        assert res["dq_rel"] <= 2e-2, res["dq_rel"]
