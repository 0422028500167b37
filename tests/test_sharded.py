"""Host logic of the head-sharded call (exact_attention_115_b200.sharded) on
CPU: the shard ranges, and forward / backward / autograd over gloo process
groups of 2 and 3 ranks, with the per-shard kernels replaced by the fp64
oracle so that only the sharding and the gathers are under test.  The
gathered outputs must equal the oracle on the whole tensors to 1e-12 (the
same fp64 computation per head; BLAS may sum in another order for a shard's
memory layout), while a misplaced or missing head would be off by O(1)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("BH", [1, 3, 5, 8, 128])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_ranges_tile_the_heads(BH, world):
    from exact_attention_115_b200.sharded import shard_range

    per = -(-BH // world)
    prev = 0
    for r in range(world):
        s, e = shard_range(BH, world, r)
        assert s == prev and s <= e and e - s <= per
        prev = e
    assert prev == BH
    with pytest.raises(ValueError):
        shard_range(BH, world, world)


def _oracle_forward(q, k, v, causal, scale):
    """The per-shard forward, on the oracle: [1, n, N, d] in, (O, L) out."""
    O, L = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), scale, causal)
    return torch.from_numpy(O).to(q.dtype), torch.from_numpy(L).float()


def _oracle_backward(q, k, v, o, do, lse, causal, scale):
    # what the kernels' C interface requires of every pointer
    for t in (q, k, v, o, do, lse):
        assert t.data_ptr() % 16 == 0, "shard pointer not 16-byte aligned"
    dq, dk, dv, _ = oracle.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(),
                                              scale, causal)
    return tuple(torch.from_numpy(x).to(q.dtype) for x in (dq, dk, dv))


def _worker(rank, world, port, shape, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    from exact_attention_115_b200 import sharded

    sharded._fa_forward = lambda q, k, v, causal, scale: _oracle_forward(q, k, v, causal, scale)
    sharded._fa_backward = (lambda q, k, v, o, do, lse, causal, scale:
                            _oracle_backward(q, k, v, o, do, lse, causal, scale))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, H, N, d = shape
        g = torch.Generator().manual_seed(7)  # the same inputs on every rank
        q, k, v, do = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(4))
        scale = d ** -0.5
        O, L = sharded.forward(q, k, v, causal=causal)
        dq, dk, dv = sharded.backward(q, k, v, O, do, L, causal=causal)
        qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
        Oa = sharded.attention(qa, ka, va, causal=causal)
        Oa.backward(do)
        O_ref, L_ref = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), scale, causal)
        g_ref = oracle.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), scale,
                                          causal)
        close = lambda a, b, tol=1e-12: np.abs(np.asarray(a, np.float64) - b).max() <= tol  # noqa: E731
        ok = (close(O.numpy(), O_ref) and close(L.numpy(), L_ref, 1e-6)
              and all(close(a.numpy(), b) for a, b in zip((dq, dk, dv), g_ref[:3]))
              and close(Oa.detach().numpy(), O_ref)
              and all(close(t.grad.numpy(), b) for t, b in zip((qa, ka, va), g_ref[:3])))
        out[rank] = (ok, tuple(O.shape), tuple(L.shape), tuple(dk.shape))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape,causal", [
    (2, (2, 3, 17, 8), True),    # 6 heads, 3 per rank
    (3, (1, 4, 9, 4), False),    # 4 heads over 3 ranks: shards of 2, 2 and 0
    (2, (1, 5, 33, 8), True),    # 5 heads: 3 and 2, the gather pads and truncates
])
def test_sharded_forward_backward_match_oracle(world, shape, causal):
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shape, causal, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    B, H, N, d = shape
    for r in range(world):
        ok, so, sl, sk = out[r]
        assert ok, f"rank {r}: sharded result differs from the oracle"
        assert so == (B, H, N, d) and sl == (B, H, N) and sk == (B, H, N, d)


def test_single_process_without_group():
    """No process group: one shard holding every head."""
    from exact_attention_115_b200 import sharded

    saved = sharded._fa_forward
    sharded._fa_forward = lambda q, k, v, causal, scale: _oracle_forward(q, k, v, causal, scale)
    try:
        g = torch.Generator().manual_seed(3)
        q, k, v = (torch.randn(2, 2, 5, 4, generator=g, dtype=torch.float64) for _ in range(3))
        O, L = sharded.forward(q, k, v, causal=True)
        O_ref, _ = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), 0.5, True)
        assert np.abs(O.numpy() - O_ref).max() <= 1e-12
    finally:
        sharded._fa_forward = saved


def test_unmergeable_layout_is_rejected():
    from exact_attention_115_b200 import sharded

    q = torch.zeros(2, 8, 3, 4).transpose(0, 1)  # [8, 2, ...] view: B and H do not merge
    with pytest.raises(ValueError):
        sharded._heads_view(q)
