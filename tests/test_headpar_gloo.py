"""Head-parallel attention's exchange logic on CPU with the gloo backend (world
sizes 2 and 4, no GPU): the token-sharded tensors are regrouped by head and
back, and a per-head attention applied in between gives, on every rank, the
full-tensor result sliced to that rank's tokens.  The attention stand-in is a
plain torch CPU function of whole heads (the product passes the library's
CUDA call instead)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _full(B, H, N, d):
    g = torch.Generator().manual_seed(3)
    return [torch.randn(B, H, N, d, generator=g) for _ in range(3)]


def _exact_per_head(q, k, v, w, block, topk):
    # depends on every token of a head (running sums along the sequence) and on
    # the head's own values only; elementwise arithmetic, so bit-reproducible
    return torch.cumsum(q * k, dim=2) + v.flip(2) * 0.5


def _softmax_attn(q, k, v, w, block, topk):
    s = torch.einsum("bhnd,bhmd->bhnm", q.double(), k.double()) / q.shape[-1] ** 0.5
    return torch.einsum("bhnm,bhmd->bhnd", torch.softmax(s, -1), v.double()).float()


def _worker(rank, world, port, ret):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from sparse_bit_attention_smoothing_b200.headpar import gather_heads, sagesla_attn_head_parallel, scatter_heads
        B, H, N, d = 2, 8, 48, 16
        q, k, v = _full(B, H, N, d)
        Nl = N // world
        sl = slice(rank * Nl, (rank + 1) * Nl)
        ql, kl, vl = q[:, :, sl], k[:, :, sl], v[:, :, sl]
        # the regrouping: rank r holds heads [r H/P, (r+1) H/P) over the whole sequence
        qh = scatter_heads(ql)
        Hp = H // world
        ok_scatter = torch.equal(qh, q[:, rank * Hp:(rank + 1) * Hp])
        ok_round = torch.equal(gather_heads(qh), ql)
        # per-head attention in between equals the full-tensor result on this rank's tokens
        y = sagesla_attn_head_parallel(ql, kl, vl, attn=_exact_per_head)
        ok_exact = torch.equal(y, _exact_per_head(q, k, v, None, 64, 1.0)[:, :, sl])
        y2 = sagesla_attn_head_parallel(ql, kl, vl, attn=_softmax_attn)
        err = float((y2 - _softmax_attn(q, k, v, None, 64, 1.0)[:, :, sl]).abs().max())
        try:  # a head count the ranks do not divide is refused before any exchange
            scatter_heads(torch.zeros(1, world + 1, Nl, d))
            ok_refuse = False
        except ValueError:
            ok_refuse = True
        ret[rank] = (ok_scatter and ok_refuse, ok_round, ok_exact, err)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_parallel_exchange(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    ret = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, ret)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    for r in range(world):
        ok_scatter, ok_round, ok_exact, err = ret[r]
        assert ok_scatter and ok_round and ok_exact, (r, ret[r])
        assert err < 1e-6, (r, err)


def test_single_process_is_identity_and_shapes_are_checked():
    from sparse_bit_attention_smoothing_b200.headpar import gather_heads, sagesla_attn_head_parallel, scatter_heads
    q, k, v = _full(1, 3, 10, 4)
    assert torch.equal(scatter_heads(q), q) and torch.equal(gather_heads(q), q)
    assert torch.equal(sagesla_attn_head_parallel(q, k, v, attn=_exact_per_head), _exact_per_head(q, k, v, None, 64, 1))
