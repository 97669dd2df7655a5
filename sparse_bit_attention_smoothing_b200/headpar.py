"""Head-parallel SageSLA attention over several GPUs (one process per GPU).

The community's top request for the reference system is multi-GPU parallel
inference ("thu-ml/TurboDiffusion" radar page, §四 维护者现在最想要的帮助:
多卡并行推理).  A DiT that splits the token sequence over P ranks holds, on
rank r, the tokens [r N/P, (r+1) N/P) of every head.  Attention needs every
token of a head together, and the heads are independent problems, so an
all-to-all regroups the shards by head (each rank gets H/P whole heads), the
path runs on those heads, and a second all-to-all returns the outputs to the
token split:

    [B, H, N/P, d] --all-to-all--> [B, H/P, N, d] --sagesla_attn--> [B, H/P, N, d]
                   --all-to-all--> [B, H, N/P, d]

Every step of the attention runs in the library's kernels on whole heads, so
the result on rank r equals the single-GPU call on the full tensors, sliced
to r's tokens (bit for bit: the kernels compute each head independently).
The exchanges use torch.distributed (NCCL over NVLink on GPUs, gloo on CPU in
the tests); this module holds only the layout logic.
"""
from __future__ import annotations


def _world(group):
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def scatter_heads(x, group=None):
    """[B, H, Nl, d] token shard (all heads) -> [B, H/P, P*Nl, d] whole sequences of this rank's heads.

    Rank r receives heads [r H/P, (r+1) H/P); the tokens are concatenated in rank order."""
    import torch
    import torch.distributed as dist
    P, _ = _world(group)
    B, H, Nl, d = x.shape
    if H % P:
        raise ValueError(f"head-parallel attention needs the head count ({H}) divisible by the ranks ({P})")
    if P == 1:
        return x.contiguous()
    Hp = H // P
    send = x.reshape(B, P, Hp, Nl, d).permute(1, 0, 2, 3, 4).contiguous()  # [dest rank][B][Hp][Nl][d]
    recv = torch.empty_like(send)                                          # [source rank][B][Hp][Nl][d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, Hp, P * Nl, d)


def gather_heads(y, group=None):
    """Inverse of scatter_heads: [B, H/P, P*Nl, d] -> [B, H, Nl, d]."""
    import torch
    import torch.distributed as dist
    P, _ = _world(group)
    if P == 1:
        return y.contiguous()
    B, Hp, N, d = y.shape
    if N % P:
        raise ValueError(f"sequence length {N} is not divisible by the ranks ({P})")
    Nl = N // P
    send = y.reshape(B, Hp, P, Nl, d).permute(2, 0, 1, 3, 4).contiguous()  # [dest rank (token shard)][B][Hp][Nl][d]
    recv = torch.empty_like(send)                                          # [source rank (head group)][B][Hp][Nl][d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * Hp, Nl, d)


def sagesla_attn_head_parallel(q, k, v, proj_w=None, block: int = 64, topk: float = 0.1, group=None, stream=None,
                               attn=None):
    """SageSLA attention of token-sharded q, k, v ([B, H, N/P, d] on each of the P ranks of `group`).

    Every rank must call it with the same shapes.  `attn(q, k, v, proj_w, block, topk)` computes attention on
    whole heads; by default the library's sagesla_attn (CUDA).  Returns this rank's [B, H, N/P, d] output."""
    if attn is None:
        from . import sagesla_attn

        def attn(qh, kh, vh, w, blk, tk):
            return sagesla_attn(qh, kh, vh, w, block=blk, topk=tk, stream=stream)
    qh, kh, vh = scatter_heads(q, group), scatter_heads(k, group), scatter_heads(v, group)
    out = attn(qh, kh, vh, proj_w, block, topk)
    return gather_heads(out, group)
