"""Ulysses head-sharded attention across the ranks of a process group.

Each rank starts with a token shard of the sequence, every head: q, k, v
[B, N_r, H, D] BF16 views (unit stride over d), ranks holding consecutive
token ranges in rank order (N_r may differ between ranks).  An all-to-all of
Q, K and V gives rank j every token of heads [j*H/W, (j+1)*H/W), in global
token order; attention then runs locally over the whole sequence (no split
of the keys, so no independently normalised partials are merged); a second
all-to-all returns the output to the token shards.  This is the layout of
"State-Ownership Architecture Decision", section "Interface And Future
Ulysses Layout": each rank receives the globally ordered KV sequence before
attention, and outputs land token-major.

The exchange buffers are token-major ([tokens, B, H/W, D]), so the received
Q/K/V and the local output are strided [B, N, H/W, D] views that the C ABI
takes as they are; the packing before the first exchange and the unpacking
after the second are strided copies.  torch.distributed carries the
exchanges (NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def _attend_library(qh, kh, vh, oh, sm_scale):
    import fp8_quantized_exact_b200 as sage
    B, N, H, D = qh.shape
    ws = sage.workspace(sage.SAGE_OP_ATTN_FWD, B, N, H, D, qh.device)
    sage.sage_attn_fwd(qh, kh, vh, oh, sm_scale, ws)
    st = sage.sage_read_device_status(ws)
    if st != sage.SAGE_OK:
        raise sage.SageError(st, "ulysses local attention")


def shard_counts(n_local: int, group=None, device=None) -> list:
    """Token counts of every rank, in rank order."""
    world = dist.get_world_size(group)
    t = torch.tensor([n_local], dtype=torch.int64, device=device)
    allc = [torch.zeros_like(t) for _ in range(world)]
    dist.all_gather(allc, t, group=group)
    return [int(c.item()) for c in allc]


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                      sm_scale: float = 0.0, group=None,
                      attend: Optional[Callable] = None) -> None:
    """out[B, N_r, H, D] = attention of this rank's tokens against the whole
    sequence, for every head.  `attend(qh, kh, vh, oh, sm_scale)` computes
    the local heads on [B, N, H/W, D] views (default: sage_attn_fwd)."""
    attend = attend or _attend_library
    W = dist.get_world_size(group)
    B, Nr, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or out.shape != q.shape:
        raise ValueError("q, k, v and out must have the same shape")
    if H % W:
        raise ValueError(f"{H} heads do not split over {W} ranks")
    Hl = H // W
    counts = shard_counts(Nr, group, q.device)
    N = sum(counts)

    def exchange_in(x):
        # send block j = this rank's tokens of rank j's heads, token-major
        send = torch.empty((W, Nr, B, Hl, D), dtype=x.dtype, device=x.device)
        send.copy_(x.unflatten(2, (W, Hl)).permute(2, 1, 0, 3, 4))
        recv = torch.empty((N, B, Hl, D), dtype=x.dtype, device=x.device)
        dist.all_to_all_single(recv, send.view(W * Nr, B, Hl, D), output_split_sizes=counts,
                               input_split_sizes=[Nr] * W, group=group)
        return recv  # [N, B, Hl, D]: every token of the local heads, in global order

    qt, kt, vt = exchange_in(q), exchange_in(k), exchange_in(v)
    ot = torch.empty_like(qt)
    view = lambda t: t.permute(1, 0, 2, 3)  # [B, N, Hl, D], stride_n = B*Hl*D
    attend(view(qt), view(kt), view(vt), view(ot), sm_scale)
    # back to the token shards: rank j gets its own tokens of the local heads
    back = torch.empty((W * Nr, B, Hl, D), dtype=ot.dtype, device=ot.device)
    dist.all_to_all_single(back, ot, output_split_sizes=[Nr] * W, input_split_sizes=counts, group=group)
    out.unflatten(2, (W, Hl)).copy_(back.view(W, Nr, B, Hl, D).permute(2, 1, 0, 3, 4))
