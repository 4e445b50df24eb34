"""Ulysses sequence parallelism for the attention of one long sequence.

"DiT, Flow Matching e 3D Attention: A Engenharia de Video com IA", section
"Engenharia de inferencia e paralelismo de contexto: Ulysses, Ring Attention e
FP8": with P GPUs, each GPU holds
N/P tokens of the sequence; an all-to-all regroups the tensors so that each GPU
holds all N tokens of H/P heads, attention runs locally per head, and a second
all-to-all returns the output to the token split (108,000 tokens on 8 GPUs: 13,500
tokens per GPU; 32 heads: 4 per GPU).

Rank r holds tokens [r N/P, (r+1) N/P) before the exchange and heads
[r H/P, (r+1) H/P) after it. Both exchanges are one ``all_to_all_single`` each
(NCCL over NVLink on GPUs); the data is bf16 and the permutation moves bytes only.
3D-RoPE positions depend on the global token index, so q and k are rotated after
the first exchange, when each rank holds whole sequences.

Packed variable-length batches need no exchange: whole sequences go to ranks by
``lpt_assign`` (longest first onto the least-loaded rank, cost L^2 per sequence).
"""
from __future__ import annotations

import heapq

import torch
import torch.distributed as dist

from . import dit3d


def ulysses_shapes(n_tokens: int, n_heads: int, world: int) -> tuple[int, int]:
    """(tokens per rank before the exchange, heads per rank after it)."""
    if world <= 0 or n_tokens % world or n_heads % world:
        raise ValueError(f"{n_tokens} tokens and {n_heads} heads do not split over {world} ranks")
    return n_tokens // world, n_heads // world


def seq_to_head(x: torch.Tensor, group=None) -> torch.Tensor:
    """[N/P, H, d] (this rank's tokens, all heads) -> [N, H/P, d] (all tokens, this
    rank's heads)."""
    world = dist.get_world_size(group)
    n_loc, H, d = x.shape
    _, h_loc = ulysses_shapes(n_loc * world, H, world)
    # chunk p = this rank's tokens of head group p, sent to rank p
    send = x.reshape(n_loc, world, h_loc, d).permute(1, 0, 2, 3).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # chunk p received = rank p's tokens of this rank's heads: token order
    return recv.reshape(world * n_loc, h_loc, d)


def head_to_seq(o: torch.Tensor, group=None) -> torch.Tensor:
    """[N, H/P, d] (all tokens, this rank's heads) -> [N/P, H, d] (this rank's
    tokens, all heads): the inverse of ``seq_to_head``."""
    world = dist.get_world_size(group)
    N, h_loc, d = o.shape
    n_loc, _ = ulysses_shapes(N, h_loc * world, world)
    send = o.reshape(world, n_loc, h_loc, d).contiguous()   # chunk p = rank p's tokens
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # chunk p received = head group p of this rank's tokens
    return recv.permute(1, 0, 2, 3).reshape(n_loc, world * h_loc, d)


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rope=None,
                      softmax_scale: float = 0.0, group=None) -> torch.Tensor:
    """Attention of one sequence split over the ranks of ``group`` by tokens.

    q, k, v: this rank's [N/P, H, d] bf16 CUDA tensors. Returns this rank's tokens of
    softmax(q_rot k_rot^T * scale) v, [N/P, H, d]. ``rope`` is a ``dit3d.RopeDesc``
    for the whole sequence, or None."""
    qh, kh, vh = seq_to_head(q, group), seq_to_head(k, group), seq_to_head(v, group)
    if rope is not None:
        qh, kh = dit3d.dit_rope3d_qk(qh, kh, rope, inplace=True)
    oh = dit3d.dit_attn_fwd(qh, kh, vh, softmax_scale=softmax_scale)
    return head_to_seq(oh, group)


def lpt_assign(lengths, world: int) -> list[list[int]]:
    """Whole sequences to ranks, longest first onto the least-loaded rank (cost L^2,
    the attention's); ties go to the lower rank. Returns each rank's sequence indices
    in ascending order."""
    if world <= 0:
        raise ValueError("world must be positive")
    heap = [(0, r) for r in range(world)]
    out: list[list[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i)):
        load, r = heapq.heappop(heap)
        out[r].append(i)
        heapq.heappush(heap, (load + int(lengths[i]) ** 2, r))
    return [sorted(s) for s in out]


def varlen_plan(cu_seqlens, world: int):
    """Placement of a packed batch's sequences on `world` ranks (``lpt_assign``).

    Returns, per rank, a dict with ``seqs`` (sequence indices), ``rows`` (the global
    row indices of those sequences, in order, as an int64 tensor) and ``cu`` (the
    packed prefix sums of the local batch, int32)."""
    cu = [int(c) for c in cu_seqlens]
    lens = [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]
    plans = []
    for seqs in lpt_assign(lens, world):
        rows = [torch.arange(cu[s], cu[s + 1], dtype=torch.int64) for s in seqs]
        local_cu = [0]
        for s in seqs:
            local_cu.append(local_cu[-1] + lens[s])
        plans.append({"seqs": seqs,
                      "rows": torch.cat(rows) if rows else torch.zeros(0, dtype=torch.int64),
                      "cu": torch.tensor(local_cu, dtype=torch.int32)})
    return plans


def varlen_gather(out_local: torch.Tensor, plans, total_rows: int, group=None) -> torch.Tensor:
    """Every rank's local rows (in its plan's order) back into the full packed batch,
    on every rank: one all_gather of row blocks padded to the longest rank."""
    world = dist.get_world_size(group)
    width = max(int(p["rows"].numel()) for p in plans)
    pad = torch.zeros((width,) + tuple(out_local.shape[1:]), dtype=out_local.dtype,
                      device=out_local.device)
    pad[: out_local.shape[0]] = out_local
    blocks = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(blocks, pad, group=group)
    full = torch.empty((total_rows,) + tuple(out_local.shape[1:]), dtype=out_local.dtype,
                       device=out_local.device)
    for r, p in enumerate(plans):
        n = int(p["rows"].numel())
        full[p["rows"].to(full.device)] = blocks[r][:n]
    return full
