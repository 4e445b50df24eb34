"""Ulysses sequence parallelism for the attention of long sequences.

"DiT, Flow Matching e 3D Attention: A Engenharia de Video com IA", section
"Engenharia de inferencia e paralelismo de contexto: Ulysses, Ring Attention e
FP8": with P GPUs, each GPU holds
N/P tokens of the sequence; an all-to-all regroups the tensors so that each GPU
holds all N tokens of H/P heads, attention runs locally per head, and a second
all-to-all returns the output to the token split (108,000 tokens on 8 GPUs: 13,500
tokens per GPU; 32 heads: 4 per GPU).

Rank r holds tokens [r N/P, (r+1) N/P) of every sequence before the exchange and
heads [r H/P, (r+1) H/P) after it. ``ulysses_attention`` takes a batch (dense or
packed, each sequence's length a multiple of P) and splits this rank's heads into
chunks: the all-to-all of chunk c+1 (NCCL over NVLink on GPUs, on NCCL's own stream)
runs while chunk c is rotated and attended, and each chunk's output goes back as soon
as it is ready. The data is bf16 and the permutations move bytes only. 3D-RoPE
positions depend on the token's place in its whole sequence, so q and k are rotated
after the first exchange, when each rank holds whole sequences.

Packed variable-length batches can also be placed whole, with no exchange: whole
sequences go to ranks by ``lpt_assign`` (longest first onto the least-loaded rank,
cost L^2 per sequence).
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


class UlyssesLayout:
    """Token placement of a batch of sequences split over `world` ranks by tokens.

    ``cu_seqlens`` holds the prefix sums of the global sequence lengths (each a
    multiple of `world`). Rank r holds, sequence after sequence, tokens
    [r L_s / P, (r+1) L_s / P) of every sequence s (its `rows_local` rows, in that
    order). After the exchange a rank holds the packed batch in the global order."""

    def __init__(self, cu_seqlens, world: int):
        cu = [int(c) for c in cu_seqlens]
        lens = [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]
        if world <= 0 or any(L % world for L in lens):
            raise ValueError(f"sequence lengths {lens} do not split over {world} ranks")
        loc = [L // world for L in lens]
        cl = [0]
        for n in loc:
            cl.append(cl[-1] + n)
        self.world, self.cu, self.lens, self.loc = world, cu, lens, loc
        self.rows_local, self.rows_global = cl[-1], cu[-1]
        self.identity = len(lens) == 1   # one sequence: rank order is token order
        # packed global row i <- row gather_idx[i] of the received [P * rows_local] block
        self.gather_idx = torch.tensor(
            [p * cl[-1] + j for s in range(len(lens)) for p in range(world)
             for j in range(cl[s], cl[s + 1])], dtype=torch.int64)
        # row (p, j) sent back to rank p <- packed global row scatter_idx[p * rows_local + j]
        self.scatter_idx = torch.tensor(
            [cu[s] + p * loc[s] + i for p in range(world) for s in range(len(lens))
             for i in range(loc[s])], dtype=torch.int64)

    def local_rows(self, rank: int) -> torch.Tensor:
        """Global packed rows that `rank` holds before the exchange, in its order."""
        return self.scatter_idx[rank * self.rows_local:(rank + 1) * self.rows_local]

    def cu_tensor(self) -> torch.Tensor:
        return torch.tensor(self.cu, dtype=torch.int32)


def attend_with_kernels(rope=None, softmax_scale: float = 0.0):
    """The per-chunk compute of ``ulysses_attention`` on the GPU: 3D-RoPE pass and
    attention of the whole (packed) sequences for the chunk's heads."""
    cache = {}

    def attend(qh, kh, vh, layout: UlyssesLayout):
        if "cu" not in cache:
            host = layout.cu_tensor()
            cache["cu"] = (host.to(qh.device), host)
        cu = cache["cu"]
        if rope is not None:
            qh, kh = dit3d.dit_rope3d_qk(qh, kh, rope, cu_seqlens=cu, inplace=True)
        return dit3d.dit_attn_fwd(qh, kh, vh, cu_seqlens=cu, softmax_scale=softmax_scale)
    return attend


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rope=None,
                      softmax_scale: float = 0.0, group=None, cu_seqlens=None,
                      head_chunks: int = 1, attend=None) -> torch.Tensor:
    """Attention of a batch of sequences split over the ranks of ``group`` by tokens.

    q, k, v: this rank's [rows_local, H, d] bf16 CUDA tensors (``UlyssesLayout``:
    its slice of every sequence, sequence after sequence). ``cu_seqlens``: prefix sums
    of the global sequence lengths (None: one sequence of rows_local * P tokens).
    Returns this rank's rows of softmax(q_rot k_rot^T * scale) v, [rows_local, H, d].
    ``rope`` is a ``dit3d.RopeDesc`` for the whole sequences, or None.

    This rank's H/P heads are handled in ``head_chunks`` chunks: the exchange of chunk
    c+1 is issued before chunk c is attended, so it travels while the kernels run, and
    chunk c's output is sent back right after its attention. ``attend(qh, kh, vh,
    layout)`` computes one chunk on the whole sequences (default: the library's RoPE
    pass and attention)."""
    world = dist.get_world_size(group)
    rows_local, H, d = q.shape
    layout = UlyssesLayout(cu_seqlens if cu_seqlens is not None else [0, rows_local * world],
                           world)
    if layout.rows_local != rows_local:
        raise ValueError(f"{rows_local} local rows, the layout needs {layout.rows_local}")
    _, h_loc = ulysses_shapes(layout.rows_global, H, world)
    if head_chunks <= 0 or h_loc % head_chunks:
        raise ValueError(f"{h_loc} heads per rank do not split into {head_chunks} chunks")
    hc = h_loc // head_chunks
    attend = attend_with_kernels(rope, softmax_scale) if attend is None else attend
    dev = q.device
    gidx = layout.gather_idx.to(dev)
    sidx = layout.scatter_idx.to(dev)

    def send_chunk(c):
        # [P, 3, rows_local, hc, d]: block p = this rank's rows of head group p, chunk c
        parts = [x.view(rows_local, world, h_loc, d)[:, :, c * hc:(c + 1) * hc] for x in (q, k, v)]
        send = torch.stack(parts).permute(2, 0, 1, 3, 4).contiguous()
        recv = torch.empty_like(send)
        return recv, dist.all_to_all_single(recv, send, group=group, async_op=True)

    out = torch.empty_like(q)
    out_v = out.view(rows_local, world, h_loc, d)
    pending = send_chunk(0)
    returning = []
    for c in range(head_chunks):
        recv, work = pending
        if c + 1 < head_chunks:
            pending = send_chunk(c + 1)          # travels while chunk c is attended
        work.wait()
        full = recv.permute(1, 0, 2, 3, 4).reshape(3, world * rows_local, hc, d)
        if not layout.identity:
            full = full.index_select(1, gidx)   # packed global order
        oh = attend(full[0].contiguous(), full[1].contiguous(), full[2].contiguous(), layout)
        send_o = oh if layout.identity else oh.index_select(0, sidx)
        send_o = send_o.reshape(world, rows_local, hc, d).contiguous()
        recv_o = torch.empty_like(send_o)
        returning.append((c, recv_o, dist.all_to_all_single(recv_o, send_o, group=group,
                                                            async_op=True)))
    for c, recv_o, work in returning:
        work.wait()
        out_v[:, :, c * hc:(c + 1) * hc] = recv_o.permute(1, 0, 2, 3)
    return out


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
