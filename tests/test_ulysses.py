"""Ulysses sequence parallelism (DiT page, "Engenharia de inferencia e paralelismo
de contexto: Ulysses, Ring Attention e FP8") on CPU gloo ranks: the two all-to-all
exchanges regroup tokens and heads exactly, and the whole flow -- exchange, 3D-RoPE
on the full sequence, per-head attention, exchange back -- equals attention of the
unsplit sequence. The attention here is the fp64 oracle (test infrastructure); on
GPUs the same exchanges feed dit_rope3d_qk and dit_attn_fwd."""
import itertools
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from diffusion_transformer_video_b200 import ulysses

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "token_grid.json")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _full(N, H, d, seed):
    g = np.random.default_rng(seed)
    return [g.standard_normal((N, H, d)) for _ in range(3)]


def _worker(rank, world, port, q, N, H, d, grid):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n_loc, h_loc = ulysses.ulysses_shapes(N, H, world)
        Q, K, V = _full(N, H, d, 5)
        mine = slice(rank * n_loc, (rank + 1) * n_loc)
        heads = slice(rank * h_loc, (rank + 1) * h_loc)
        # exchange 1: this rank's tokens -> all tokens of this rank's heads
        qh = ulysses.seq_to_head(torch.from_numpy(Q[mine].copy()))
        kh = ulysses.seq_to_head(torch.from_numpy(K[mine].copy()))
        vh = ulysses.seq_to_head(torch.from_numpy(V[mine].copy()))
        exact = bool(np.array_equal(qh.numpy(), Q[:, heads]))
        # round trip
        back = ulysses.head_to_seq(qh)
        round_trip = bool(np.array_equal(back.numpy(), Q[mine]))
        # whole flow: RoPE on the full sequence (global positions), attention per head
        rope = dict(grid_h=grid[0], grid_w=grid[1], bands=(d // 4, d // 4 + d // 8, d // 2 - d // 8),
                    base=10000.0, offsets=(0, 0, 0))
        cu = np.array([0, N], np.int32)
        qr = oracle.rope3d(qh.numpy(), cu, rope["grid_h"], rope["grid_w"], rope["bands"])
        kr = oracle.rope3d(kh.numpy(), cu, rope["grid_h"], rope["grid_w"], rope["bands"])
        oh, _ = oracle.attn_fwd(qr, kr, vh.numpy(), cu)
        o_loc = ulysses.head_to_seq(torch.from_numpy(np.ascontiguousarray(oh))).numpy()
        ref, _ = oracle.attn_fwd(Q, K, V, cu, qrows=np.arange(mine.start, mine.stop), rope=rope)
        err = float(np.abs(o_loc - ref).max())
        q.put((rank, exact, round_trip, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_exchanges_and_attention_equal_the_unsplit_sequence(world):
    N, H, d, grid = 96, 8, 16, (4, 6)       # 4 frames of a 4x6 patch grid
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, N, H, d, grid))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, exact, round_trip, err in res:
        assert exact, f"rank {rank}: seq_to_head is not the head slice of the full tensor"
        assert round_trip, f"rank {rank}: head_to_seq does not invert seq_to_head"
        assert err < 1e-12, f"rank {rank}: split attention differs from the whole by {err}"


def test_ulysses_shapes_match_the_pages_example():
    g = json.load(open(GOLDEN))
    n, h = ulysses.ulysses_shapes(g["tokens"], g["ulysses"]["heads"], g["ulysses"]["gpus"])
    assert (n, h) == (g["ulysses"]["tokens_per_gpu"], g["ulysses"]["heads_per_gpu"])
    with pytest.raises(ValueError):
        ulysses.ulysses_shapes(108000, 24, 7)


def _makespan(lengths, parts):
    return max(sum(int(lengths[i]) ** 2 for i in p) for p in parts)


@pytest.mark.parametrize("seed", range(6))
def test_lpt_assign_is_a_partition_within_four_thirds_of_optimal(seed):
    rng = np.random.default_rng(seed)
    lengths = rng.integers(3, 22, 7) * 1560
    world = 3
    parts = ulysses.lpt_assign(lengths, world)
    assert sorted(i for p in parts for i in p) == list(range(len(lengths)))
    best = min(_makespan(lengths, [[i for i in range(len(lengths)) if a[i] == r] for r in range(world)])
               for a in itertools.product(range(world), repeat=len(lengths)))
    assert _makespan(lengths, parts) <= 4 / 3 * best + 1e-9   # Graham's LPT bound
    assert parts == ulysses.lpt_assign(list(lengths), world)  # deterministic


def test_lpt_assign_small_cases():
    assert ulysses.lpt_assign([5, 4, 3, 3], 2) == [[0, 3], [1, 2]]
    assert ulysses.lpt_assign([1, 1, 1], 4) == [[0], [1], [2], []]


def _varlen_worker(rank, world, port, q, lens):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        N = int(cu[-1])
        Q, K, V = _full(N, 2, 16, 9)
        plans = ulysses.varlen_plan(cu, world)
        mine = plans[rank]
        idx = mine["rows"].numpy()
        # this rank attends over its whole sequences only (the oracle stands in for the kernel)
        o_loc, _ = oracle.attn_fwd(Q[idx], K[idx], V[idx], mine["cu"].numpy())
        full = ulysses.varlen_gather(torch.from_numpy(np.ascontiguousarray(o_loc)), plans, N).numpy()
        ref, _ = oracle.attn_fwd(Q, K, V, cu)
        q.put((rank, float(np.abs(full - ref).max()), sorted(mine["seqs"])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_varlen_sequences_placed_by_lpt_give_the_packed_result(world):
    lens = [40, 7, 64, 1, 33, 20, 50]
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_varlen_worker, args=(r, world, port, q, lens)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    placed = sorted(s for _, _, seqs in res for s in seqs)
    assert placed == list(range(len(lens)))                 # every sequence exactly once
    for rank, err, _ in res:
        assert err == 0.0, f"rank {rank}: gathered output differs from the packed batch by {err}"


def _oracle_attend(rope):
    """The chunk compute of ulysses_attention with the fp64 oracle in place of the
    kernels (RoPE on the whole packed sequences, then attention per sequence)."""
    def attend(qh, kh, vh, layout):
        cu = np.asarray(layout.cu, np.int32)
        qr = oracle.rope3d(qh.numpy(), cu, rope["grid_h"], rope["grid_w"], rope["bands"])
        kr = oracle.rope3d(kh.numpy(), cu, rope["grid_h"], rope["grid_w"], rope["bands"])
        oh, _ = oracle.attn_fwd(qr, kr, vh.numpy(), cu)
        return torch.from_numpy(np.ascontiguousarray(oh))
    return attend


def _chunked_worker(rank, world, port, q, lens, H, d, grid, chunks):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        Q, K, V = _full(int(cu[-1]), H, d, 11)
        layout = ulysses.UlyssesLayout(cu, world)
        mine = layout.local_rows(rank).numpy()
        rope = dict(grid_h=grid[0], grid_w=grid[1], bands=(d // 4, d // 4 + d // 8, d // 2 - d // 8))
        o = ulysses.ulysses_attention(*(torch.from_numpy(np.ascontiguousarray(t[mine]))
                                        for t in (Q, K, V)),
                                      cu_seqlens=cu, head_chunks=chunks,
                                      attend=_oracle_attend(rope))
        ref, _ = oracle.attn_fwd(Q, K, V, cu, qrows=mine, rope=dict(rope, base=10000.0))
        q.put((rank, float(np.abs(o.numpy() - ref).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,lens,chunks", [(2, [96], 2), (2, [48, 24, 72], 2), (4, [96, 48], 2),
                                              (4, [24, 96], 1)])
def test_chunked_ulysses_on_packed_batches_equals_the_unsplit_attention(world, lens, chunks):
    # 4x6 patch frames; each sequence's length a multiple of the rank count; this rank's
    # heads in `chunks` chunks whose exchanges overlap the previous chunk's attention
    H, d, grid = 8, 16, (4, 6)
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_chunked_worker, args=(r, world, port, q, lens, H, d, grid, chunks))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err in res:
        assert err < 1e-12, f"rank {rank}: chunked split attention differs by {err}"


def test_ulysses_layout_places_every_row_once():
    lay = ulysses.UlyssesLayout([0, 8, 20], 2)
    assert lay.rows_local == 10
    assert lay.local_rows(0).tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 12, 13]
    assert lay.local_rows(1).tolist() == [4, 5, 6, 7, 14, 15, 16, 17, 18, 19]
    # gather after the exchange undoes the rank-major order exactly
    received = torch.cat([lay.local_rows(0), lay.local_rows(1)])
    assert received.index_select(0, lay.gather_idx).tolist() == list(range(20))
    with pytest.raises(ValueError):
        ulysses.UlyssesLayout([0, 9], 2)
