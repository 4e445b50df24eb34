"""The Ulysses attention path on one GPU: a single-rank NCCL group, so both
all-to-all exchanges are copies through NCCL. The result is compared with the fp64
oracle's 3D-RoPE attention on sampled rows (the attention tolerances) and must equal
the plain RoPE pass + attention bit for bit. (The multi-rank data movement is tested
on CPU gloo ranks in test_ulysses.py; every run here has one GPU.)"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from diffusion_transformer_video_b200 import dit3d, ulysses
from tests.helpers import check_attention, from_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    yield
    dist.destroy_process_group()


def _check(o, q, k, v, cu, gh, gw, bands, desc):
    # against the oracle: first, last, the ragged last tile of each sequence, random rows
    rows = []
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        rows += [a, b - 1, *range(a + (b - a - 1) // 128 * 128, b)]
    rows = np.unique(np.concatenate([rows, np.random.default_rng(4).integers(0, int(cu[-1]), 64)]))
    q64, k64, v64 = (t.double().cpu().numpy() for t in (q, k, v))
    ref_o, _ = oracle.attn_fwd(q64, k64, v64, np.asarray(cu, np.int32), qrows=rows,
                               rope=dict(grid_h=gh, grid_w=gw, bands=bands))
    check_attention(from_dev(o[torch.from_numpy(rows).cuda()]), ref_o, "ulysses vs oracle")
    # and the same bits as the plain RoPE pass + attention over the packed batch
    cu_arg = None if len(cu) == 2 else np.asarray(cu, np.int32)
    qr, kr = dit3d.dit_rope3d_qk(q, k, desc, cu_seqlens=cu_arg)
    ref = dit3d.dit_attn_fwd(qr, kr, v, cu_seqlens=cu_arg)
    dit3d.dit_check_device()
    assert torch.equal(o, ref)


def test_single_rank_ulysses_equals_plain_attention(nccl_group):
    gh, gw, T, H, d = 6, 8, 5, 4, 128
    N = T * gh * gw
    g = torch.Generator(device="cuda").manual_seed(3)
    q, k, v = [torch.randn(N, H, d, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3)]
    desc = dit3d.rope_desc(gh, gw, (44, 42, 42))
    o = ulysses.ulysses_attention(q.clone(), k.clone(), v, rope=desc)
    dit3d.dit_check_device()
    _check(o, q, k, v, [0, N], gh, gw, (44, 42, 42), desc)


def test_single_rank_ulysses_packed_batch_in_head_chunks(nccl_group):
    # a packed batch (frames 3, 7, 2 of a 5x6 grid) with the heads in two chunks, each
    # chunk's exchange issued before the previous chunk's attention
    gh, gw, frames, H, d = 5, 6, [3, 7, 2], 4, 128
    lens = [f * gh * gw for f in frames]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    g = torch.Generator(device="cuda").manual_seed(5)
    q, k, v = [torch.randn(int(cu[-1]), H, d, device="cuda", generator=g).to(torch.bfloat16)
               for _ in range(3)]
    desc = dit3d.rope_desc(gh, gw, (44, 42, 42))
    o = ulysses.ulysses_attention(q, k, v, rope=desc, cu_seqlens=cu, head_chunks=2)
    dit3d.dit_check_device()
    _check(o, q, k, v, cu, gh, gw, (44, 42, 42), desc)
