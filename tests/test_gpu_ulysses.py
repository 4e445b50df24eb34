"""The Ulysses attention path on one GPU: a single-rank NCCL group, so both
all-to-all exchanges are copies through NCCL and the result must equal the plain
RoPE pass + attention bit for bit. (The multi-rank data movement is tested on CPU
gloo ranks in test_ulysses.py; every run here has one GPU.)"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from diffusion_transformer_video_b200 import dit3d, ulysses

pytestmark = pytest.mark.gpu


def test_single_rank_ulysses_equals_plain_attention():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        gh, gw, T, H, d = 6, 8, 5, 4, 128
        N = T * gh * gw
        g = torch.Generator(device="cuda").manual_seed(3)
        q, k, v = [torch.randn(N, H, d, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3)]
        desc = dit3d.rope_desc(gh, gw, (44, 42, 42))
        o = ulysses.ulysses_attention(q.clone(), k.clone(), v, rope=desc)
        qr, kr = dit3d.dit_rope3d_qk(q, k, desc)
        ref = dit3d.dit_attn_fwd(qr, kr, v)
        dit3d.dit_check_device()
        assert torch.equal(o, ref)
    finally:
        dist.destroy_process_group()
