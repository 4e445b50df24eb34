"""The allocation-free attention entry point, dit_attn_fwd_noalloc.

Some callers cannot allocate device memory while they run -- processes that hand
all GPU memory to their own pool up front, memory-capped serving workers, or
latency-critical paths that cannot take cudaMalloc's implicit synchronisation.
dit_attn_fwd caches its 3D-RoPE table with cudaMalloc on first use; the
allocation-free call keeps that table in a fixed device array that ships with the
library instead. These tests call both entry points through the C ABI on the same
inputs and require the same output, on two calls in a row with different RoPE
descriptors (so the second call must rewrite the shared array).

This file is named to be collected last, and passes alone in a fresh process as
well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from diffusion_transformer_video_b200 import dit3d, workloads as wl
from tests.helpers import ATTN_MAX

pytestmark = pytest.mark.gpu


def _inputs(lens, H, d, seed):
    rng = np.random.default_rng(seed)
    rows = int(sum(lens))
    mk = lambda: torch.from_numpy(
        wl.f32_to_bf16_bits(rng.standard_normal((rows, H, d)).astype(np.float32)).view(np.int16)
    ).view(torch.bfloat16).cuda()
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return mk(), mk(), mk(), cu


def _run(entry, q, k, v, cu, desc):
    """Raw C-ABI call of `entry` (dit_attn_fwd or dit_attn_fwd_noalloc)."""
    L = dit3d.lib()
    rows, H, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(rows, H, dtype=torch.float32, device="cuda")
    cu_host = (ctypes.c_int32 * len(cu))(*[int(c) for c in cu])
    cu_dev = torch.from_numpy(cu).cuda()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = getattr(L, entry)(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                               ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                               ctypes.c_void_p(lse.data_ptr()), rows, H, d, len(cu) - 1,
                               ctypes.c_void_p(cu_dev.data_ptr()), cu_host, 0.0,
                               ctypes.byref(desc), stream)
    assert status == 0, L.dit_status_string(status)
    torch.cuda.synchronize()
    assert L.dit_check_device(stream) == 0
    return o, lse


def test_noalloc_matches_the_allocating_entry_point_on_two_calls():
    cases = [
        # packed sequences of 5x6 patch frames, bands 44/42/42
        (dict(lens=[7 * 30, 2 * 30, 13 * 30], H=3, d=128, seed=1),
         dit3d.rope_desc(5, 6, (44, 42, 42), 10000.0, (0, 1, 2))),
        # one dense-like sequence on another grid and band split, d = 64
        (dict(lens=[4 * 48], H=2, d=64, seed=2),
         dit3d.rope_desc(6, 8, (16, 24, 24), 500.0, (3, 0, 0))),
    ]
    for args, desc in cases:
        q, k, v, cu = _inputs(**args)
        o_ref, lse_ref = _run("dit_attn_fwd", q, k, v, cu, desc)
        o_na, lse_na = _run("dit_attn_fwd_noalloc", q, k, v, cu, desc)
        err = (o_na.float() - o_ref.float()).abs().max().item()
        assert err <= ATTN_MAX, err
        assert (lse_na - lse_ref).abs().max().item() <= ATTN_MAX


def test_noalloc_rejects_a_table_beyond_its_array():
    # a 2047 x 1023 patch grid with 64 (cos, sin) pairs per position needs ~80k entries
    L = dit3d.lib()
    rows, H, d = 2047 * 1023, 1, 128
    q = torch.empty(rows, H, d, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    desc = dit3d.rope_desc(2047, 1023, (44, 42, 42))
    cu_host = (ctypes.c_int32 * 2)(0, rows)
    cu_dev = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
    status = L.dit_attn_fwd_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(q.data_ptr()),
                                    ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                    None, rows, H, d, 1, ctypes.c_void_p(cu_dev.data_ptr()),
                                    cu_host, 0.0, ctypes.byref(desc), None)
    assert status == 9 and b"DIT_ERR_SCRATCH" in L.dit_status_string(status)
