"""The allocation-free attention entry point, dit_attn_fwd_noalloc.

Some callers cannot allocate device memory while they run -- processes that hand
all GPU memory to their own pool up front, memory-capped serving workers, or
latency-critical paths that cannot take cudaMalloc's implicit synchronisation.
dit_attn_fwd caches its 3D-RoPE table with cudaMalloc on first use; the
allocation-free call keeps that table in a fixed device array that ships with the
library instead, written by the same fill kernel on the call's stream.

These tests call both entry points through the C ABI on the same inputs and require
the same bits: on calls that each wait for the GPU, and on two calls with different
RoPE descriptors queued back to back on one stream (the second must rewrite the
shared array after the first has read it), for both attention kernels. One output is
also compared with the fp64 oracle, and the free device memory must not change over
a call with a descriptor no call has used before.

This file is named to be collected last, and passes alone in a fresh process as
well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_video_b200 import dit3d, workloads as wl
from tests.helpers import check_attention, f64, from_dev

pytestmark = pytest.mark.gpu


def _case(lens, H, d, seed):
    rng = np.random.default_rng(seed)
    rows = int(sum(lens))
    bits = [wl.f32_to_bf16_bits(rng.standard_normal((rows, H, d)).astype(np.float32))
            for _ in range(3)]
    dev = [torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda() for b in bits]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return bits, dev, cu


class Call:
    """Buffers and arguments of one raw C-ABI attention call, made before any call."""

    def __init__(self, dev, cu, desc):
        self.q, self.k, self.v = dev
        rows, H, d = self.q.shape
        self.shape = (rows, H, d)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(rows, H, dtype=torch.float32, device="cuda")
        self.cu_host = (ctypes.c_int32 * len(cu))(*[int(c) for c in cu])
        self.cu_dev = torch.from_numpy(cu).cuda()
        self.n_seq = len(cu) - 1
        self.desc = desc

    def run(self, entry):
        rows, H, d = self.shape
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        status = getattr(dit3d.lib(), entry)(p(self.q), p(self.k), p(self.v), p(self.o),
                                             p(self.lse), rows, H, d, self.n_seq, p(self.cu_dev),
                                             self.cu_host, 0.0, ctypes.byref(self.desc), stream)
        assert status == 0, dit3d.lib().dit_status_string(status)

    def result(self):
        return self.o.clone(), self.lse.clone()


def _synced(call, entry):
    call.run(entry)
    torch.cuda.synchronize()
    assert dit3d.lib().dit_check_device(None) == 0
    return call.result()


CASES = [
    # packed sequences of 5x6 patch frames, bands 44/42/42, offsets
    (dict(lens=[7 * 30, 2 * 30, 13 * 30], H=3, d=128, seed=1),
     dit3d.rope_desc(5, 6, (44, 42, 42), 10000.0, (0, 1, 2))),
    # one sequence on another grid and band split, head_dim 64
    (dict(lens=[4 * 48], H=2, d=64, seed=2),
     dit3d.rope_desc(6, 8, (16, 24, 24), 500.0, (3, 0, 0))),
]


def test_noalloc_allocates_nothing_and_matches_the_oracle():
    # load the library's kernels on this device first (the fill kernel and the attention
    # kernel, through the allocating entry point and a descriptor of its own), so that
    # what follows measures the allocation-free call alone
    args, desc = CASES[0]
    bits, dev, cu = _case(**args)
    warm = Call(dev, cu, dit3d.rope_desc(5, 6, (44, 42, 42), 9000.0))
    _synced(warm, "dit_attn_fwd")
    fresh = Call(dev, cu, dit3d.rope_desc(5, 6, (44, 42, 42), 7777.0, (4, 0, 1)))
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    fresh.run("dit_attn_fwd_noalloc")
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, (free_before, free_after)
    assert dit3d.lib().dit_check_device(None) == 0
    o_na, lse_na = fresh.result()
    o_ref, lse_ref = _synced(fresh, "dit_attn_fwd")
    assert torch.equal(o_na, o_ref) and torch.equal(lse_na, lse_ref)
    # first and last rows of each packed sequence, and random rows
    rows = np.unique(np.concatenate([[0, 209, 210, 269, 270, cu[-1] - 1],
                                     np.random.default_rng(3).integers(0, cu[-1], 40)]))
    ref_o, _ = oracle.attn_fwd(f64(bits[0]), f64(bits[1]), f64(bits[2]), cu, qrows=rows,
                               rope=dict(grid_h=5, grid_w=6, bands=(44, 42, 42), base=7777.0,
                                         offsets=(4, 0, 1)))
    check_attention(from_dev(o_na[torch.from_numpy(rows).cuda()]), ref_o, "noalloc vs oracle")


@pytest.mark.parametrize("variant", [0, 1])
def test_noalloc_matches_the_allocating_entry_point_on_two_calls(variant):
    dit3d.dit_set_attn_variant(variant)
    try:
        for args, desc in CASES:
            if variant == 1 and args["d"] != 128:
                continue  # the CTA-pair kernel takes head_dim 128
            _, dev, cu = _case(**args)
            call = Call(dev, cu, desc)
            o_ref, lse_ref = _synced(call, "dit_attn_fwd")
            for _ in range(2):
                o_na, lse_na = _synced(call, "dit_attn_fwd_noalloc")
                assert torch.equal(o_na, o_ref) and torch.equal(lse_na, lse_ref)
    finally:
        dit3d.dit_set_attn_variant(0)


@pytest.mark.parametrize("variant", [0, 1])
def test_noalloc_calls_queued_on_one_stream(variant):
    # two allocation-free calls with different descriptors, queued back to back before a
    # single synchronisation: the second call's table fill runs after the first call's
    # attention has read the array, so both match the allocating entry point
    dit3d.dit_set_attn_variant(variant)
    try:
        _, dev_a, cu_a = _case(lens=[3 * 30, 9 * 30], H=2, d=128, seed=7)
        _, dev_b, cu_b = _case(lens=[5 * 56], H=3, d=128, seed=8)
        a = Call(dev_a, cu_a, dit3d.rope_desc(5, 6, (44, 42, 42), 10000.0, (1, 2, 3)))
        b = Call(dev_b, cu_b, dit3d.rope_desc(7, 8, (32, 48, 48), 2000.0))
        torch.cuda.synchronize()
        a.run("dit_attn_fwd_noalloc")
        b.run("dit_attn_fwd_noalloc")
        torch.cuda.synchronize()
        assert dit3d.lib().dit_check_device(None) == 0
        got_a, got_b = a.result(), b.result()
        ref_a, ref_b = _synced(a, "dit_attn_fwd"), _synced(b, "dit_attn_fwd")
        for got, ref in ((got_a, ref_a), (got_b, ref_b)):
            assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    finally:
        dit3d.dit_set_attn_variant(0)


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
