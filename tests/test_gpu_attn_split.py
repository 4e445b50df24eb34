"""Key-range split of a dense attention launch's last partial wave.

When the work units of a dense batch (a pair of 128-row query tiles of one sequence
and head, one CTA per SM) end in a wave that would leave most SMs idle, those units
run as clusters of 2-8 CTAs, each over a share of the key tiles, which merge their
partial (O, m, l) through distributed shared memory. These tests pin that path
against the fp64 oracle: bf16 and E4M3 kernels, head_dim 64 and 128, a ragged last
key tile, sharpened scores (partial maxima far apart), a launch of whole waves
followed by split units, the log-sum-exp, and a bounded wait that runs out inside a
cluster. Each case checks that the split really ran.
"""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_video_b200 import dit3d
from tests.helpers import check_attention, f64, from_dev, to_dev
from tests.test_gpu_kernels import _attn_case

pytestmark = pytest.mark.gpu


def _last_split() -> int:
    return dit3d.lib().dit_debug_last_attn_split()


def _rows_sample(n_rows, seed, extra=()):
    rng = np.random.default_rng(seed)
    rows = np.concatenate([rng.integers(0, n_rows, 96), np.arange(n_rows - 40, n_rows), extra])
    return np.unique(rows.astype(np.int64))


@pytest.mark.parametrize("lens,H,d,q_scale", [
    ([1024], 6, 128, 1.0),       # 24 units of 8 key tiles: no whole wave, every unit split
    ([1024], 6, 128, 4.0),       # sharpened scores: the shares' maxima differ widely
    ([700, 700], 3, 64, 1.0),    # head_dim 64; 6 key tiles, the last one ragged
    ([1100], 3, 128, 1.0),       # a last pair of query tiles with one empty tile
])
def test_split_parity_against_the_oracle(lens, H, d, q_scale):
    q, k, v, cu = _attn_case(lens, H, d, q_scale=q_scale, seed=31 + len(lens) + H)
    o, lse = dit3d.dit_attn_fwd(to_dev(q), to_dev(k), to_dev(v), n_seq=len(lens),
                                return_lse=True)
    dit3d.dit_check_device()
    assert _last_split() >= 2
    ref_o, ref_lse = oracle.attn_fwd(f64(q), f64(k), f64(v), cu)
    check_attention(from_dev(o), ref_o, f"split {lens} H={H} d={d}")
    np.testing.assert_allclose(lse.cpu().double().numpy(), ref_lse, atol=5e-2 if q_scale > 1 else 2e-2)


def test_split_after_whole_waves():
    # 8 pairs x 19 heads = 152 units: 148 in the first launch, the last 4 (head 18, query
    # rows 1024-2047) split 8 ways over the 16 key tiles
    lens, H, d = [2048], 19, 128
    q, k, v, cu = _attn_case(lens, H, d, seed=41)
    o, lse = dit3d.dit_attn_fwd(to_dev(q), to_dev(k), to_dev(v), return_lse=True)
    dit3d.dit_check_device()
    assert _last_split() >= 2
    rows = _rows_sample(2048, 3, extra=np.arange(1024, 2048, 7))
    ref_o, ref_lse = oracle.attn_fwd(f64(q), f64(k), f64(v), cu, qrows=rows)
    got = from_dev(o)[rows]
    check_attention(got, ref_o, "split after whole waves")
    np.testing.assert_allclose(lse.cpu().double().numpy()[rows], ref_lse, atol=2e-2)
    # the tail units in particular (head 18, rows 1024 on)
    tail = rows >= 1024
    check_attention(got[tail][:, 18], ref_o[tail][:, 18], "split units")


def test_split_matches_the_unsplit_packed_form():
    # the packed form of the same batch never splits: equal within rounding
    q, k, v, cu = _attn_case([1024, 1024], 4, 128, seed=43)
    o_dense = dit3d.dit_attn_fwd(to_dev(q), to_dev(k), to_dev(v), n_seq=2)
    dit3d.dit_check_device()
    assert _last_split() >= 2
    o_pack = dit3d.dit_attn_fwd(to_dev(q), to_dev(k), to_dev(v), cu_seqlens=cu)
    dit3d.dit_check_device()
    assert _last_split() == 1
    diff = (o_dense.float() - o_pack.float()).abs()
    assert float(diff.max()) <= 2 ** -7 and float(diff.mean()) <= 2e-4


def test_split_is_deterministic():
    q, k, v, _ = _attn_case([1024], 6, 128, seed=45)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    a = dit3d.dit_attn_fwd(qd, kd, vd)
    b = dit3d.dit_attn_fwd(qd, kd, vd)
    dit3d.dit_check_device()
    assert _last_split() >= 2 and torch.equal(a, b)


def test_split_e4m3_kernels():
    lens, H = [1024], 6
    q, k, v, cu = _attn_case(lens, H, 128, seed=47)
    inv = 64.0
    q8, k8, v8 = (dit3d.dit_quantize_e4m3(to_dev(t), inv) for t in (q, k, v))
    o = dit3d.dit_attn_fwd_qk8(q8, k8, to_dev(v), 1 / inv, 1 / inv)
    dit3d.dit_check_device()
    assert _last_split() >= 2
    ref, _ = oracle.attn_fwd_qk8(f64(q), f64(k), f64(v), cu, 1 / inv, 1 / inv)
    check_attention(from_dev(o), ref, "split qk8")
    o8 = dit3d.dit_attn_fwd_fp8(q8, k8, v8, 1 / inv, 1 / inv, 1 / inv)
    dit3d.dit_check_device()
    assert _last_split() >= 2
    v_q = oracle.quantize_e4m3(f64(v), inv) / inv
    ref8, _ = oracle.attn_fwd_qk8(f64(q), f64(k), v_q, cu, 1 / inv, 1 / inv)
    err = np.abs(from_dev(o8) - ref8)
    assert err.max() <= 3e-2 and err.mean() <= 4e-3, (err.max(), err.mean())


def test_split_bounded_waits_end_with_an_error_and_no_hang():
    # every CTA of every cluster gives up (forced), or waits run out after 1 ns: the
    # clusters still meet at both barriers of the merge, and the context stays usable
    q, k, v, _ = _attn_case([1024], 6, 128, seed=49)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    ref = dit3d.dit_attn_fwd(qd, kd, vd)
    dit3d.dit_check_device()
    L = dit3d.lib()
    for arm, disarm, must_fail in (
            (lambda: L.dit_debug_force_timeout(1), lambda: L.dit_debug_force_timeout(0), True),
            (lambda: L.dit_debug_wait_limit_ns(1), lambda: L.dit_debug_wait_limit_ns(0), False)):
        arm()
        try:
            dit3d.dit_attn_fwd(qd, kd, vd)
            assert _last_split() >= 2
            # a 1 ns limit fails only the waits not already satisfied when first tried
            status = L.dit_check_device(None)
            assert status == 7 or (status == 0 and not must_fail), status
        finally:
            disarm()
        o = dit3d.dit_attn_fwd(qd, kd, vd)
        dit3d.dit_check_device()
        assert torch.equal(o, ref)
