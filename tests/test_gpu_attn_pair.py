"""Parity of the CTA-pair attention kernel (dit_set_attn_variant(1): two SMs share
each tcgen05 MMA, each loading and rotating half of every K tile) against the fp64
oracle, on the same cases as the single-CTA kernel, and bit-equality of the two
variants where both use the same rounding steps."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_video_b200 import dit3d
from tests.helpers import check_attention, f64, from_dev, to_dev
from tests.test_gpu_kernels import _attn_case, _run_attn

pytestmark = pytest.mark.gpu


@pytest.fixture
def pair_variant():
    dit3d.dit_set_attn_variant(1)
    yield
    dit3d.dit_set_attn_variant(0)


@pytest.mark.parametrize("lens", [[128], [300], [513], [1], [130, 1, 255, 16, 400], [7, 0, 90],
                                  [1024, 600]])
def test_pair_attn_parity(pair_variant, lens):
    q, k, v, cu = _attn_case(lens, 2, 128, seed=21)
    o, lse = _run_attn(q, k, v, cu)
    ref_o, ref_lse = oracle.attn_fwd(f64(q), f64(k), f64(v), cu)
    check_attention(o, ref_o, f"pair {lens}")
    np.testing.assert_allclose(lse, ref_lse, atol=2e-2)


@pytest.mark.parametrize("gh,gw,frames,bands", [(3, 5, [9, 2, 20], (44, 42, 42)),
                                                (16, 16, [1], (44, 42, 42)),
                                                (30, 52, [3], (44, 42, 42)),
                                                (3, 4, [11, 2], (6, 0, 122)),
                                                (3, 3, [30], (2, 4, 122))])
def test_pair_fused_rope_parity(pair_variant, gh, gw, frames, bands):
    lens = [f * gh * gw for f in frames]
    q, k, v, cu = _attn_case(lens, 2, 128, seed=23)
    rope_kw = dict(grid_h=gh, grid_w=gw, bands=bands, base=10000.0, offsets=(0, 1, 2))
    o, lse = _run_attn(q, k, v, cu, rope_kw)
    ref_o, ref_lse = oracle.attn_fwd(f64(q), f64(k), f64(v), cu, rope=rope_kw)
    check_attention(o, ref_o, "pair fused rope")


def test_pair_dense_batch_and_sharpened(pair_variant):
    q, k, v, cu = _attn_case([700, 700], 2, 128, q_scale=4.0, seed=25)
    o, _ = _run_attn(q, k, v, cu, varlen=False, n_seq=2)
    ref, _ = oracle.attn_fwd(f64(q), f64(k), f64(v), cu)
    check_attention(o, ref, "pair dense sharpened")


def test_variants_agree_bit_for_bit():
    gh, gw, frames = 5, 6, [7, 3, 11]
    lens = [f * gh * gw for f in frames]
    q, k, v, cu = _attn_case(lens, 3, 128, seed=27)
    desc = dit3d.rope_desc(gh, gw, (44, 42, 42))
    outs = []
    for variant in (0, 1):
        dit3d.dit_set_attn_variant(variant)
        try:
            outs.append(dit3d.dit_attn_fwd(to_dev(q), to_dev(k), to_dev(v), cu_seqlens=cu,
                                           rope=desc))
            dit3d.dit_check_device()
        finally:
            dit3d.dit_set_attn_variant(0)
    # the variants differ only in how MMA work is split across SMs; the fp32 sums of a
    # tile may associate differently, so compare within one bf16 ulp
    diff = (outs[0].float() - outs[1].float()).abs()
    scale = outs[0].float().abs().clamp_min(2 ** -20)
    assert (diff <= scale * 2 ** -7 + 1e-6).all(), diff.max().item()


def test_pair_bounded_wait_timeout(pair_variant):
    q = torch.randn(600, 2, 128, device="cuda").to(torch.bfloat16)
    dit3d.lib().dit_debug_force_timeout(1)
    try:
        dit3d.dit_attn_fwd(q, q, q)
        with pytest.raises(dit3d.DitError) as e:
            dit3d.dit_check_device()
        assert e.value.status == 7
    finally:
        dit3d.lib().dit_debug_force_timeout(0)
    o = dit3d.dit_attn_fwd(q, q, q)
    dit3d.dit_check_device()
    assert torch.isfinite(o.float()).all()


def test_variant_values():
    with pytest.raises(dit3d.DitError):
        dit3d.dit_set_attn_variant(2)
