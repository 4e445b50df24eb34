"""Parity of dit_linear (tcgen05 GEMM with bias / GELU / adaLN-Zero gate epilogues)
against the fp64 oracle, on single tiles, ragged M/N/K, several waves of the
persistent grid, and the gate's zero-identity."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_video_b200 import dit3d, workloads as wl
from tests.helpers import check_modulation, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(31)
DEFAULT_VARIANT = 1  # CTA pairs


def bits(shape, std=1.0):
    return wl.f32_to_bf16_bits((RNG.standard_normal(shape) * std).astype(np.float32))


@pytest.fixture(params=[0, 1], ids=["single_cta", "cta_pair"])
def variant(request):
    dit3d.dit_set_linear_variant(request.param)
    yield request.param
    dit3d.dit_set_linear_variant(DEFAULT_VARIANT)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (1, 8, 8), (300, 520, 200), (1000, 1024, 512),
                                   (4096, 768, 1024), (77, 3072, 136)])
@pytest.mark.parametrize("mode", ["plain", "bias_gelu", "gated"])
def test_linear_parity(variant, M, N, K, mode):
    x, w = bits((M, K)), bits((N, K), std=K ** -0.5)
    kw = {}
    ref_kw = {}
    if mode == "bias_gelu":
        b = bits((N,), std=0.5)
        kw = dict(bias=to_dev(b), gelu=True)
        ref_kw = dict(bias=f64(b), act=1)
    elif mode == "gated":
        rpg = next(r for r in (64, 7, 1) if M % r == 0)
        res, alpha = bits((M, N)), bits((M // rpg, N), std=0.5)
        alpha[0] = 0  # the first group's gate is zero: its rows must be the residual's bits
        kw = dict(residual=to_dev(res), alpha=to_dev(alpha), rows_per_group=rpg)
        ref_kw = dict(res=f64(res), alpha=f64(alpha), rows_per_group=rpg)
    out = dit3d.dit_linear(to_dev(x), to_dev(w), **kw)
    dit3d.dit_check_device()
    ref = oracle.linear(f64(x), f64(w), **ref_kw)
    check_modulation(from_dev(out), ref, f"linear {mode} {M}x{N}x{K}")
    if mode == "gated":
        np.testing.assert_array_equal(out[:rpg].view(torch.int16).cpu().numpy(),
                                      res[:rpg].view(np.int16))


def test_linear_in_place_residual_and_errors(variant):
    M, N, K = 256, 512, 256
    x, w, res, alpha = bits((M, K)), bits((N, K), std=K ** -0.5), bits((M, N)), bits((2, N))
    r_dev = to_dev(res)
    ref = dit3d.dit_linear(to_dev(x), to_dev(w), residual=r_dev, alpha=to_dev(alpha), rows_per_group=128)
    dit3d.dit_linear(to_dev(x), to_dev(w), residual=r_dev, alpha=to_dev(alpha), rows_per_group=128,
                     out=r_dev)
    dit3d.dit_check_device()
    assert torch.equal(ref, r_dev)
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_linear(to_dev(x), to_dev(bits((12, K))))  # N % 8 != 0
    assert e.value.status == 2
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_linear(to_dev(x), to_dev(w), residual=r_dev, alpha=to_dev(alpha), rows_per_group=100)
    assert e.value.status == 2
    L = dit3d.lib()
    assert L.dit_linear(None, None, None, None, 1, 8, 8, 0, None, None, 1, None) == 1


def test_linear_variants_agree():
    M, N, K = 700, 1280, 960
    x, w = to_dev(bits((M, K))), to_dev(bits((N, K), std=K ** -0.5))
    outs = []
    for v in (0, 1):
        dit3d.dit_set_linear_variant(v)
        outs.append(dit3d.dit_linear(x, w))
    dit3d.dit_set_linear_variant(DEFAULT_VARIANT)
    dit3d.dit_check_device()
    # same products, fp32 sums in possibly different order: within one bf16 ulp
    diff = (outs[0].float() - outs[1].float()).abs()
    assert (diff <= outs[0].float().abs() * 2 ** -7 + 1e-6).all()
    with pytest.raises(dit3d.DitError):
        dit3d.dit_set_linear_variant(3)


def test_linear_bounded_wait_reports_timeout(variant):
    x = torch.randn(512, 256, device="cuda").to(torch.bfloat16)
    w = torch.randn(512, 256, device="cuda").to(torch.bfloat16)
    dit3d.lib().dit_debug_force_timeout(1)
    try:
        dit3d.dit_linear(x, w)
        with pytest.raises(dit3d.DitError) as e:
            dit3d.dit_check_device()
        assert e.value.status == 7
    finally:
        dit3d.lib().dit_debug_force_timeout(0)
    o = dit3d.dit_linear(x, w)
    dit3d.dit_check_device()
    ref = (x.float() @ w.float().T)
    assert (o.float() - ref).abs().max().item() < 0.5


def test_linear_wait_that_runs_out_reports_timeout():
    # single-CTA GEMM with a wait limit of 1 ns: a wait runs out mid-pipeline (the CTA-pair
    # form keeps its 2 s limit)
    g = torch.Generator(device="cuda").manual_seed(9)
    x = torch.randn(4096, 2048, device="cuda", generator=g).to(torch.bfloat16)
    w = torch.randn(4096, 2048, device="cuda", generator=g).to(torch.bfloat16)
    dit3d.dit_set_linear_variant(0)
    try:
        ref = dit3d.dit_linear(x, w)
        dit3d.dit_check_device()
        dit3d.lib().dit_debug_wait_limit_ns(1)
        try:
            dit3d.dit_linear(x, w)
            with pytest.raises(dit3d.DitError) as e:
                dit3d.dit_check_device()
            assert e.value.status == 7
        finally:
            dit3d.lib().dit_debug_wait_limit_ns(0)
        o = dit3d.dit_linear(x, w)
        dit3d.dit_check_device()
        assert torch.equal(o, ref)
    finally:
        dit3d.dit_set_linear_variant(DEFAULT_VARIANT)


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (300, 520, 208), (1000, 1024, 512), (77, 3072, 144)])
@pytest.mark.parametrize("mode", ["plain", "bias_gelu", "gated"])
def test_linear_fp8_parity(variant, M, N, K, mode):
    x, w = bits((M, K)), bits((N, K), std=K ** -0.5)
    inv_x, inv_w = 16.0, 256.0
    x8 = dit3d.dit_quantize_e4m3(to_dev(x), inv_x)
    w8 = dit3d.dit_quantize_e4m3(to_dev(w), inv_w)
    kw, ref_kw = {}, {}
    if mode == "bias_gelu":
        b = bits((N,), std=0.5)
        kw, ref_kw = dict(bias=to_dev(b), gelu=True), dict(bias=f64(b), act=1)
    elif mode == "gated":
        rpg = next(r for r in (64, 7, 1) if M % r == 0)
        res, alpha = bits((M, N)), bits((M // rpg, N), std=0.5)
        kw = dict(residual=to_dev(res), alpha=to_dev(alpha), rows_per_group=rpg)
        ref_kw = dict(res=f64(res), alpha=f64(alpha), rows_per_group=rpg)
    out = dit3d.dit_linear_fp8(x8, w8, 1 / inv_x, 1 / inv_w, **kw)
    dit3d.dit_check_device()
    xd = oracle.quantize_e4m3(f64(x), inv_x) / inv_x
    wd = oracle.quantize_e4m3(f64(w), inv_w) / inv_w
    ref = oracle.linear(xd, wd, **ref_kw)
    check_modulation(from_dev(out), ref, f"linear fp8 {mode} {M}x{N}x{K}")


def test_linear_fp8_variants_agree():
    M, N, K = 700, 1280, 960
    x8 = dit3d.dit_quantize_e4m3(to_dev(bits((M, K))), 16.0)
    w8 = dit3d.dit_quantize_e4m3(to_dev(bits((N, K), std=K ** -0.5)), 256.0)
    outs = []
    try:
        for v in (0, 1):
            dit3d.dit_set_linear_variant(v)
            outs.append(dit3d.dit_linear_fp8(x8, w8, 1 / 16, 1 / 256))
    finally:
        dit3d.dit_set_linear_variant(DEFAULT_VARIANT)
    dit3d.dit_check_device()
    diff = (outs[0].float() - outs[1].float()).abs()
    assert (diff <= outs[0].float().abs() * 2 ** -7 + 1e-6).all()


def test_linear_fp8_errors():
    x8 = torch.zeros(64, 40, dtype=torch.uint8, device="cuda")
    w8 = torch.zeros(64, 40, dtype=torch.uint8, device="cuda")
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_linear_fp8(x8, w8, 1.0, 1.0)  # K = 40 is not a multiple of 16
    assert e.value.status == 2
    x8 = torch.zeros(64, 64, dtype=torch.uint8, device="cuda")
    w8 = torch.zeros(64, 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_linear_fp8(x8, w8, -1.0, 1.0)
    assert e.value.status == 2
