"""FP8 E4M3 Q K^T (DiT page, "Engenharia de inferencia e paralelismo de contexto:
Ulysses, Ring Attention e FP8"): the quantisation kernel matches the oracle's E4M3
rounding code for code, and the attention over E4M3 q/k matches the oracle's
attention over the same quantised operands."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_video_b200 import dit3d, workloads as wl
from tests.helpers import check_attention, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(51)


def _decode(codes: torch.Tensor) -> np.ndarray:
    return codes.cpu().view(torch.float8_e4m3fn).double().numpy()


@pytest.mark.parametrize("inv_scale", [1.0, 64.0, 0.25, 512.0])
def test_quantize_e4m3_code_for_code(inv_scale):
    n = 3 * 4096 + 8
    mags = 10.0 ** RNG.uniform(-5, 2.5, n)
    x = wl.f32_to_bf16_bits((RNG.choice([-1, 1], n) * mags).astype(np.float32))
    codes = dit3d.dit_quantize_e4m3(to_dev(x), inv_scale)
    dit3d.dit_check_device()
    np.testing.assert_array_equal(_decode(codes), oracle.quantize_e4m3(f64(x), inv_scale))


def _qk8_case(lens, H, seed, scale=64.0):
    rng = np.random.default_rng(seed)
    rows = int(sum(lens))
    mk = lambda: wl.f32_to_bf16_bits(rng.standard_normal((rows, H, 128)).astype(np.float32))
    q, k, v = mk(), mk(), mk()
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return q, k, v, cu


@pytest.mark.parametrize("lens,varlen", [([128], False), ([300], False), ([700, 700], False),
                                         ([130, 1, 255, 16, 400], True), ([1], False)])
def test_attn_qk8_parity(lens, varlen):
    q, k, v, cu = _qk8_case(lens, 2, seed=len(lens) * 7 + lens[0])
    inv = 64.0
    q8, k8 = dit3d.dit_quantize_e4m3(to_dev(q), inv), dit3d.dit_quantize_e4m3(to_dev(k), inv)
    o, lse = dit3d.dit_attn_fwd_qk8(q8, k8, to_dev(v), 1 / inv, 1 / inv,
                                    n_seq=1 if varlen else len(lens),
                                    cu_seqlens=cu if varlen else None, return_lse=True)
    dit3d.dit_check_device()
    ref_o, ref_lse = oracle.attn_fwd_qk8(f64(q), f64(k), f64(v), cu, 1 / inv, 1 / inv)
    check_attention(from_dev(o), ref_o, f"qk8 {lens}")
    np.testing.assert_allclose(lse.cpu().double().numpy(), ref_lse, atol=2e-2)


def test_attn_qk8_after_rope_pass():
    gh, gw, frames = 5, 6, [7, 3]
    lens = [f * gh * gw for f in frames]
    q, k, v, cu = _qk8_case(lens, 3, seed=5)
    desc = dit3d.rope_desc(gh, gw, (44, 42, 42))
    qr, kr = dit3d.dit_rope3d_qk(to_dev(q), to_dev(k), desc, cu_seqlens=cu)
    inv = 64.0
    o = dit3d.dit_attn_fwd_qk8(dit3d.dit_quantize_e4m3(qr, inv), dit3d.dit_quantize_e4m3(kr, inv),
                               to_dev(v), 1 / inv, 1 / inv, cu_seqlens=cu)
    dit3d.dit_check_device()
    rope_kw = dict(grid_h=gh, grid_w=gw, bands=(44, 42, 42))
    ref, _ = oracle.attn_fwd_qk8(f64(q), f64(k), f64(v), cu, 1 / inv, 1 / inv, rope=rope_kw)
    check_attention(from_dev(o), ref, "qk8 after rope")


def test_attn_qk8_errors():
    v = torch.zeros(10, 1, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(10, 1, 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_attn_fwd_qk8(c, c, v, 1.0, 1.0)  # head_dim 64 is not supported
    assert e.value.status == 2
    v = torch.zeros(10, 1, 128, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(10, 1, 128, dtype=torch.uint8, device="cuda")
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_attn_fwd_qk8(c, c, v, 0.0, 1.0)
    assert e.value.status == 2


# E4M3 P in the P V product: each probability is rounded to 3 mantissa bits (relative
# error up to 2^-4, about 2^-4/sqrt(3) rms); over N_eff keys of similar weight the output
# error averages to ~2^-4/sqrt(3) * rms(v) / sqrt(N_eff). With >= 300 keys and unit-normal
# v that is <= 2.1e-3 rms, so the bounds below leave about 4 sigma for the maximum.
FP8_MAX, FP8_MEAN = 3e-2, 4e-3


@pytest.mark.parametrize("lens,varlen", [([300], False), ([700, 700], False),
                                         ([330, 512, 400], True), ([1], False)])
def test_attn_fp8_parity(lens, varlen):
    q, k, v, cu = _qk8_case(lens, 2, seed=len(lens) * 11 + lens[0])
    inv = 64.0
    q8, k8, v8 = (dit3d.dit_quantize_e4m3(to_dev(t), inv) for t in (q, k, v))
    o, lse = dit3d.dit_attn_fwd_fp8(q8, k8, v8, 1 / inv, 1 / inv, 1 / inv,
                                    n_seq=1 if varlen else len(lens),
                                    cu_seqlens=cu if varlen else None, return_lse=True)
    dit3d.dit_check_device()
    v_q = oracle.quantize_e4m3(f64(v), inv) / inv
    ref_o, ref_lse = oracle.attn_fwd_qk8(f64(q), f64(k), v_q, cu, 1 / inv, 1 / inv)
    err = np.abs(from_dev(o) - ref_o)
    assert np.isfinite(err).all()
    assert err.max() <= FP8_MAX and err.mean() <= FP8_MEAN, (err.max(), err.mean())
    # the scores are E4M3 but exact in fp32 accumulation: the LSE keeps the QK8 bound
    np.testing.assert_allclose(lse.cpu().double().numpy(), ref_lse, atol=2e-2)


def test_attn_fp8_single_key_is_exact_v():
    # one key: P = 1 exactly in E4M3, so O is v's dequantised value rounded to bf16
    q, k, v, cu = _qk8_case([1], 3, seed=9)
    inv = 64.0
    q8, k8, v8 = (dit3d.dit_quantize_e4m3(to_dev(t), inv) for t in (q, k, v))
    o = dit3d.dit_attn_fwd_fp8(q8, k8, v8, 1 / inv, 1 / inv, 1 / inv)
    dit3d.dit_check_device()
    v_q = oracle.quantize_e4m3(f64(v), inv) / inv
    np.testing.assert_array_equal(from_dev(o), oracle.round_bf16(v_q))
