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


def _e4m3_step(v: np.ndarray) -> np.ndarray:
    """Spacing of E4M3 values at |v| (3 mantissa bits; subnormal step 2^-9)."""
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6)))
    return np.ldexp(1.0, (e - 3).astype(np.int64))


@pytest.mark.parametrize("d,bands,gh,gw,frames,H,q_inv,k_inv,with_k", [
    (128, (44, 42, 42), 5, 6, [7, 3], 3, 64.0, 16.0, True),
    (128, (44, 42, 42), 30, 52, [1], 40, 256.0, 256.0, True),  # the 480P row width
    (64, (16, 24, 24), 4, 4, [2, 1, 3], 2, 1.0, 512.0, True),   # saturation at 448
    (128, (6, 0, 122), 3, 4, [2, 3], 5, 64.0, 0.25, True),      # empty middle band
    (64, (20, 44, 0), 3, 3, [2], 7, 8.0, 1.0, False),           # q only
])
def test_rope3d_e4m3_equals_rope_then_quantize(d, bands, gh, gw, frames, H, q_inv, k_inv, with_k):
    lens = [f * gh * gw for f in frames]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rows = int(cu[-1])
    rng = np.random.default_rng(rows + H)
    mk = lambda: wl.f32_to_bf16_bits(rng.standard_normal((rows, H, d)).astype(np.float32))
    q, k = mk(), mk() if with_k else None
    desc = dit3d.rope_desc(gh, gw, bands, 10000.0, (1, 0, 2))
    qd, kd = to_dev(q), (to_dev(k) if with_k else None)
    q8, k8 = dit3d.dit_rope3d_qk_e4m3(qd, kd, desc, q_inv, k_inv, cu_seqlens=cu)
    qr, kr = dit3d.dit_rope3d_qk(qd, kd, desc, cu_seqlens=cu)
    dit3d.dit_check_device()
    # byte for byte the two-pass route
    assert torch.equal(q8, dit3d.dit_quantize_e4m3(qr, q_inv))
    if with_k:
        assert torch.equal(k8, dit3d.dit_quantize_e4m3(kr, k_inv))
    else:
        assert k8 is None
    # and the oracle's codes of its own rotation rounded to bf16: equal, except where
    # the fp32 and fp64 rotations round to neighbouring bf16 values, one E4M3 step
    for got, src, inv in ((q8, q, q_inv),) + (((k8, k, k_inv),) if with_k else ()):
        rot = oracle.rope3d(f64(src), cu, gh, gw, bands, 10000.0, (1, 0, 2))
        ref = oracle.quantize_e4m3(oracle.round_bf16(rot), inv)
        dec = _decode(got)
        diff = np.abs(dec - ref)
        assert (diff <= _e4m3_step(np.maximum(np.abs(dec), np.abs(ref)))).all()
        assert (diff == 0).mean() > 0.999


def test_rope3d_e4m3_errors():
    desc = dit3d.rope_desc(2, 2, (44, 42, 42))
    q = torch.zeros(8, 1, 128, dtype=torch.bfloat16, device="cuda")
    L = dit3d.lib()
    import ctypes
    args = lambda qi, ki, qo, ko, qs=1.0: (qi, ki, qo, ko, 8, 1, 128, 2, None, None,
                                           ctypes.byref(desc), qs, 1.0, None)
    qp = q.data_ptr()
    # the codes may not overwrite their own (or the other) source
    assert L.dit_rope3d_qk_e4m3(*args(qp, None, qp, None)) == 2
    assert L.dit_rope3d_qk_e4m3(*args(qp, None, qp + 1024, None)) == 2
    out = torch.empty(8, 1, 128, dtype=torch.uint8, device="cuda")
    assert L.dit_rope3d_qk_e4m3(*args(qp, None, out.data_ptr() + 4, None)) == 3  # 8-byte alignment
    assert L.dit_rope3d_qk_e4m3(*args(qp, None, out.data_ptr(), None, float("inf"))) == 2
    assert L.dit_rope3d_qk_e4m3(*args(qp, None, None, None)) == 1
    assert L.dit_rope3d_qk_e4m3(*args(qp, None, out.data_ptr(), None)) == 0
    dit3d.dit_check_device()


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
