"""GPU parity on the five synthetic workloads at full size, in the launch
configuration the benchmark times: adaLN modulation and the gated residual are
checked on every element, standalone 3D-RoPE on every element, and the fused
3D-RoPE attention on sampled query rows (first, last, the whole ragged last tile
of each sequence, plus random rows), for which the oracle's value is exact."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_video_b200 import dit3d, workloads as wl
from tests.helpers import check_attention, check_modulation, f64, from_dev, half_ulp_bf16, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=list(wl.WORKLOADS))
def case(request):
    w = wl.get_workload(request.param)
    inp = wl.make_inputs(w, seed=0)
    yield w, inp
    torch.cuda.empty_cache()


def test_workload_modulation_and_residual(case):
    w, inp = case
    rpg = w.rows_per_group
    x = to_dev(inp["x"])
    for ps in range(w.param_sets):
        prm = wl.make_inputs(w, seed=0, which=("gamma", "beta", "alpha"), param_set=ps)
        u = dit3d.dit_adaln_modulate(x, to_dev(prm["gamma"]), to_dev(prm["beta"]), rpg)
        ref = oracle.adaln_modulate(f64(inp["x"]), f64(prm["gamma"]), f64(prm["beta"]), rpg)
        check_modulation(from_dev(u), ref, f"{w.name} modulate set {ps}")
        del u, ref
        y = to_dev(inp["y"])
        r = dit3d.dit_gated_residual(x, y, to_dev(prm["alpha"]), rpg)
        ref = oracle.gated_residual(f64(inp["x"]), f64(inp["y"]), f64(prm["alpha"]), rpg)
        check_modulation(from_dev(r), ref, f"{w.name} residual set {ps}")
        del r, ref
    z = torch.zeros(w.groups, w.d_model, dtype=torch.bfloat16, device="cuda")
    r0 = dit3d.dit_gated_residual(x, to_dev(inp["y"]), z, rpg)
    assert torch.equal(r0.view(torch.int16), x.view(torch.int16)), "alpha = 0 must be the identity"


def test_workload_rope(case):
    w, inp = case
    desc = dit3d.rope_desc(w.grid_h, w.grid_w, w.bands, w.base)
    cu = w.cu_seqlens
    qo, _ = dit3d.dit_rope3d_qk(to_dev(inp["q"]), None, desc,
                                cu_seqlens=cu if w.varlen else None, n_seq=w.n_seq)
    ref = oracle.rope3d(f64(inp["q"]), cu, w.grid_h, w.grid_w, w.bands, w.base)
    err = np.abs(from_dev(qo) - ref)
    assert (err <= half_ulp_bf16(ref) * 1.01 + 1e-6).all(), err.max()


def test_workload_attention_sampled(case):
    w, inp = case
    desc = dit3d.rope_desc(w.grid_h, w.grid_w, w.bands, w.base)
    cu = w.cu_seqlens
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    o, lse = dit3d.dit_attn_fwd(q, k, v, n_seq=w.n_seq, cu_seqlens=cu if w.varlen else None,
                                rope=desc, return_lse=True)
    dit3d.dit_check_device()
    rows = wl.sample_rows(w, per_seq=256)
    if w.name == "tiny":
        rows = np.arange(w.rows)
    ref_o, ref_lse = oracle.attn_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), cu,
                                     qrows=rows, rope=w.rope_desc())
    got = from_dev(o[torch.from_numpy(rows).cuda()])
    check_attention(got, ref_o, f"{w.name} attention")
    got_lse = lse[torch.from_numpy(rows).cuda()].cpu().double().numpy()
    np.testing.assert_allclose(got_lse, ref_lse, atol=2e-2)


def test_workload_attention_product_step_equals_fused(case):
    # the benchmark's step rotates q and k in one pass and attends over the rotated
    # operands; the rotation is the same fp32 arithmetic, so the output has the same bits
    w, inp = case
    desc = dit3d.rope_desc(w.grid_h, w.grid_w, w.bands, w.base)
    cu = w.cu_seqlens if w.varlen else None
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    o_fused = dit3d.dit_attn_fwd(q, k, v, n_seq=w.n_seq, cu_seqlens=cu, rope=desc)
    qr, kr = dit3d.dit_rope3d_qk(q, k, desc, n_seq=w.n_seq, cu_seqlens=cu)
    o_step = dit3d.dit_attn_fwd(qr, kr, v, n_seq=w.n_seq, cu_seqlens=cu)
    dit3d.dit_check_device()
    assert torch.equal(o_fused, o_step)


def test_workload_linear_sampled_and_euler(case):
    w, inp = case
    D, rows, rpg = w.d_model, w.rows, w.rows_per_group
    rng = np.random.default_rng(41)
    x = to_dev(inp["x"])
    sample = np.unique(np.concatenate([[0, rows - 1], np.arange(max(rows - 130, 0), rows, 7),
                                       rng.integers(0, rows, 24)]))
    # QKV-shaped projection with bias
    wq = wl.f32_to_bf16_bits((rng.standard_normal((3 * D, D)) * D ** -0.5).astype(np.float32))
    bq = wl.f32_to_bf16_bits((rng.standard_normal(3 * D) * 0.1).astype(np.float32))
    y = dit3d.dit_linear(x, to_dev(wq), bias=to_dev(bq))
    dit3d.dit_check_device()
    got = from_dev(y[torch.from_numpy(sample).cuda()])
    del y
    ref = oracle.linear(f64(inp["x"][sample]), f64(wq), bias=f64(bq))
    check_modulation(got, ref, f"{w.name} qkv projection")
    # output projection with the gate fused, written over the residual
    wo = wl.f32_to_bf16_bits((rng.standard_normal((D, D)) * D ** -0.5).astype(np.float32))
    alpha = wl.make_inputs(w, seed=0, which=("alpha",))["alpha"]
    h = to_dev(inp["y"])
    res = x.clone()
    dit3d.dit_linear(h, to_dev(wo), residual=res, alpha=to_dev(alpha), rows_per_group=rpg, out=res)
    dit3d.dit_check_device()
    got = from_dev(res[torch.from_numpy(sample).cuda()])
    ref = oracle.linear(f64(inp["y"][sample]), f64(wo), res=f64(inp["x"][sample]),
                        alpha=f64(alpha[sample // rpg]), rows_per_group=1)
    check_modulation(got, ref, f"{w.name} gated output projection")
    # one Euler step per frame on the whole latent
    frame = w.grid_h * w.grid_w
    dt = rng.uniform(0.0, 0.1, rows // frame).astype(np.float32)
    xn = dit3d.dit_flow_euler_step(x, h, torch.from_numpy(dt).cuda(), frame)
    dit3d.dit_check_device()
    ref = oracle.flow_euler_step(f64(inp["x"]), f64(inp["y"]), dt.astype(np.float64), frame)
    check_modulation(from_dev(xn), ref, f"{w.name} euler step")


def test_workload_fp8_attention_sampled(case):
    # the FP8 modes at full size, operands rotated by the RoPE pass as the bench runs them
    w, inp = case
    if w.head_dim != 128:
        pytest.skip("the E4M3 attention modes take head_dim 128")
    from tests.test_gpu_fp8 import FP8_MAX, FP8_MEAN
    desc = dit3d.rope_desc(w.grid_h, w.grid_w, w.bands, w.base)
    cu = w.cu_seqlens
    cu_arg = cu if w.varlen else None
    qr, kr = dit3d.dit_rope3d_qk(to_dev(inp["q"]), to_dev(inp["k"]), desc, n_seq=w.n_seq,
                                 cu_seqlens=cu_arg)
    inv = 64.0
    q8, k8 = dit3d.dit_quantize_e4m3(qr, inv), dit3d.dit_quantize_e4m3(kr, inv)
    v = to_dev(inp["v"])
    v8 = dit3d.dit_quantize_e4m3(v, inv)
    o_qk8 = dit3d.dit_attn_fwd_qk8(q8, k8, v, 1 / inv, 1 / inv, n_seq=w.n_seq, cu_seqlens=cu_arg)
    o_fp8 = dit3d.dit_attn_fwd_fp8(q8, k8, v8, 1 / inv, 1 / inv, 1 / inv, n_seq=w.n_seq,
                                   cu_seqlens=cu_arg)
    dit3d.dit_check_device()
    del q8, k8, v8, qr, kr
    rows = wl.sample_rows(w, per_seq=32)
    idx = torch.from_numpy(rows).cuda()
    rope_kw = w.rope_desc()
    ref, _ = oracle.attn_fwd_qk8(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), cu, 1 / inv,
                                 1 / inv, qrows=rows, rope=rope_kw)
    check_attention(from_dev(o_qk8[idx]), ref, f"{w.name} qk8 attention")
    v_q = oracle.quantize_e4m3(f64(inp["v"]), inv) / inv
    ref8, _ = oracle.attn_fwd_qk8(f64(inp["q"]), f64(inp["k"]), v_q, cu, 1 / inv, 1 / inv,
                                  qrows=rows, rope=rope_kw)
    err = np.abs(from_dev(o_fp8[idx]) - ref8)
    assert err.max() <= FP8_MAX and err.mean() <= FP8_MEAN, (w.name, err.max(), err.mean())
