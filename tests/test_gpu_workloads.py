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
    rows = wl.sample_rows(w, per_seq=64 if w.name in ("480p", "720p", "varlen") else 256)
    if w.name == "tiny":
        rows = np.arange(w.rows)
    ref_o, ref_lse = oracle.attn_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), cu,
                                     qrows=rows, rope=w.rope_desc())
    got = from_dev(o[torch.from_numpy(rows).cuda()])
    check_attention(got, ref_o, f"{w.name} attention")
    got_lse = lse[torch.from_numpy(rows).cuda()].cpu().double().numpy()
    np.testing.assert_allclose(got_lse, ref_lse, atol=2e-2)
