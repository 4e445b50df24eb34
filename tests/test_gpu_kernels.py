"""GPU parity of every libdit3d call against the fp64 oracle on small and ragged
cases (several tiles plus a ragged tail), edge cases and error paths. All calls
go through the C ABI via the ctypes binding."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_video_b200 import dit3d, workloads as wl
from tests.helpers import check_attention, check_modulation, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(7)


def bits(shape, std=1.0):
    return wl.f32_to_bf16_bits(RNG.standard_normal(shape).astype(np.float32) * np.float32(std))


# ----------------------------------------------------------------------------- modulation

@pytest.mark.parametrize("rows,D,rpg", [(1, 8, 1), (37, 128, 37), (64, 3072, 16), (20, 5120, 10),
                                        (3, 1032, 1), (5, 9216, 5)])
@pytest.mark.parametrize("s0", [1.0, 0.0])
def test_adaln_modulate_parity(rows, D, rpg, s0):
    x, g, b = bits((rows, D)), bits((rows // rpg, D), 0.1), bits((rows // rpg, D), 0.1)
    out = dit3d.dit_adaln_modulate(to_dev(x), to_dev(g), to_dev(b), rpg, eps=1e-6, scale_offset=s0)
    ref = oracle.adaln_modulate(f64(x), f64(g), f64(b), rpg, 1e-6, s0)
    check_modulation(from_dev(out), ref, f"modulate rows={rows} D={D}")


@pytest.mark.parametrize("rows,D,rpg", [(9000, 3072, 1500), (4000, 5120, 400), (30000, 128, 1000),
                                        (20000, 1032, 20), (16384, 1032, 16384), (10000, 2048, 10000)])
def test_adaln_modulate_large_and_in_place(rows, D, rpg):
    # many rows and groups (ragged widths included), out of place and in place over x; groups
    # of 8192 rows or more take the late form (64 threads per row up to d_model 3072), shorter
    # ones the form with gamma / beta staged in shared memory
    x, g, b = bits((rows, D)), bits((rows // rpg, D), 0.1), bits((rows // rpg, D), 0.1)
    xt = to_dev(x)
    out = dit3d.dit_adaln_modulate(xt, to_dev(g), to_dev(b), rpg)
    ref = oracle.adaln_modulate(f64(x), f64(g), f64(b), rpg)
    check_modulation(from_dev(out), ref, f"modulate rows={rows} D={D}")
    dit3d.dit_adaln_modulate(xt, to_dev(g), to_dev(b), rpg, out=xt)
    dit3d.dit_check_device()
    assert torch.equal(xt, out)


def test_adaln_modulate_in_place_and_constant_rows():
    rows, D = 6, 256
    x = np.repeat(wl.f32_to_bf16_bits(np.linspace(-3, 3, rows, dtype=np.float32))[:, None], D, 1)
    g, b = bits((2, D), 0.1), bits((2, D), 0.1)
    xt = to_dev(x)
    dit3d.dit_adaln_modulate(xt, to_dev(g), to_dev(b), 3, out=xt)
    # a constant row normalises to 0: the output is beta of the row's group, exactly
    np.testing.assert_array_equal(from_dev(xt), np.repeat(f64(b), 3, axis=0))


# ----------------------------------------------------------------------------- residual

@pytest.mark.parametrize("rows,D,rpg", [(1, 8, 1), (64, 128, 64), (33, 3072, 11), (8, 5120, 2),
                                        (2, 10240, 1)])
def test_gated_residual_parity(rows, D, rpg):
    x, y, a = bits((rows, D)), bits((rows, D)), bits((rows // rpg, D), 0.1)
    out = dit3d.dit_gated_residual(to_dev(x), to_dev(y), to_dev(a), rpg)
    ref = oracle.gated_residual(f64(x), f64(y), f64(a), rpg)
    check_modulation(from_dev(out), ref, "residual")


def test_gated_residual_alpha_zero_is_bitwise_identity():
    x, y = bits((50, 3072)), bits((50, 3072), 30.0)
    xt = to_dev(x)
    out = dit3d.dit_gated_residual(xt, to_dev(y), torch.zeros(2, 3072, dtype=torch.bfloat16,
                                                              device="cuda"), 25)
    assert torch.equal(out.view(torch.int16), xt.view(torch.int16))


# ----------------------------------------------------------------------------- Euler step

@pytest.mark.parametrize("rows,D,rpg", [(1, 8, 1), (60, 136, 12), (64, 3072, 16), (21, 5120, 3),
                                        (6, 9216, 2), (0, 64, 1)])
def test_flow_euler_step_parity(rows, D, rpg):
    x, u = bits((rows, D)), bits((rows, D))
    G = max(rows // rpg, 1)
    dt = RNG.uniform(-0.2, 0.2, G).astype(np.float32)
    dt[0] = 0.0  # a frame already at its final time
    out = dit3d.dit_flow_euler_step(to_dev(x), to_dev(u), torch.from_numpy(dt).cuda(), rpg)
    dit3d.dit_check_device()
    if rows == 0:
        return
    got, ref = from_dev(out), oracle.flow_euler_step(f64(x), f64(u), dt.astype(np.float64), rpg)
    check_modulation(got, ref, "euler")
    # zero step: the frame's rows keep their bits
    np.testing.assert_array_equal(out[:rpg].view(torch.int16).cpu().numpy(),
                                  x[:rpg].view(np.int16))


def test_flow_euler_step_in_place_and_errors():
    rows, D, rpg = 48, 1024, 16
    x, u = bits((rows, D)), bits((rows, D))
    dt = torch.tensor([0.1, -0.3, 0.05], dtype=torch.float32, device="cuda")
    xa = to_dev(x)
    ref = dit3d.dit_flow_euler_step(xa, to_dev(u), dt, rpg)
    dit3d.dit_flow_euler_step(xa, to_dev(u), dt, rpg, out=xa)
    assert torch.equal(xa, ref)
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_flow_euler_step(xa, to_dev(u), dt, 5)  # 48 rows do not split into groups of 5
    assert e.value.status == 2
    L = dit3d.lib()
    assert L.dit_flow_euler_step(None, None, None, None, rows, D, rpg, None) == 1


# ----------------------------------------------------------------------------- RoPE

def _rope_ref(v_bits, cu, grid_h, grid_w, bands, base=10000.0, offsets=(0, 0, 0)):
    return oracle.rope3d(f64(v_bits), cu, grid_h, grid_w, bands, base, offsets)


@pytest.mark.parametrize("d,bands,gh,gw,frames,H", [
    (64, (16, 24, 24), 4, 4, [4], 3),
    (128, (44, 42, 42), 3, 5, [2, 7, 1], 3),
    (128, (32, 48, 48), 8, 8, [1, 1], 3),
    (128, (44, 42, 42), 30, 52, [2], 40),   # the 480P row width: 40 heads
    (128, (6, 0, 122), 3, 4, [2, 3], 5),    # empty middle band inside a chunk
    (128, (0, 64, 64), 2, 3, [3], 2),       # empty first band
    (64, (20, 44, 0), 3, 3, [2], 7),        # empty last band
    (64, (2, 2, 60), 2, 2, [5], 1),         # one chunk turned by all three bands
])
def test_rope3d_parity(d, bands, gh, gw, frames, H):
    lens = [f * gh * gw for f in frames]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rows = int(cu[-1])
    q, k = bits((rows, H, d)), bits((rows, H, d))
    desc = dit3d.rope_desc(gh, gw, bands, 10000.0, (1, 2, 3))
    qo, ko = dit3d.dit_rope3d_qk(to_dev(q), to_dev(k), desc, cu_seqlens=cu)
    for got, src in ((qo, q), (ko, k)):
        ref = _rope_ref(src, cu, gh, gw, bands, 10000.0, (1, 2, 3))
        err = np.abs(from_dev(got) - ref)
        # fp32 rotation then one bf16 rounding: within a bf16 half-ulp (+ fp32 slack)
        from tests.helpers import half_ulp_bf16
        assert (err <= half_ulp_bf16(ref) * 1.01 + 1e-6).all(), err.max()


def test_rope3d_dense_in_place_equals_out_of_place():
    gh, gw, T, H, d = 6, 7, 3, 4, 128
    rows = 2 * T * gh * gw
    q, k = bits((rows, H, d)), bits((rows, H, d))
    desc = dit3d.rope_desc(gh, gw, (44, 42, 42))
    qa, ka = dit3d.dit_rope3d_qk(to_dev(q), to_dev(k), desc, n_seq=2)
    qt, kt = to_dev(q), to_dev(k)
    dit3d.dit_rope3d_qk(qt, kt, desc, n_seq=2, inplace=True)
    assert torch.equal(qa, qt) and torch.equal(ka, kt)
    # dense with two sequences == packed layout with the same boundaries
    qp, _ = dit3d.dit_rope3d_qk(to_dev(q), None, desc, cu_seqlens=[0, rows // 2, rows])
    assert torch.equal(qp, qa)


# ----------------------------------------------------------------------------- attention

def _attn_case(lens, H, d, rope=None, q_scale=1.0, same_qk=False, seed=0):
    rng = np.random.default_rng(seed)
    rows = int(sum(lens))
    mk = lambda s=1.0: wl.f32_to_bf16_bits(rng.standard_normal((rows, H, d)).astype(np.float32) * np.float32(s))
    q, k, v = mk(q_scale), mk(), mk()
    if same_qk:
        k = q.copy()
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return q, k, v, cu


def _run_attn(q, k, v, cu, rope_kw=None, varlen=True, n_seq=1):
    desc = dit3d.rope_desc(**rope_kw) if rope_kw else None
    o, lse = dit3d.dit_attn_fwd(to_dev(q), to_dev(k), to_dev(v), n_seq=n_seq,
                                cu_seqlens=cu if varlen else None, rope=desc, return_lse=True)
    dit3d.dit_check_device()
    return from_dev(o), lse.cpu().double().numpy()


@pytest.mark.parametrize("lens,H,d", [([64], 2, 64), ([128], 1, 128), ([300], 2, 128),
                                      ([256], 2, 64), ([1], 1, 128), ([513], 1, 128)])
def test_attn_dense_parity(lens, H, d):
    q, k, v, cu = _attn_case(lens, H, d)
    o, lse = _run_attn(q, k, v, cu, varlen=False)
    ref_o, ref_lse = oracle.attn_fwd(f64(q), f64(k), f64(v), cu)
    check_attention(o, ref_o, f"attn {lens}")
    np.testing.assert_allclose(lse, ref_lse, atol=2e-2)


def test_attn_dense_batch_equals_packed():
    q, k, v, cu = _attn_case([200, 200, 200], 2, 128)
    o_dense, _ = _run_attn(q, k, v, cu, varlen=False, n_seq=3)
    o_pack, _ = _run_attn(q, k, v, cu, varlen=True)
    np.testing.assert_array_equal(o_dense, o_pack)
    ref, _ = oracle.attn_fwd(f64(q), f64(k), f64(v), cu)
    check_attention(o_dense, ref, "batch")


@pytest.mark.parametrize("lens", [[130, 1, 255, 16, 400], [128, 256], [7, 0, 90]])
def test_attn_varlen_parity(lens):
    q, k, v, cu = _attn_case(lens, 2, 128, seed=3)
    o, lse = _run_attn(q, k, v, cu)
    ref_o, ref_lse = oracle.attn_fwd(f64(q), f64(k), f64(v), cu)
    check_attention(o, ref_o, f"varlen {lens}")
    np.testing.assert_allclose(lse, ref_lse, atol=2e-2)


@pytest.mark.parametrize("d,bands,gh,gw,frames", [(64, (16, 24, 24), 4, 4, [4]),
                                                   (128, (44, 42, 42), 3, 5, [9, 2, 20]),
                                                   (128, (32, 48, 48), 16, 16, [1]),
                                                   (128, (6, 0, 122), 3, 4, [11, 2]),
                                                   (128, (2, 4, 122), 3, 3, [30]),
                                                   (64, (2, 2, 60), 4, 4, [9])])
def test_attn_fused_rope_parity(d, bands, gh, gw, frames):
    lens = [f * gh * gw for f in frames]
    q, k, v, cu = _attn_case(lens, 2, d, seed=11)
    rope_kw = dict(grid_h=gh, grid_w=gw, bands=bands, base=10000.0, offsets=(0, 1, 2))
    o, lse = _run_attn(q, k, v, cu, rope_kw)
    ref_o, ref_lse = oracle.attn_fwd(f64(q), f64(k), f64(v), cu, rope=rope_kw)
    check_attention(o, ref_o, "fused rope")
    np.testing.assert_allclose(lse, ref_lse, atol=2e-2)


@pytest.mark.parametrize("d,bands", [(128, (44, 42, 42)), (128, (6, 0, 122)), (128, (2, 4, 122)),
                                     (64, (2, 2, 60))])
def test_attn_fused_rope_equals_rope_then_attn(d, bands):
    gh, gw, frames = 5, 6, [7, 3]
    lens = [f * gh * gw for f in frames]
    q, k, v, cu = _attn_case(lens, 3, d, seed=5)
    desc = dit3d.rope_desc(gh, gw, bands, 10000.0, (2, 1, 3))
    qr, kr = dit3d.dit_rope3d_qk(to_dev(q), to_dev(k), desc, cu_seqlens=cu)
    o_two = dit3d.dit_attn_fwd(qr, kr, to_dev(v), cu_seqlens=cu)
    o_fused = dit3d.dit_attn_fwd(to_dev(q), to_dev(k), to_dev(v), cu_seqlens=cu, rope=desc)
    # both round the rotated operands to bf16 with the same fp32 rotation: identical
    assert torch.equal(o_two, o_fused)


@pytest.mark.parametrize("case", ["sharp_q", "q_equals_k"])
def test_attn_sharpened_softmax(case):
    # unit-normal scores are nearly uniform; sharpen them to exercise the online rescale
    q, k, v, cu = _attn_case([700], 2, 128, q_scale=4.0 if case == "sharp_q" else 1.0,
                             same_qk=(case == "q_equals_k"), seed=9)
    o, lse = _run_attn(q, k, v, cu)
    ref_o, ref_lse = oracle.attn_fwd(f64(q), f64(k), f64(v), cu)
    check_attention(o, ref_o, case)
    np.testing.assert_allclose(lse, ref_lse, atol=5e-2)


def test_attn_softmax_scale_and_invariants():
    q, k, _, cu = _attn_case([333], 2, 64, seed=2)
    ones = np.full((333, 2, 64), 0x3F80, np.uint16)  # bf16(1.0)
    o, _ = _run_attn(q, k, ones, cu)
    np.testing.assert_allclose(o, 1.0, atol=4e-3)  # rows of P sum to one
    vrand = wl.f32_to_bf16_bits(RNG.standard_normal((333, 2, 64)).astype(np.float32))
    o2 = dit3d.dit_attn_fwd(to_dev(q), to_dev(k), to_dev(vrand), softmax_scale=0.05)
    ref, _ = oracle.attn_fwd(f64(q), f64(k), f64(vrand), cu, scale=0.05)
    check_attention(from_dev(o2), ref, "scale")


# ----------------------------------------------------------------------------- errors

def test_validation_errors_return_status():
    x = torch.zeros(4, 16, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(1, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_adaln_modulate(x, g, g, rows_per_group=3)
    assert e.value.status == 2
    q = torch.zeros(10, 1, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_attn_fwd(q, q, q)
    assert e.value.status == 2
    q = torch.zeros(10, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_attn_fwd(q, q, q, cu_seqlens=[0, 6, 5, 10])
    assert e.value.status == 4
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_attn_fwd(q, q, q, rope=dit3d.rope_desc(2, 2, (44, 42, 40)))
    assert e.value.status == 2
    raw = dit3d.lib().dit_attn_fwd(None, None, None, None, None, 10, 1, 128, 1, None, None, 0.0,
                                   None, None)
    assert raw == 1


def test_bounded_wait_reports_timeout_without_hanging():
    q = torch.randn(300, 2, 128, device="cuda").to(torch.bfloat16)
    dit3d.lib().dit_debug_force_timeout(1)
    try:
        dit3d.dit_attn_fwd(q, q, q)
        with pytest.raises(dit3d.DitError) as e:
            dit3d.dit_check_device()
        assert e.value.status == 7
    finally:
        dit3d.lib().dit_debug_force_timeout(0)
    # the context is still usable and the error word was cleared
    o = dit3d.dit_attn_fwd(q, q, q)
    dit3d.dit_check_device()
    assert torch.isfinite(o.float()).all()


def test_a_wait_that_runs_out_reports_timeout():
    # A wait limit of 1 ns: the first wait of the attention kernel that is not already
    # satisfied runs out on its %globaltimer check (not the forced-abort path); the CTA
    # leaves its work mid-pipeline, drains its copies and MMAs, frees tensor memory and
    # raises the error bit, and the context stays usable.
    g = torch.Generator(device="cuda").manual_seed(8)
    q, k, v = [torch.randn(8192, 4, 128, device="cuda", generator=g).to(torch.bfloat16)
               for _ in range(3)]
    ref = dit3d.dit_attn_fwd(q, k, v)
    dit3d.dit_check_device()
    dit3d.lib().dit_debug_wait_limit_ns(1)
    try:
        dit3d.dit_attn_fwd(q, k, v)
        with pytest.raises(dit3d.DitError) as e:
            dit3d.dit_check_device()
        assert e.value.status == 7
    finally:
        dit3d.lib().dit_debug_wait_limit_ns(0)
    o = dit3d.dit_attn_fwd(q, k, v)
    dit3d.dit_check_device()
    assert torch.equal(o, ref)


def test_host_watchdog_returns_while_work_runs_then_reports_success():
    # dit_wait_device polls an event: on an attention that needs milliseconds, a 50 us
    # limit returns DIT_ERR_TIMEOUT without blocking; a generous one then returns OK.
    q = torch.randn(32768, 8, 128, device="cuda").to(torch.bfloat16)
    dit3d.dit_check_device()
    dit3d.dit_attn_fwd(q, q, q)
    with pytest.raises(dit3d.DitError) as e:
        dit3d.dit_wait_device(50)
    assert e.value.status == 7
    dit3d.dit_wait_device(60_000_000)
    # and it reports a kernel that gave up a wait, as dit_check_device does
    dit3d.lib().dit_debug_force_timeout(1)
    try:
        dit3d.dit_attn_fwd(q[:300], q[:300], q[:300])
        with pytest.raises(dit3d.DitError) as e:
            dit3d.dit_wait_device(60_000_000)
        assert e.value.status == 7
    finally:
        dit3d.lib().dit_debug_force_timeout(0)
    dit3d.dit_wait_device(60_000_000)


def test_fma_pipe_exp2_meets_its_error_bound():
    # the E4M3 modes' FMA-pipe exponential against 2^t in fp64: the degree-3 minimax of 2^f
    # on [-1/2, 1/2] has relative error 7.5e-5 (Remez exchange), the split t = j + f and
    # the exponent insertion are exact
    t = torch.cat([torch.linspace(-125.9, 8.0, 400001), torch.arange(-125, 9).float(),
                   torch.tensor([-0.5, 0.5, -1.5, 2.5, 7.999, -125.5, 0.0, 1e-7, -1e-7])]).cuda()
    e = dit3d.dit_debug_exp2_fma(t).double().cpu().numpy()
    ref = np.exp2(t.double().cpu().numpy())
    rel = np.abs(e / ref - 1.0)
    assert rel.max() <= 8e-5, (rel.max(), t.cpu().numpy()[rel.argmax()])
    # at t = -126 the result is subnormal (within 2e-4); below it the input is clamped:
    # positive and at most 2^-125
    at = dit3d.dit_debug_exp2_fma(torch.tensor([-126.0], device="cuda")).double().item()
    assert abs(at / 2.0 ** -126 - 1.0) <= 2e-4
    lo = dit3d.dit_debug_exp2_fma(torch.tensor([-126.7, -200.0, -1e30, float("-inf")],
                                               device="cuda")).double().cpu().numpy()
    assert (lo > 0).all() and (lo <= 2.0 ** -125).all()
    # odd length: the lone last element is evaluated too
    odd = dit3d.dit_debug_exp2_fma(torch.tensor([1.0, 2.0, 3.0], device="cuda")).double().cpu().numpy()
    np.testing.assert_allclose(odd, [2.0, 4.0, 8.0], rtol=8e-5)
