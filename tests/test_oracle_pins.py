"""Pins for the fp64 oracle: closed forms, invariants, library special cases and
brute force on tiny inputs -- never the oracle's own formula retyped.

Each pin names what it would catch (a dropped term, a wrong sign, index or band,
a transposed operand)."""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from diffusion_transformer_video_b200 import workloads as wl

RNG = np.random.default_rng(20261202)


# ----------------------------------------------------------------------------- token grid

def test_token_count_pages_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "token_grid.json")))
    c = g["clip_720p_5s_24fps"]
    assert c["frames"] * c["channels"] * c["height"] * c["width"] == c["pixel_values"]
    lat = g["latent"]
    assert c["frames"] // lat["time_factor"] == lat["T_lat"]
    assert c["height"] // lat["space_factor"] == lat["H_lat"]
    assert c["width"] // lat["space_factor"] == lat["W_lat"]
    p = g["patch"]
    n = oracle.patch_grid_tokens(lat["T_lat"], lat["H_lat"], lat["W_lat"], p["p_t"], p["p_h"],
                                 p["p_w"])
    assert n == g["tokens"] == 108000
    u = g["ulysses"]
    assert n // u["gpus"] == u["tokens_per_gpu"] and n % u["gpus"] == 0
    assert u["heads"] // u["gpus"] == u["heads_per_gpu"]


def test_workload_token_counts(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "workload_tokens.json")))
    for name in ("480p", "720p"):
        e = g[name]
        T = 1 + (e["frames"] - 1) // e["vae"][0]
        H, W = e["pixels"][0] // e["vae"][1], e["pixels"][1] // e["vae"][2]
        assert [T, H, W] == e["latent"]
        assert oracle.patch_grid_tokens(T, H, W, *e["patch"]) == e["tokens"]
    for name in ("tiny", "image"):
        e = g[name]
        assert oracle.patch_grid_tokens(*e["latent"], *e["patch"]) == e["tokens"]
    f = g["varlen_frame"]
    assert (f["latent_frame"][0] // f["patch"][0]) * (f["latent_frame"][1] // f["patch"][1]) \
        == f["tokens_per_frame"]
    for name in ("tiny", "image", "480p", "720p"):
        w = wl.get_workload(name)
        assert w.seqlens[0] == g[name]["tokens"]
    w = wl.get_workload("varlen")
    assert w.frame_tokens == f["tokens_per_frame"]
    assert all(3 <= t <= 21 for t in w.frames) and len(w.frames) == 8


# ----------------------------------------------------------------------------- adaLN

def _ln_torch(x, eps):
    t = torch.from_numpy(np.asarray(x, dtype=np.float64))
    return torch.nn.functional.layer_norm(t, (t.shape[-1],), eps=eps).numpy()


@pytest.mark.parametrize("D", [8, 128, 3072])
def test_adaln_reduces_to_layernorm(D):
    # s0 = 1, gamma = beta = 0 is plain LayerNorm (library routine, no affine).
    rows = 12
    x = RNG.standard_normal((rows, D)) * 3 + 1.5
    z = np.zeros((2, D))
    got = oracle.adaln_modulate(x, z, z, rows_per_group=6, eps=1e-6, scale_offset=1.0)
    np.testing.assert_allclose(got, _ln_torch(x, 1e-6), rtol=0, atol=1e-12)
    # page form gamma*LN(x)+beta with gamma = 1
    got0 = oracle.adaln_modulate(x, np.ones((2, D)), z, rows_per_group=6, eps=1e-6,
                                 scale_offset=0.0)
    np.testing.assert_allclose(got0, got, rtol=0, atol=1e-15)


def test_adaln_scale_offset_forms_agree():
    # gamma_page = 1 + gamma: the two parameterisations are the same map.
    D = 64
    x = RNG.standard_normal((4, D))
    g = RNG.standard_normal((1, D)) * 0.1
    b = RNG.standard_normal((1, D)) * 0.1
    a = oracle.adaln_modulate(x, g, b, 4, scale_offset=1.0)
    c = oracle.adaln_modulate(x, 1.0 + g, b, 4, scale_offset=0.0)
    np.testing.assert_allclose(a, c, atol=1e-14)


def test_adaln_constant_rows_give_beta_of_their_group():
    # LN of a constant row is 0, so u = beta_g exactly: pins g = r // rows_per_group.
    # (values k/4 and D = 16 keep the mean exact in binary)
    D, G, rpg = 16, 5, 3
    x = np.repeat(np.arange(G * rpg, dtype=np.float64)[:, None] * 0.25 - 2.0, D, axis=1)
    gamma = RNG.standard_normal((G, D))
    beta = RNG.standard_normal((G, D))
    got = oracle.adaln_modulate(x, gamma, beta, rpg)
    expect = np.repeat(beta, rpg, axis=0)
    np.testing.assert_array_equal(got, expect)


def test_adaln_alternating_row_closed_form():
    # x = [a, -a, a, -a, ...]: mean 0, biased variance a^2, xhat = +-a / sqrt(a^2 + eps).
    D, a, eps = 10, 1e-3, 1e-6
    x = np.array([[a if c % 2 == 0 else -a for c in range(D)]])
    gamma = np.full((1, D), 0.25)
    beta = np.full((1, D), -0.5)
    got = oracle.adaln_modulate(x, gamma, beta, 1, eps=eps, scale_offset=1.0)
    xhat = a / math.sqrt(a * a + eps)
    expect = np.array([[(xhat if c % 2 == 0 else -xhat) * 1.25 - 0.5 for c in range(D)]])
    np.testing.assert_allclose(got, expect, rtol=0, atol=1e-15)


def test_adaln_output_moments():
    # With gamma = beta = 0, s0 = 1: mean 0 and variance var/(var+eps) per row.
    D, eps = 256, 1e-2
    x = RNG.standard_normal((3, D)) * np.array([[0.05], [1.0], [4.0]])
    z = np.zeros((1, D))
    u = oracle.adaln_modulate(x, z, z, 3, eps=eps)
    var = x.var(axis=1)
    np.testing.assert_allclose(u.mean(axis=1), 0, atol=1e-14)
    np.testing.assert_allclose(u.var(axis=1), var / (var + eps), rtol=1e-12)


# ----------------------------------------------------------------------------- gated residual

def test_residual_alpha_zero_is_identity():
    # adaLN-Zero: alpha = 0 makes the block the identity, bit for bit.
    x = RNG.standard_normal((6, 32))
    y = RNG.standard_normal((6, 32)) * 100
    got = oracle.gated_residual(x, y, np.zeros((2, 32)), 3)
    assert np.array_equal(got, x)


def test_residual_cancellation_and_groups():
    x = RNG.standard_normal((6, 32))
    got = oracle.gated_residual(x, -x, np.ones((3, 32)), 2)
    assert np.array_equal(got, np.zeros_like(x))
    alpha = RNG.standard_normal((3, 32))
    got = oracle.gated_residual(np.zeros((6, 32)), np.ones((6, 32)), alpha, 2)
    assert np.array_equal(got, np.repeat(alpha, 2, axis=0))


# ----------------------------------------------------------------------------- 3D-RoPE

def _rope(v, cu, gh, gw, bands, base=10000.0, offsets=(0, 0, 0)):
    return oracle.rope3d(v, cu, gh, gw, bands, base, offsets)


# ----------------------------------------------------------------------------- Euler step
# DiT page, "Flow Matching e Rectified Flow": on the straight path
# x_t = (1 - t) x_0 + t x_1 the velocity is the constant x_1 - x_0, so one Euler step of
# any size lands exactly on the path; Flowception, "Metodologia": frames keep their own
# local times, so each frame moves along its own path by its own step.

def test_euler_step_is_exact_on_the_straight_path():
    rng = np.random.default_rng(7)
    G, rpg, D = 5, 6, 16
    x0 = rng.standard_normal((G * rpg, D))
    x1 = rng.standard_normal((G * rpg, D))
    t = rng.uniform(0.0, 0.9, G)          # local time of each frame
    t_next = np.minimum(t + rng.uniform(0.01, 0.3, G), 1.0)
    tr, tr_next = np.repeat(t, rpg)[:, None], np.repeat(t_next, rpg)[:, None]
    x_t = (1 - tr) * x0 + tr * x1
    out = oracle.flow_euler_step(x_t, x1 - x0, t_next - t, rpg)
    np.testing.assert_allclose(out, (1 - tr_next) * x0 + tr_next * x1, rtol=0, atol=1e-12)


def test_euler_frames_use_their_own_step():
    # frame g gets step dt[g]: a constant velocity of ones moves frame g by exactly dt[g]
    dt = np.array([0.0, 0.5, -0.25, 2.0])
    x = np.zeros((8, 4))
    out = oracle.flow_euler_step(x, np.ones_like(x), dt, 2)
    np.testing.assert_array_equal(out[:, 0], np.repeat(dt, 2))


def test_euler_zero_step_is_identity_and_steps_compose():
    rng = np.random.default_rng(8)
    x, u = rng.standard_normal((6, 8)), rng.standard_normal((6, 8))
    np.testing.assert_array_equal(oracle.flow_euler_step(x, u, np.zeros(3), 2), x)
    a, b = np.array([0.125, 0.25, 0.5]), np.array([0.25, 0.5, 0.125])
    two = oracle.flow_euler_step(oracle.flow_euler_step(x, u, a, 2), u, b, 2)
    np.testing.assert_allclose(two, oracle.flow_euler_step(x, u, a + b, 2), atol=1e-14)


# ----------------------------------------------------------------------------- linear layers
# Cost page, "Matematica por tras": Y = X W; DiT page: projections and MLP inside the
# adaLN-Zero residuals. GELU's tanh form and the bias are this library's reading.

def test_linear_equals_library_matmul_with_bias():
    rng = np.random.default_rng(11)
    x, w, b = rng.standard_normal((7, 24)), rng.standard_normal((10, 24)), rng.standard_normal(10)
    np.testing.assert_allclose(oracle.linear(x, w, b), x @ w.T + b, rtol=1e-13, atol=1e-13)


def test_linear_identity_weight_and_gate():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((6, 8))
    np.testing.assert_array_equal(oracle.linear(x, np.eye(8)), x)
    # adaLN-Zero: a zero gate returns the residual; gate 1 with w = -I cancels it
    alpha0 = np.zeros((3, 8))
    np.testing.assert_array_equal(oracle.linear(x, np.eye(8), res=x, alpha=alpha0, rows_per_group=2), x)
    np.testing.assert_array_equal(oracle.linear(x, -np.eye(8), res=x, alpha=np.ones((3, 8)),
                                                rows_per_group=2), np.zeros_like(x))
    # gate group index: group g scales its rows only
    alpha = np.repeat(np.array([[1.0], [2.0], [3.0]]), 8, axis=1)
    out = oracle.linear(x, np.eye(8), res=np.zeros_like(x), alpha=alpha, rows_per_group=2)
    np.testing.assert_array_equal(out, x * np.repeat([1.0, 2.0, 3.0], 2)[:, None])


def test_gelu_tanh_form_matches_library_and_its_odd_part():
    y = np.linspace(-6, 6, 97)
    got = oracle.linear(y[:, None], np.ones((1, 1)), act=1)[:, 0]
    ref = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
    # gelu(y) - gelu(-y) = y exactly for the tanh form
    np.testing.assert_allclose(got - got[::-1], y, atol=1e-12)


# ----------------------------------------------------------------------------- FP8 (E4M3)
# DiT page, "Engenharia de inferencia e paralelismo de contexto: ... FP8": activations in
# FP8 E4M3. The format (OCP E4M3: bias 7, 3 mantissa bits, max 448) is pinned against
# torch's float8_e4m3fn conversion inside its range, and saturation by closed form.

def test_e4m3_matches_library_conversion_in_range():
    rng = np.random.default_rng(13)
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    grid = np.sort(codes[np.isfinite(codes)])
    mids = (grid[1:] + grid[:-1]) / 2                   # exact ties: nearest-even decides
    x = np.concatenate([grid, mids, rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 0.01])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(oracle.quantize_e4m3(x), ref)


def test_e4m3_saturates_and_scales():
    np.testing.assert_array_equal(oracle.quantize_e4m3(np.array([449.0, 1e9, -500.0])),
                                  [448.0, 448.0, -448.0])
    # inv_scale multiplies before rounding: 3 * 0.5 = 1.5 is exact; 1.2 * 64 = 76.8 lies
    # in [64, 128), where e4m3 values are 8 apart: 80
    np.testing.assert_array_equal(oracle.quantize_e4m3(np.array([3.0, 1.2]), 0.5), [1.5, 0.625])
    np.testing.assert_array_equal(oracle.quantize_e4m3(np.array([1.2]), 64.0), [80.0])


def test_bf16_rounding_matches_library():
    rng = np.random.default_rng(14)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-6, 6, 5000),
                        [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)]])
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x), ref)


def test_attn_qk8_is_attention_of_the_quantised_operands():
    rng = np.random.default_rng(15)
    N, H, d = 40, 2, 32
    # operands already on the e4m3 grid times a power of two: quantisation is exact
    q = oracle.quantize_e4m3(rng.standard_normal((N, H, d)) * 8) / 8
    k = oracle.quantize_e4m3(rng.standard_normal((N, H, d)) * 8) / 8
    v = rng.standard_normal((N, H, d))
    cu = np.array([0, N], np.int32)
    o8, l8 = oracle.attn_fwd_qk8(q, k, v, cu, 1 / 8, 1 / 8)
    o, l = oracle.attn_fwd(q, k, v, cu)
    np.testing.assert_allclose(o8, o, atol=1e-13)
    np.testing.assert_allclose(l8, l, atol=1e-13)


def test_attn_qk8_rope_on_a_single_frame_with_time_band_energy_is_plain_attention():
    # T = 1: every token has t = 0, so the t band turns by nothing; q and k hold energy in
    # the t band only, so the h and w bands rotate zeros. The rotation is then the
    # identity, the bf16 rounding of operands already on the e4m3 grid is exact, and the
    # E4M3 attention with RoPE must equal plain attention of the unrotated operands.
    rng = np.random.default_rng(16)
    gh, gw, H, d, bands = 3, 4, 2, 32, (16, 8, 8)
    N = gh * gw
    q = np.zeros((N, H, d))
    k = np.zeros((N, H, d))
    q[..., :16] = oracle.quantize_e4m3(rng.standard_normal((N, H, 16)) * 8) / 8
    k[..., :16] = oracle.quantize_e4m3(rng.standard_normal((N, H, 16)) * 8) / 8
    v = rng.standard_normal((N, H, d))
    cu = np.array([0, N], np.int32)
    rope = dict(grid_h=gh, grid_w=gw, bands=bands)
    o8, l8 = oracle.attn_fwd_qk8(q, k, v, cu, 1 / 8, 1 / 8, rope=rope)
    o, l = oracle.attn_fwd(q, k, v, cu)
    np.testing.assert_allclose(o8, o, atol=1e-13)
    np.testing.assert_allclose(l8, l, atol=1e-13)
    # energy outside the t band does turn (w > 0 tokens): the two must then differ
    q2 = q.copy()
    q2[..., 16:] = 1.0
    k2 = k.copy()
    k2[..., 24:] = 1.0
    o8c, _ = oracle.attn_fwd_qk8(q2, k2, v, cu, 1 / 8, 1 / 8, rope=rope)
    oc, _ = oracle.attn_fwd(q2, k2, v, cu)
    assert not np.allclose(o8c, oc, atol=1e-6)


def test_attn_qk8_rope_order_rotate_round_bf16_then_e4m3_two_keys():
    # Hand-computed case that fixes the order of the steps (DiT page, 3D-RoPE section:
    # the scores use the rotated q and k; FP8 section: E4M3 operands; the rotated
    # operand is a bf16 tensor before it is quantised). d = 2 with one w-band pair of
    # frequency base^0 = 1; a 1 x 2 patch grid, so token 0 sits at w = 0 (no turn) and
    # token 1 at w = 1 (a turn of 1 rad). q_0 = (1, 0); k_0 = (1.5, 0); k_1 = (1.96875, 0).
    #   k_1 rotated: (1.96875 cos 1, 1.96875 sin 1) = (1.063720..., 1.656673...)
    #   bf16:        (1.0625, 1.65625)        (bf16 spacing 2^-7 in [1, 2))
    #   E4M3:        (1.0,    1.625)          (1.0625 is the tie between 1.0 and 1.125:
    #                                          nearest even keeps 1.0)
    # so with scale 1 the scores of query 0 are s_0 = 1.5 and s_1 = 1.0, and
    #   o_0 = sigmoid(0.5) v_0 + sigmoid(-0.5) v_1,  lse_0 = log(e^1.5 + e^1.0).
    # Skipping the bf16 rounding gives s_1 = 1.125; quantising before rotating gives
    # s_1 = bf16(2 cos 1) = 1.078125: both fail below.
    q = np.array([[[1.0, 0.0]], [[0.25, 0.5]]])
    k = np.array([[[1.5, 0.0]], [[1.96875, 0.0]]])
    v = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    cu = np.array([0, 2], np.int32)
    rope = dict(grid_h=1, grid_w=2, bands=(0, 0, 2))
    o, lse = oracle.attn_fwd_qk8(q, k, v, cu, 1.0, 1.0, scale=1.0, qrows=[0], rope=rope)
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    np.testing.assert_allclose(o[0, 0], [sig(0.5), sig(-0.5)], atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], math.log(math.exp(1.5) + math.exp(1.0)), atol=1e-15)
    # the same case with the scales moved onto the codes (q_scale = k_scale = 1/2, codes
    # e4m3(2 x)): a power-of-two scale moves the E4M3 grid with the values, so the same
    # values come out and the tie at 1.0625 (2.125 in code units) again keeps the even 1.0
    o2, _ = oracle.attn_fwd_qk8(q, k, v, cu, 0.5, 0.5, scale=1.0, qrows=[0], rope=rope)
    np.testing.assert_allclose(o2[0, 0], [sig(0.5), sig(-0.5)], atol=1e-15)


def test_rope_preserves_norm():
    # Orthogonal rotations (DiT page, 3D-RoPE section): |R q| = |q| per head.
    gh, gw, T, H, d = 3, 5, 4, 3, 64
    v = RNG.standard_normal((T * gh * gw, H, d))
    out = _rope(v, [0, T * gh * gw], gh, gw, (16, 24, 24))
    np.testing.assert_allclose(np.linalg.norm(out, axis=-1), np.linalg.norm(v, axis=-1),
                               rtol=1e-13)
    assert not np.allclose(out, v)


def test_rope_position_zero_is_identity():
    v = RNG.standard_normal((1, 2, 32))
    assert np.array_equal(_rope(v, [0, 1], 1, 1, (8, 12, 12)), v)


def test_rope_single_frame_leaves_time_band():
    # T = 1 (image workload): every token has t = 0, so the t band is untouched.
    gh, gw, d_t = 4, 4, 32
    v = RNG.standard_normal((gh * gw, 2, 128))
    out = _rope(v, [0, gh * gw], gh, gw, (d_t, 48, 48))
    assert np.array_equal(out[..., :d_t], v[..., :d_t])
    assert not np.allclose(out[..., d_t:], v[..., d_t:])


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_rope_frequency_law_closed_form(axis):
    # theta_{a,i} = base^(-2i/d_a): with d_a = 16 and i = 4 the frequency is 1/100, so a
    # position of 100 turns the pair by exactly 1 radian; pair (2i, 2i+1) inside band a.
    bands = (16, 16, 16)
    off = [0, 16, 32][axis]
    i = 4
    offsets = [0, 0, 0]
    offsets[axis] = 100
    for comp, expect in ((0, (math.cos(1.0), math.sin(1.0))), (1, (-math.sin(1.0), math.cos(1.0)))):
        v = np.zeros((1, 1, 48))
        v[0, 0, off + 2 * i + comp] = 1.0
        out = _rope(v, [0, 1], 1, 1, bands, 10000.0, tuple(offsets))
        np.testing.assert_allclose(out[0, 0, off + 2 * i:off + 2 * i + 2], expect, atol=1e-15)
        mask = np.ones(48, bool)
        mask[off + 2 * i:off + 2 * i + 2] = False
        assert np.all(out[0, 0, mask] == 0)
    # i = 0 always has frequency 1; the last pair of band 16 has base^(-14/16)
    v = np.zeros((1, 1, 48))
    v[0, 0, off + 14] = 1.0
    out = _rope(v, [0, 1], 1, 1, bands, 10000.0, tuple(offsets))
    ang = 100 * 10000.0 ** (-14 / 16)
    np.testing.assert_allclose(out[0, 0, off + 14:off + 16], (math.cos(ang), math.sin(ang)),
                               atol=1e-14)


def test_rope_token_coordinates_row_major():
    # token j = t*(gh*gw) + h*gw + w; the i = 0 pair of each band turns by its coordinate.
    gh, gw, T = 3, 5, 2
    bands = (8, 8, 8)
    t, h, w = 1, 2, 3
    j = t * gh * gw + h * gw + w
    v = np.zeros((T * gh * gw, 1, 24))
    v[:, 0, [0, 8, 16]] = 1.0
    out = _rope(v, [0, T * gh * gw], gh, gw, bands)
    for band, pos in zip((0, 8, 16), (t, h, w)):
        np.testing.assert_allclose(out[j, 0, band:band + 2], (math.cos(pos), math.sin(pos)),
                                   atol=1e-15)


def test_rope_matches_matrix_exponential_of_generator():
    # Brute force: R3D = expm(sum phi_k J_k), J_k the plane generator of pair k (scipy).
    gh, gw, bands, base = 2, 3, (4, 6, 6), 500.0
    d = sum(bands)
    v = RNG.standard_normal((2 * gh * gw, 1, d))
    out = _rope(v, [0, 2 * gh * gw], gh, gw, bands, base, (1, 2, 3))
    for j in range(v.shape[0]):
        t, h, w = j // (gh * gw) + 1, (j // gw) % gh + 2, j % gw + 3
        G = np.zeros((d, d))
        o = 0
        for da, pos in zip(bands, (t, h, w)):
            for i in range(da // 2):
                phi = pos * base ** (-2.0 * i / da)
                G[o + 2 * i + 1, o + 2 * i] = phi
                G[o + 2 * i, o + 2 * i + 1] = -phi
            o += da
        R = scipy.linalg.expm(G)
        np.testing.assert_allclose(out[j, 0], R @ v[j, 0], atol=1e-12)


def test_rope_scores_invariant_to_position_shift():
    # <R(p) q, R(p') k> depends only on p - p': a common shift of (t, h, w) leaves QK^T.
    gh, gw, T, d = 3, 4, 3, 48
    n = T * gh * gw
    q = RNG.standard_normal((n, 1, d))
    k = RNG.standard_normal((n, 1, d))
    s0 = _rope(q, [0, n], gh, gw, (16, 16, 16))[:, 0] @ _rope(k, [0, n], gh, gw, (16, 16, 16))[:, 0].T
    sh = (5, -2, 7)
    s1 = _rope(q, [0, n], gh, gw, (16, 16, 16), offsets=sh)[:, 0] @ \
        _rope(k, [0, n], gh, gw, (16, 16, 16), offsets=sh)[:, 0].T
    np.testing.assert_allclose(s1, s0, atol=1e-12)
    assert not np.allclose(s0, q[:, 0] @ k[:, 0].T)


def test_rope_positions_restart_per_sequence():
    gh, gw = 2, 3
    lens = [2 * gh * gw, 3 * gh * gw]
    cu = [0, lens[0], lens[0] + lens[1]]
    v = RNG.standard_normal((cu[-1], 2, 16))
    out = _rope(v, cu, gh, gw, (4, 6, 6))
    a = _rope(v[:lens[0]], [0, lens[0]], gh, gw, (4, 6, 6))
    b = _rope(v[lens[0]:], [0, lens[1]], gh, gw, (4, 6, 6))
    assert np.array_equal(out, np.concatenate([a, b]))


# ----------------------------------------------------------------------------- attention

def _sdpa(q, k, v):
    # q, k, v: [N, H, d] -> torch [H, N, d]
    t = [torch.from_numpy(np.ascontiguousarray(a.transpose(1, 0, 2))) for a in (q, k, v)]
    o = torch.nn.functional.scaled_dot_product_attention(*t)
    return o.numpy().transpose(1, 0, 2)


@pytest.mark.parametrize("N,H,d", [(1, 1, 8), (7, 2, 16), (130, 3, 64), (257, 2, 128)])
def test_attn_matches_library_sdpa(N, H, d):
    q, k, v = (RNG.standard_normal((N, H, d)) for _ in range(3))
    o, lse = oracle.attn_fwd(q, k, v, [0, N])
    np.testing.assert_allclose(o, _sdpa(q, k, v), atol=1e-12)
    s = np.einsum("ihc,jhc->hij", q, k) / math.sqrt(d)
    ref_lse = torch.logsumexp(torch.from_numpy(s), dim=-1).numpy().T
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12)


def test_attn_ones_values_give_ones():
    q, k = (RNG.standard_normal((40, 2, 16)) * 3 for _ in range(2))
    o, _ = oracle.attn_fwd(q, k, np.ones((40, 2, 16)), [0, 40])
    np.testing.assert_allclose(o, 1.0, atol=1e-14)


def test_attn_probabilities_sum_to_one_and_follow_ratio_law():
    # V = identity exposes P itself: rows sum to 1 and P_ij / P_ik = exp(s_ij - s_ik).
    N, d = 12, 16
    q = RNG.standard_normal((N, 1, d))
    k = RNG.standard_normal((N, 1, d))
    v = np.zeros((N, 1, d))
    v[np.arange(N), 0, np.arange(N)] = 1.0
    o, _ = oracle.attn_fwd(q, k, v, [0, N], scale=0.7)
    P = o[:, 0, :N]
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(P > 0)
    s = 0.7 * q[:, 0] @ k[:, 0].T
    np.testing.assert_allclose(P[:, 3] / P[:, 5], np.exp(s[:, 3] - s[:, 5]), rtol=1e-12)


def test_attn_identical_keys_give_mean_of_values():
    N, d = 9, 32
    k = np.repeat(RNG.standard_normal((1, 1, d)), N, axis=0)
    q = RNG.standard_normal((N, 1, d))
    v = RNG.standard_normal((N, 1, d))
    o, _ = oracle.attn_fwd(q, k, v, [0, N])
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-14)


def test_attn_single_key_returns_value():
    q, k, v = (RNG.standard_normal((1, 3, 8)) for _ in range(3))
    o, lse = oracle.attn_fwd(q, k, v, [0, 1])
    np.testing.assert_allclose(o, v, atol=1e-15)
    np.testing.assert_allclose(lse[0], np.einsum("hc,hc->h", q[0], k[0]) / math.sqrt(8),
                               atol=1e-14)


def test_attn_two_keys_closed_form():
    # o = sigmoid(s0 - s1) v0 + sigmoid(s1 - s0) v1 (not symmetric in q and k).
    d = 4
    q = np.array([[[1.0, 2.0, 0.0, -1.0]], [[0.5, 0.0, 1.0, 0.0]]])
    k = np.array([[[0.0, 1.0, 1.0, 0.0]], [[2.0, 0.0, 0.0, 1.0]]])
    v = np.array([[[1.0, 0.0, 3.0, 0.0]], [[0.0, -2.0, 1.0, 5.0]]])
    o, _ = oracle.attn_fwd(q, k, v, [0, 2])
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    for i in range(2):
        s = [float(q[i, 0] @ k[j, 0]) / 2.0 for j in range(2)]
        expect = sig(s[0] - s[1]) * v[0, 0] + sig(s[1] - s[0]) * v[1, 0]
        np.testing.assert_allclose(o[i, 0], expect, atol=1e-15)


def test_attn_dominant_score_selects_its_value():
    N, d = 16, 8
    k = RNG.standard_normal((N, 1, d)) * 0.01
    k[6, 0] = 100.0 * np.ones(d)
    q = np.ones((N, 1, d))
    v = RNG.standard_normal((N, 1, d))
    o, _ = oracle.attn_fwd(q, k, v, [0, N])
    np.testing.assert_allclose(o, np.broadcast_to(v[6], o.shape), atol=1e-12)


def test_attn_packed_sequences_are_independent():
    lens = [5, 17, 1, 40]
    cu = np.concatenate([[0], np.cumsum(lens)])
    n = cu[-1]
    q, k, v = (RNG.standard_normal((n, 2, 16)) for _ in range(3))
    o, lse = oracle.attn_fwd(q, k, v, cu)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        os_, ls_ = oracle.attn_fwd(q[a:b], k[a:b], v[a:b], [0, b - a])
        np.testing.assert_array_equal(o[a:b], os_)
        np.testing.assert_array_equal(lse[a:b], ls_)
    # tokens of another sequence never leak in
    k2, v2 = k.copy(), v.copy()
    k2[cu[1]:cu[2]] += 5
    v2[cu[1]:cu[2]] -= 3
    o2, _ = oracle.attn_fwd(q, k2, v2, cu)
    np.testing.assert_array_equal(o2[:cu[1]], o[:cu[1]])
    np.testing.assert_array_equal(o2[cu[2]:], o[cu[2]:])


def test_attn_sampled_rows_equal_full_rows():
    n = 50
    q, k, v = (RNG.standard_normal((n, 2, 16)) for _ in range(3))
    o, lse = oracle.attn_fwd(q, k, v, [0, 20, n])
    rows = np.array([0, 19, 20, 49, 33])
    os_, ls_ = oracle.attn_fwd(q, k, v, [0, 20, n], qrows=rows)
    np.testing.assert_array_equal(os_, o[rows])
    np.testing.assert_array_equal(ls_, lse[rows])


def test_attn_rope_relative_positions():
    # 3D-RoPE attention only sees relative positions: shifting every coordinate by the
    # same offsets leaves the output unchanged; rotating only q would not.
    gh, gw, T, H, d = 2, 3, 3, 2, 64
    n = T * gh * gw
    q, k, v = (RNG.standard_normal((n, H, d)) for _ in range(3))
    rope = dict(grid_h=gh, grid_w=gw, bands=(16, 24, 24), base=10000.0, offsets=(0, 0, 0))
    o0, _ = oracle.attn_fwd(q, k, v, [0, n], rope=rope)
    o1, _ = oracle.attn_fwd(q, k, v, [0, n], rope=dict(rope, offsets=(3, 1, 7)))
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    onr, _ = oracle.attn_fwd(q, k, v, [0, n])
    assert not np.allclose(o0, onr, atol=1e-3)
    qr = oracle.rope3d(q, [0, n], gh, gw, (16, 24, 24))
    kr = oracle.rope3d(k, [0, n], gh, gw, (16, 24, 24))
    np.testing.assert_allclose(o0, _sdpa(qr, kr, v), atol=1e-12)


# ----------------------------------------------------------------------------- input generator

def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 3.0e-3, 1.0 + 2**-9], np.float32)
    bits = wl.f32_to_bf16_bits(vals)
    back = wl.bf16_bits_to_f64(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa wins (1.0)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2**-6
    assert back[3] == -2.5
    assert abs(back[4] - 3.0e-3) <= 3.0e-3 * 2**-8
    ref = torch.tensor(vals).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(back, ref)


def test_inputs_are_seeded_and_shaped():
    w = wl.get_workload("tiny")
    a = wl.make_inputs(w, seed=3)
    b = wl.make_inputs(w, seed=3)
    c = wl.make_inputs(w, seed=4)
    for name in a:
        assert np.array_equal(a[name], b[name])
    assert not np.array_equal(a["q"], c["q"])
    assert a["x"].shape == (64, 128) and a["q"].shape == (64, 2, 64)
    assert a["gamma"].shape == (1, 128)
    x = wl.bf16_bits_to_f64(a["x"])
    assert abs(x.mean()) < 0.1 and abs(x.std() - 1) < 0.1
    g = wl.bf16_bits_to_f64(a["gamma"])
    assert g.std() < 0.2
    z = wl.make_inputs(w, which=("alpha",), alpha_zero=True)["alpha"]
    assert not z.any()
