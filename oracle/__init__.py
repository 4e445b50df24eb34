"""fp64 CPU oracle for the DiT attention-block hot path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may import this package; the product path never does. It shares
no code with the CUDA library: the arithmetic lives in ``dit3d_oracle.c`` and
this module only marshals numpy float64 arrays into it.

Each wrapper cites the passage it restates:

* ``adaln_modulate`` / ``gated_residual`` -- "DiT, Flow Matching e 3D Attention",
  section "A ruptura da U-Net" (adaLN-Zero).
* ``flow_euler_step`` -- same page, section "Flow Matching e Rectified Flow"
  (Euler sampler on the straight path), with the per-frame local times of
  "Flowception: Temporally Expansive Flow Matching for Video Generation",
  section "Metodologia".
* ``quantize_e4m3`` / ``attn_fwd_qk8`` -- DiT page, section "Engenharia de inferencia e
  paralelismo de contexto: Ulysses, Ring Attention e FP8" (FP8 E4M3 activations).
* ``linear`` -- "Por que e absurdamente dificil gerar um filme inteiro usando IA",
  section "Matematica por tras" (Y = X W), with the DiT page's MLP and gates.
* ``rope3d`` -- same page, section "3D-RoPE e atencao espaco-temporal".
* ``attn_fwd`` -- same section, and "Por que e absurdamente dificil gerar um
  filme inteiro usando IA", section "Matematica por tras".
* ``patch_grid_tokens`` -- same DiT page, the patchify diagram of section
  "A ruptura da U-Net": N = (T/p_t)(H/p_h)(W/p_w).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dit3d_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        lib.oracle_adaln_modulate.argtypes = [P, P, P, P, i64, i32, i64, f64, f64]
        lib.oracle_gated_residual.argtypes = [P, P, P, P, i64, i32, i64]
        lib.oracle_flow_euler_step.argtypes = [P, P, P, P, i64, i32, i64]
        lib.oracle_linear.argtypes = [P, P, P, P, i64, i32, i32, i32, P, P, i64]
        lib.oracle_quantize_e4m3.argtypes = [P, P, i64, f64]
        lib.oracle_round_bf16.argtypes = [P, P, i64]
        lib.oracle_rope3d.argtypes = [P, P, i64, i32, i32, P, i32, i32, i32, i32, i32, i32, f64,
                                      i32, i32, i32]
        lib.oracle_attn_fwd.argtypes = [P, P, P, P, P, i64, i32, i32, P, i32, f64, P, i64]
        lib.oracle_threads.argtypes = []
        lib.oracle_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = None
        for f in (lib.oracle_adaln_modulate, lib.oracle_gated_residual, lib.oracle_rope3d,
                  lib.oracle_attn_fwd, lib.oracle_flow_euler_step, lib.oracle_linear,
                  lib.oracle_quantize_e4m3, lib.oracle_round_bf16):
            f.restype = None
        _lib = lib
    return _lib


def threads() -> int:
    """Threads the oracle's OpenMP loops run on."""
    return int(_load().oracle_threads())


def set_threads(n: int) -> None:
    """Run the oracle's OpenMP loops on n threads from now on."""
    _load().oracle_set_threads(int(n))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _cu(cu_seqlens) -> np.ndarray:
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    assert cu.ndim == 1 and cu[0] == 0 and np.all(np.diff(cu) >= 0)
    return cu


def patch_grid_tokens(T: int, H: int, W: int, p_t: int, p_h: int, p_w: int) -> int:
    """Number of patch tokens N = (T/p_t)(H/p_h)(W/p_w) of a C x T x H x W latent."""
    assert T % p_t == 0 and H % p_h == 0 and W % p_w == 0
    return (T // p_t) * (H // p_h) * (W // p_w)


def adaln_modulate(x, gamma, beta, rows_per_group: int, eps: float = 1e-6,
                   scale_offset: float = 1.0) -> np.ndarray:
    """u = LayerNorm(x) * (scale_offset + gamma_g) + beta_g, fp64. x: [rows, D]; gamma, beta: [G, D]."""
    x, gamma, beta = _f64(x), _f64(gamma), _f64(beta)
    rows, D = x.shape
    assert rows % rows_per_group == 0 and gamma.shape == beta.shape == (rows // rows_per_group, D)
    out = np.empty_like(x)
    _load().oracle_adaln_modulate(_ptr(x), _ptr(gamma), _ptr(beta), _ptr(out), rows, D,
                                  rows_per_group, eps, scale_offset)
    return out


def gated_residual(x, y, alpha, rows_per_group: int) -> np.ndarray:
    """out = x + alpha_g * y, fp64. x, y: [rows, D]; alpha: [G, D]."""
    x, y, alpha = _f64(x), _f64(y), _f64(alpha)
    rows, D = x.shape
    assert y.shape == x.shape and alpha.shape == (rows // rows_per_group, D)
    out = np.empty_like(x)
    _load().oracle_gated_residual(_ptr(x), _ptr(y), _ptr(alpha), _ptr(out), rows, D,
                                  rows_per_group)
    return out


def flow_euler_step(x, u, dt, rows_per_group: int) -> np.ndarray:
    """out = x + dt[g] * u for the rows of frame g, fp64. x, u: [rows, D]; dt: [G]."""
    x, u, dt = _f64(x), _f64(u), _f64(dt)
    rows, D = x.shape
    assert u.shape == x.shape and dt.shape == (rows // rows_per_group,)
    out = np.empty_like(x)
    _load().oracle_flow_euler_step(_ptr(x), _ptr(u), _ptr(dt), _ptr(out), rows, D,
                                   rows_per_group)
    return out


def linear(x, w, bias=None, act: int = 0, res=None, alpha=None,
           rows_per_group: int = 1) -> np.ndarray:
    """y = x w^T (+ bias), GELU (tanh form) if act == 1, then res + alpha_g * y when res
    is given; fp64. x: [M, K]; w: [N, K]; bias: [N]; res: [M, N]; alpha: [G, N]."""
    x, w = _f64(x), _f64(w)
    M, K = x.shape
    N = w.shape[0]
    assert w.shape == (N, K)
    b = None if bias is None else _f64(bias)
    r = None if res is None else _f64(res)
    a = None if alpha is None else _f64(alpha)
    if r is not None:
        assert r.shape == (M, N) and a is not None and a.shape == (M // rows_per_group, N)
    out = np.empty((M, N))
    _load().oracle_linear(_ptr(x), _ptr(w), None if b is None else _ptr(b), _ptr(out), M, N, K,
                          int(act), None if r is None else _ptr(r), None if a is None else _ptr(a),
                          rows_per_group)
    return out


def quantize_e4m3(x, inv_scale: float = 1.0) -> np.ndarray:
    """e4m3(x * inv_scale) (nearest, ties to even, saturated at 448) as fp64 values."""
    x = _f64(x)
    out = np.empty_like(x)
    _load().oracle_quantize_e4m3(_ptr(x), _ptr(out), x.size, float(inv_scale))
    return out


def round_bf16(x) -> np.ndarray:
    """Nearest bf16 value of each element (ties to even), fp64."""
    x = _f64(x)
    out = np.empty_like(x)
    _load().oracle_round_bf16(_ptr(x), _ptr(out), x.size)
    return out


def attn_fwd_qk8(q, k, v, cu_seqlens, q_scale: float, k_scale: float, scale: float | None = None,
                 qrows=None, rope=None):
    """Attention whose Q K^T runs on FP8 E4M3 operands: q and k (rotated by ``rope3d``
    and rounded to bf16 first, when ``rope`` is given) are quantised as
    e4m3(q / q_scale), e4m3(k / k_scale) and the scores use q_scale * k_scale times
    their product; P and V stay exact. Returns (o, lse) like ``attn_fwd``."""
    q, k = _f64(q), _f64(k)
    if rope is not None:
        cu = _cu(cu_seqlens)
        q = round_bf16(rope3d(q, cu, rope["grid_h"], rope["grid_w"], rope["bands"],
                              rope.get("base", 10000.0), rope.get("offsets", (0, 0, 0))))
        k = round_bf16(rope3d(k, cu, rope["grid_h"], rope["grid_w"], rope["bands"],
                              rope.get("base", 10000.0), rope.get("offsets", (0, 0, 0))))
    q8 = quantize_e4m3(q, 1.0 / q_scale) * q_scale
    k8 = quantize_e4m3(k, 1.0 / k_scale) * k_scale
    return attn_fwd(q8, k8, v, cu_seqlens, scale=scale, qrows=qrows)


def rope3d(v, cu_seqlens, grid_h: int, grid_w: int, bands, base: float = 10000.0,
           offsets=(0, 0, 0)) -> np.ndarray:
    """3D-RoPE of v: [rows, H, d] (fp64), positions restarting at every sequence start."""
    v = _f64(v)
    rows, H, d = v.shape
    cu = _cu(cu_seqlens)
    assert cu[-1] == rows
    d_t, d_h, d_w = bands
    assert d_t + d_h + d_w == d and d_t % 2 == 0 and d_h % 2 == 0 and d_w % 2 == 0
    out = np.empty_like(v)
    _load().oracle_rope3d(_ptr(v), _ptr(out), rows, H, d, _ptr(cu), len(cu) - 1, grid_h, grid_w,
                          d_t, d_h, d_w, float(base), *[int(o) for o in offsets])
    return out


def attn_fwd(q, k, v, cu_seqlens, scale: float | None = None, qrows=None, rope=None):
    """softmax(q k^T * scale) v per sequence and head, fp64.

    q, k, v: [rows, H, d]. ``rope`` (optional) = dict(grid_h, grid_w, bands, base, offsets):
    q and k are rotated by ``rope3d`` first. ``qrows`` (optional) lists the query rows to
    compute. Returns (o [n_q, H, d], lse [n_q, H]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    rows, H, d = k.shape
    cu = _cu(cu_seqlens)
    assert cu[-1] == rows and q.shape == k.shape == v.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rope is not None:
        q = rope3d(q, cu, **rope)
        k = rope3d(k, cu, **rope)
    if qrows is None:
        n_q, qr_ptr, qr = rows, None, None
    else:
        qr = np.ascontiguousarray(qrows, dtype=np.int64)
        assert qr.min() >= 0 and qr.max() < rows
        n_q, qr_ptr = len(qr), _ptr(qr)
    o = np.empty((n_q, H, d), dtype=np.float64)
    lse = np.empty((n_q, H), dtype=np.float64)
    _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), rows, H, d, _ptr(cu),
                            len(cu) - 1, float(scale), qr_ptr, n_q)
    return o, lse
