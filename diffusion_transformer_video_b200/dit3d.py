"""Thin ctypes binding of libdit3d (include/dit3d.h).

Argument marshalling only: torch tensors become device pointers, the current
torch CUDA stream becomes the call's stream, and a non-zero status becomes a
``DitError``. Every computation runs in the library's CUDA kernels; there is no
fallback. The functions carry the C names.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdit3d.so")

DIT_OK = 0
STATUS_NAMES = {0: "DIT_OK", 1: "DIT_ERR_NULL", 2: "DIT_ERR_SHAPE", 3: "DIT_ERR_ALIGN",
                4: "DIT_ERR_SEQLENS", 5: "DIT_ERR_DEVICE", 6: "DIT_ERR_LAUNCH",
                7: "DIT_ERR_TIMEOUT", 8: "DIT_ERR_ALLOC", 9: "DIT_ERR_SCRATCH"}

# every symbol include/dit3d.h declares
EXPORTS = ("dit_adaln_modulate", "dit_gated_residual", "dit_flow_euler_step", "dit_linear",
           "dit_linear_fp8",
           "dit_set_linear_variant", "dit_attn_fwd_qk8", "dit_attn_fwd_fp8", "dit_quantize_e4m3",
           "dit_rope3d_qk", "dit_rope3d_qk_e4m3", "dit_attn_fwd",
           "dit_attn_fwd_noalloc", "dit_check_device", "dit_status_string", "dit_shutdown",
           "dit_set_attn_variant", "dit_debug_force_timeout",
           "dit_debug_wait_limit_ns", "dit_wait_device", "dit_debug_poll_fake", "dit_debug_exp2_fma",
           "dit_debug_last_attn_split", "dit_debug_tail_split")


class DitError(RuntimeError):
    def __init__(self, status: int, lib):
        self.status = status
        super().__init__(lib.dit_status_string(status).decode())


class RopeDesc(ctypes.Structure):
    """dit_rope3d_desc: patch grid, band widths (t|h|w), frequency base, position offsets."""
    _fields_ = [("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("d_t", ctypes.c_int32), ("d_h", ctypes.c_int32), ("d_w", ctypes.c_int32),
                ("base", ctypes.c_float),
                ("t0", ctypes.c_int32), ("h0", ctypes.c_int32), ("w0", ctypes.c_int32)]


def rope_desc(grid_h, grid_w, bands, base=10000.0, offsets=(0, 0, 0)) -> RopeDesc:
    return RopeDesc(int(grid_h), int(grid_w), int(bands[0]), int(bands[1]), int(bands[2]),
                    float(base), int(offsets[0]), int(offsets[1]), int(offsets[2]))


_lib = None


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m "
                               "diffusion_transformer_video_b200.build` (there is no fallback)")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        L.dit_adaln_modulate.argtypes = [P, P, P, P, i64, i32, i64, f32, f32, P]
        L.dit_gated_residual.argtypes = [P, P, P, P, i64, i32, i64, P]
        L.dit_flow_euler_step.argtypes = [P, P, P, P, i64, i32, i64, P]
        L.dit_linear.argtypes = [P, P, P, P, i64, i32, i32, i32, P, P, i64, P]
        L.dit_linear_fp8.argtypes = [P, P, P, P, i64, i32, i32, i32, P, P, i64, f32, f32, P]
        L.dit_attn_fwd_qk8.argtypes = [P, P, P, P, P, i64, i32, i32, i32, P, P, f32, f32, f32, P]
        L.dit_quantize_e4m3.argtypes = [P, P, i64, f32, P]
        L.dit_attn_fwd_fp8.argtypes = [P, P, P, P, P, i64, i32, i32, i32, P, P, f32, f32, f32, f32, P]
        L.dit_rope3d_qk.argtypes = [P, P, P, P, i64, i32, i32, i32, P, P,
                                    ctypes.POINTER(RopeDesc), P]
        L.dit_rope3d_qk_e4m3.argtypes = [P, P, P, P, i64, i32, i32, i32, P, P,
                                         ctypes.POINTER(RopeDesc), f32, f32, P]
        L.dit_attn_fwd.argtypes = [P, P, P, P, P, i64, i32, i32, i32, P, P, f32,
                                   ctypes.POINTER(RopeDesc), P]
        L.dit_attn_fwd_noalloc.argtypes = [P, P, P, P, P, i64, i32, i32, i32, P, P, f32,
                                           ctypes.POINTER(RopeDesc), P]
        L.dit_attn_fwd_noalloc.restype = ctypes.c_int
        L.dit_check_device.argtypes = [P]
        L.dit_status_string.argtypes = [ctypes.c_int]
        L.dit_status_string.restype = ctypes.c_char_p
        L.dit_shutdown.argtypes = []
        L.dit_shutdown.restype = None
        L.dit_set_attn_variant.argtypes = [ctypes.c_int]
        L.dit_set_attn_variant.restype = ctypes.c_int
        L.dit_debug_force_timeout.argtypes = [ctypes.c_int]
        L.dit_debug_force_timeout.restype = None
        L.dit_debug_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.dit_debug_wait_limit_ns.restype = None
        L.dit_wait_device.argtypes = [P, i64]
        L.dit_wait_device.restype = ctypes.c_int
        L.dit_debug_poll_fake.argtypes = [i64, ctypes.c_int, i64, ctypes.POINTER(i64)]
        L.dit_debug_poll_fake.restype = ctypes.c_int
        L.dit_debug_exp2_fma.argtypes = [P, P, i64, P]
        L.dit_debug_last_attn_split.argtypes = []
        L.dit_debug_tail_split.argtypes = [i64, i64, i64, P, P]
        L.dit_debug_exp2_fma.restype = ctypes.c_int
        for name in ("dit_adaln_modulate", "dit_gated_residual", "dit_rope3d_qk", "dit_attn_fwd",
                     "dit_check_device"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != DIT_OK:
        raise DitError(status, lib())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _bf16(t: torch.Tensor, name: str):
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
        raise TypeError(f"{name} must be a contiguous bf16 CUDA tensor")


def _keep(cu_dev):
    # a device copy made here must outlive the kernel that reads it
    if cu_dev is not None:
        cu_dev.record_stream(torch.cuda.current_stream())


def _cu_args(cu_seqlens):
    """(device tensor, host tensor, n_seq) for a packed layout, or Nones for dense.

    ``cu_seqlens`` is a host sequence/tensor of n_seq + 1 int32 prefix sums, or a
    ``(device_tensor, host_tensor)`` pair prepared once by the caller."""
    if cu_seqlens is None:
        return None, None, None
    if isinstance(cu_seqlens, tuple):
        dev, host = cu_seqlens
        return dev, host, host.numel() - 1
    if isinstance(cu_seqlens, torch.Tensor):
        host = cu_seqlens.detach().to("cpu", torch.int32).contiguous()
    else:
        host = torch.as_tensor(cu_seqlens, dtype=torch.int32).contiguous()
    dev = host.to("cuda", non_blocking=False)
    return dev, host, host.numel() - 1


def dit_adaln_modulate(x, gamma, beta, rows_per_group, out=None, eps=1e-6, scale_offset=1.0):
    """out = LayerNorm(x) * (scale_offset + gamma_g) + beta_g (x: [rows, D] bf16)."""
    for t, n in ((x, "x"), (gamma, "gamma"), (beta, "beta")):
        _bf16(t, n)
    out = torch.empty_like(x) if out is None else out
    _bf16(out, "out")
    rows, D = x.shape[0], x.shape[-1]
    _check(lib().dit_adaln_modulate(_ptr(x), _ptr(gamma), _ptr(beta), _ptr(out), rows, D,
                                    int(rows_per_group), float(eps), float(scale_offset),
                                    _stream()))
    return out


def dit_gated_residual(x, y, alpha, rows_per_group, out=None):
    """out = x + alpha_g * y (all [rows, D] bf16; alpha [G, D])."""
    for t, n in ((x, "x"), (y, "y"), (alpha, "alpha")):
        _bf16(t, n)
    out = torch.empty_like(x) if out is None else out
    _bf16(out, "out")
    rows, D = x.shape[0], x.shape[-1]
    _check(lib().dit_gated_residual(_ptr(x), _ptr(y), _ptr(alpha), _ptr(out), rows, D,
                                    int(rows_per_group), _stream()))
    return out


def dit_flow_euler_step(x, u, dt, rows_per_group, out=None):
    """out = x + dt[g] * u for the rows of frame g (x, u [rows, D] bf16; dt [G] fp32 on the
    device). out=x updates the latent in place."""
    _bf16(x, "x")
    _bf16(u, "u")
    if not (isinstance(dt, torch.Tensor) and dt.dtype == torch.float32 and dt.is_cuda
            and dt.is_contiguous()):
        raise TypeError("dt must be a contiguous float32 CUDA tensor")
    out = torch.empty_like(x) if out is None else out
    _bf16(out, "out")
    rows, D = x.shape[0], x.shape[-1]
    if rows == 0:
        return out
    _check(lib().dit_flow_euler_step(_ptr(x), _ptr(u), _ptr(dt), _ptr(out), rows, D,
                                     int(rows_per_group), _stream()))
    return out


def dit_linear(x, w, bias=None, gelu=False, residual=None, alpha=None, rows_per_group=1,
               out=None):
    """out = [residual + alpha_g *] act(x w^T [+ bias]); x [M, K], w [N, K], bias [N],
    residual [M, N], alpha [G, N], all bf16 on the device."""
    _bf16(x, "x")
    _bf16(w, "w")
    for t, n in ((bias, "bias"), (residual, "residual"), (alpha, "alpha")):
        if t is not None:
            _bf16(t, n)
    M, K = x.shape
    N = w.shape[0]
    out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
    _bf16(out, "out")
    if M == 0:
        return out
    opt = lambda t: None if t is None else _ptr(t)
    _check(lib().dit_linear(_ptr(x), _ptr(w), opt(bias), _ptr(out), M, N, K, 1 if gelu else 0,
                            opt(residual), opt(alpha), int(rows_per_group), _stream()))
    return out


def dit_linear_fp8(x8, w8, x_scale: float, w_scale: float, bias=None, gelu=False, residual=None,
                   alpha=None, rows_per_group=1, out=None):
    """dit_linear on E4M3 codes: x8 [M, K], w8 [N, K] uint8 standing for x_scale * x8 and
    w_scale * w8; bias, residual, alpha bf16; returns bf16 [M, N]."""
    _u8(x8, "x8")
    _u8(w8, "w8")
    for t, n in ((bias, "bias"), (residual, "residual"), (alpha, "alpha")):
        if t is not None:
            _bf16(t, n)
    M, K = x8.shape
    N = w8.shape[0]
    out = torch.empty(M, N, dtype=torch.bfloat16, device=x8.device) if out is None else out
    _bf16(out, "out")
    if M == 0:
        return out
    opt = lambda t: None if t is None else _ptr(t)
    _check(lib().dit_linear_fp8(_ptr(x8), _ptr(w8), opt(bias), _ptr(out), M, N, K,
                                1 if gelu else 0, opt(residual), opt(alpha), int(rows_per_group),
                                float(x_scale), float(w_scale), _stream()))
    return out


def dit_rope3d_qk(q, k, rope: RopeDesc, n_seq=1, cu_seqlens=None, q_out=None, k_out=None,
                  inplace=False):
    """3D-RoPE of q and k ([rows, H, d] bf16). Returns (q_rot, k_rot)."""
    _bf16(q, "q")
    if k is not None:
        _bf16(k, "k")
    if inplace:
        q_out, k_out = q, k
    q_out = torch.empty_like(q) if q_out is None else q_out
    if k is not None:
        k_out = torch.empty_like(k) if k_out is None else k_out
    rows, H, d = q.shape
    cu_dev, cu_host, ns = _cu_args(cu_seqlens)
    n = ns if ns is not None else n_seq
    _check(lib().dit_rope3d_qk(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), rows, H, d, n,
                               _ptr(cu_dev), _ptr(cu_host), ctypes.byref(rope), _stream()))
    _keep(cu_dev)
    return q_out, k_out


def dit_attn_fwd(q, k, v, n_seq=1, cu_seqlens=None, rope: RopeDesc | None = None,
                 softmax_scale=0.0, out=None, return_lse=False):
    """softmax(q_rot k_rot^T * scale) v per sequence and head ([rows, H, d] bf16)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, n)
    rows, H, d = q.shape
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((rows, H), dtype=torch.float32, device=q.device) if return_lse else None
    cu_dev, cu_host, ns = _cu_args(cu_seqlens)
    n = ns if ns is not None else n_seq
    _check(lib().dit_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), rows, H, d, n,
                              _ptr(cu_dev), _ptr(cu_host), float(softmax_scale),
                              ctypes.byref(rope) if rope is not None else None, _stream()))
    _keep(cu_dev)
    return (out, lse) if return_lse else out


def _u8(t: torch.Tensor, name: str):
    if not (isinstance(t, torch.Tensor) and t.dtype == torch.uint8 and t.is_cuda and t.is_contiguous()):
        raise TypeError(f"{name} must be a contiguous uint8 (E4M3 codes) CUDA tensor")


def dit_rope3d_qk_e4m3(q, k, rope: RopeDesc, q_inv_scale: float, k_inv_scale: float = 1.0,
                       n_seq=1, cu_seqlens=None, q8_out=None, k8_out=None):
    """3D-RoPE of q and k ([rows, H, d] bf16) written as E4M3 codes of the rotated
    values times q_inv_scale / k_inv_scale. Returns (q8, k8) as uint8 tensors."""
    _bf16(q, "q")
    if k is not None:
        _bf16(k, "k")
    q8_out = torch.empty(q.shape, dtype=torch.uint8, device=q.device) if q8_out is None else q8_out
    _u8(q8_out, "q8_out")
    if k is not None:
        k8_out = (torch.empty(k.shape, dtype=torch.uint8, device=k.device) if k8_out is None
                  else k8_out)
        _u8(k8_out, "k8_out")
    rows, H, d = q.shape
    cu_dev, cu_host, ns = _cu_args(cu_seqlens)
    n = ns if ns is not None else n_seq
    _check(lib().dit_rope3d_qk_e4m3(_ptr(q), _ptr(k), _ptr(q8_out), _ptr(k8_out), rows, H, d, n,
                                    _ptr(cu_dev), _ptr(cu_host), ctypes.byref(rope),
                                    float(q_inv_scale), float(k_inv_scale), _stream()))
    _keep(cu_dev)
    return q8_out, k8_out


def dit_quantize_e4m3(x, inv_scale: float, out=None):
    """E4M3 codes of x * inv_scale (x bf16 CUDA tensor, numel % 8 == 0) as uint8."""
    _bf16(x, "x")
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device) if out is None else out
    _u8(out, "out")
    _check(lib().dit_quantize_e4m3(_ptr(x), _ptr(out), x.numel(), float(inv_scale), _stream()))
    return out


def dit_attn_fwd_qk8(q8, k8, v, q_scale: float, k_scale: float, n_seq=1, cu_seqlens=None,
                     softmax_scale=0.0, out=None, return_lse=False):
    """Attention with an E4M3 Q K^T: q8, k8 [rows, H, 128] uint8 codes standing for
    q_scale * q8 and k_scale * k8; v bf16. Returns o (and lse)."""
    _u8(q8, "q8")
    _u8(k8, "k8")
    _bf16(v, "v")
    rows, H, d = v.shape
    if q8.shape != v.shape or k8.shape != v.shape:
        raise ValueError("q8, k8 and v must have the same [rows, H, d] shape")
    out = torch.empty_like(v) if out is None else out
    lse = torch.empty((rows, H), dtype=torch.float32, device=v.device) if return_lse else None
    cu_dev, cu_host, ns = _cu_args(cu_seqlens)
    n = ns if ns is not None else n_seq
    _check(lib().dit_attn_fwd_qk8(_ptr(q8), _ptr(k8), _ptr(v), _ptr(out), _ptr(lse), rows, H, d, n,
                                  _ptr(cu_dev), _ptr(cu_host), float(softmax_scale),
                                  float(q_scale), float(k_scale), _stream()))
    _keep(cu_dev)
    return (out, lse) if return_lse else out


def dit_attn_fwd_fp8(q8, k8, v8, q_scale: float, k_scale: float, v_scale: float, n_seq=1,
                     cu_seqlens=None, softmax_scale=0.0, out=None, return_lse=False):
    """Attention with E4M3 q, k and v ([rows, H, 128] uint8 codes standing for
    scale * code); P rounded to E4M3 for the P V product. Returns bf16 o (and lse)."""
    for t, n in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        _u8(t, n)
    rows, H, d = q8.shape
    if k8.shape != q8.shape or v8.shape != q8.shape:
        raise ValueError("q8, k8 and v8 must have the same [rows, H, d] shape")
    out = torch.empty(rows, H, d, dtype=torch.bfloat16, device=q8.device) if out is None else out
    _bf16(out, "out")
    lse = torch.empty((rows, H), dtype=torch.float32, device=q8.device) if return_lse else None
    cu_dev, cu_host, ns = _cu_args(cu_seqlens)
    n = ns if ns is not None else n_seq
    _check(lib().dit_attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(out), _ptr(lse), rows, H, d, n,
                                  _ptr(cu_dev), _ptr(cu_host), float(softmax_scale),
                                  float(q_scale), float(k_scale), float(v_scale), _stream()))
    _keep(cu_dev)
    return (out, lse) if return_lse else out


def dit_set_attn_variant(variant: int):
    """0: single-CTA attention kernel (default); 1: CTA-pair kernel (head_dim 128)."""
    _check(lib().dit_set_attn_variant(int(variant)))


def dit_set_linear_variant(variant: int):
    """0: one CTA per 128x256 tile (default); 1: CTA-pair GEMM on 256x256 tiles."""
    _check(lib().dit_set_linear_variant(int(variant)))


def dit_check_device():
    """Synchronises the current stream and raises DitError if a kernel gave up a wait."""
    _check(lib().dit_check_device(_stream()))


def dit_wait_device(timeout_us: int):
    """Waits for the current stream for at most timeout_us of wall time (polling, no
    blocking synchronisation); raises DitError with DIT_ERR_TIMEOUT if it has not
    finished by then or if a kernel gave up a wait."""
    _check(lib().dit_wait_device(_stream(), int(timeout_us)))


def dit_debug_exp2_fma(t):
    """2^t (t: fp32 CUDA tensor) by the attention's FMA-pipe exponential (test hook)."""
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
        raise TypeError("t must be a contiguous fp32 CUDA tensor")
    out = torch.empty_like(t)
    _check(lib().dit_debug_exp2_fma(_ptr(t), _ptr(out), t.numel(), _stream()))
    return out


def dit_shutdown():
    lib().dit_shutdown()
