"""Out-of-bounds write detection without a sanitizer: every output is placed inside a
larger buffer whose guard regions before and after hold a known pattern, and the
guards must be intact after the call (ragged sizes that end mid-tile)."""
import numpy as np
import pytest
import torch

from diffusion_transformer_video_b200 import dit3d

pytestmark = pytest.mark.gpu
GUARD = 4096  # elements of guard on each side (16-byte aligned for bf16 and fp32)


def _guarded(shape, dtype):
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
    buf.view(torch.uint8).fill_(0xA5)
    return buf, buf[GUARD:GUARD + n].view(shape)


def _intact(buf, n):
    b = buf.view(torch.uint8)
    es = buf.element_size()
    lo, hi = b[: GUARD * es], b[(GUARD + n) * es:]
    return bool((lo == 0xA5).all()) and bool((hi == 0xA5).all())


def test_guards_survive_every_kernel():
    g = torch.Generator(device="cuda").manual_seed(4)
    rows, H, d = 333, 3, 128                      # 333 = 2 x 128 + 77: a ragged last tile
    D = H * d
    bf = lambda *s: torch.randn(*s, device="cuda", generator=g).to(torch.bfloat16)
    q, k, v, x, y = bf(rows, H, d), bf(rows, H, d), bf(rows, H, d), bf(rows, D), bf(rows, D)
    gamma, beta, alpha = bf(3, D), bf(3, D), bf(3, D)
    checks = []

    buf, o = _guarded((rows, H, d), torch.bfloat16)
    lbuf, lse = _guarded((rows, H), torch.float32)
    dit3d.dit_attn_fwd(q, k, v, out=o)
    dit3d.dit_check_device()
    checks.append(("attention", _intact(buf, o.numel())))
    L = dit3d.lib()
    import ctypes
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.dit_attn_fwd(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                          ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                          ctypes.c_void_p(lse.data_ptr()), rows, H, d, 1, None, None, 0.0, None, st) == 0
    dit3d.dit_check_device()
    checks.append(("attention lse", _intact(lbuf, lse.numel())))

    desc = dit3d.rope_desc(9, 37, (44, 42, 42))   # 333 tokens = 1 frame of 9 x 37
    qb, qo = _guarded((rows, H, d), torch.bfloat16)
    kb, ko = _guarded((rows, H, d), torch.bfloat16)
    dit3d.dit_rope3d_qk(q, k, desc, q_out=qo, k_out=ko)
    dit3d.dit_check_device()
    checks += [("rope q", _intact(qb, qo.numel())), ("rope k", _intact(kb, ko.numel()))]
    q8b, q8o = _guarded((rows, H, d), torch.uint8)
    k8b, k8o = _guarded((rows, H, d), torch.uint8)
    dit3d.dit_rope3d_qk_e4m3(q, k, desc, 64.0, 32.0, q8_out=q8o, k8_out=k8o)
    dit3d.dit_check_device()
    checks += [("rope e4m3 q", _intact(q8b, q8o.numel())), ("rope e4m3 k", _intact(k8b, k8o.numel()))]

    mb, mo = _guarded((rows, D), torch.bfloat16)
    dit3d.dit_adaln_modulate(x, gamma, beta, 111, out=mo)
    rb, ro = _guarded((rows, D), torch.bfloat16)
    dit3d.dit_gated_residual(x, y, alpha, 111, out=ro)
    eb, eo = _guarded((rows, D), torch.bfloat16)
    dit3d.dit_flow_euler_step(x, y, torch.tensor([0.1, 0.2, 0.3], device="cuda"), 111, out=eo)
    dit3d.dit_check_device()
    checks += [("modulate", _intact(mb, mo.numel())), ("residual", _intact(rb, ro.numel())),
               ("euler", _intact(eb, eo.numel()))]

    w = bf(200, D)                                 # N = 200: not a multiple of the 256-wide tile
    lb, lo = _guarded((rows, 200), torch.bfloat16)
    dit3d.dit_linear(x, w, out=lo)
    dit3d.dit_check_device()
    checks.append(("linear", _intact(lb, lo.numel())))

    cb, codes = _guarded((rows, H, d), torch.uint8)
    dit3d.dit_quantize_e4m3(q, 64.0, out=codes)
    q8, k8, v8 = (dit3d.dit_quantize_e4m3(t, 64.0) for t in (q, k, v))
    fb, fo = _guarded((rows, H, d), torch.bfloat16)
    dit3d.dit_attn_fwd_fp8(q8, k8, v8, 1 / 64, 1 / 64, 1 / 64, out=fo)
    dit3d.dit_check_device()
    checks += [("quantize", _intact(cb, codes.numel())), ("fp8 attention", _intact(fb, fo.numel()))]

    # dense rows whose units run split by key range (clusters merging partial results)
    rs = 1100                                     # a last query-tile pair with one empty tile
    qs, ks, vs = bf(rs, H, d), bf(rs, H, d), bf(rs, H, d)
    sb, so = _guarded((rs, H, d), torch.bfloat16)
    slb, sl = _guarded((rs, H), torch.float32)
    assert L.dit_attn_fwd(ctypes.c_void_p(qs.data_ptr()), ctypes.c_void_p(ks.data_ptr()),
                          ctypes.c_void_p(vs.data_ptr()), ctypes.c_void_p(so.data_ptr()),
                          ctypes.c_void_p(sl.data_ptr()), rs, H, d, 1, None, None, 0.0, None, st) == 0
    dit3d.dit_check_device()
    assert L.dit_debug_last_attn_split() >= 2
    checks += [("split attention", _intact(sb, so.numel())), ("split lse", _intact(slb, sl.numel()))]

    bad = [name for name, ok in checks if not ok]
    assert not bad, f"guard regions overwritten by: {bad}"


def _raw_attn(entry, q, k, v, o, lse, desc):
    import ctypes
    rows, H, d = q.shape
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = getattr(dit3d.lib(), entry)(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), rows, H, d, 1, None, None,
        0.0, None if desc is None else ctypes.byref(desc), st)
    assert status == 0, dit3d.lib().dit_status_string(status)
    dit3d.dit_check_device()


@pytest.mark.parametrize("variant", [0, 1])
def test_guards_survive_rope_attention_and_the_pair_kernel(variant):
    # The CTA-pair kernel covers 512 query rows per pair, so 333 rows leave most of its
    # last pair past the end; the in-kernel RoPE rotates the ragged tile in place; the
    # allocation-free call writes its table into the library's own array.
    g = torch.Generator(device="cuda").manual_seed(5)
    rows, H, d = 333, 3, 128
    bf = lambda *s: torch.randn(*s, device="cuda", generator=g).to(torch.bfloat16)
    q, k, v = bf(rows, H, d), bf(rows, H, d), bf(rows, H, d)
    desc = dit3d.rope_desc(9, 37, (44, 42, 42))
    dit3d.dit_set_attn_variant(variant)
    try:
        bad = []
        for entry, rope in (("dit_attn_fwd", None), ("dit_attn_fwd", desc),
                            ("dit_attn_fwd_noalloc", desc)):
            ob, o = _guarded((rows, H, d), torch.bfloat16)
            lb, lse = _guarded((rows, H), torch.float32)
            _raw_attn(entry, q, k, v, o, lse, rope)
            if not (_intact(ob, o.numel()) and _intact(lb, lse.numel())):
                bad.append((entry, rope is not None))
        assert not bad, f"variant {variant}: guard regions overwritten by {bad}"
    finally:
        dit3d.dit_set_attn_variant(0)
