"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/dit3d.h declares, and rejects bad arguments with the
documented status codes before touching any device."""
import ctypes
import os
import re

import pytest

from diffusion_transformer_video_b200 import build, dit3d

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return dit3d.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "dit3d.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dit_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("dit_adaln_modulate", "dit_rope3d_qk", "dit_attn_fwd", "dit_gated_residual"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert set(names) == set(dit3d.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, name in dit3d.STATUS_NAMES.items():
        assert L.dit_status_string(code).decode().startswith(name)
    assert L.dit_status_string(99) == b"unknown dit_status"


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p(0x10008)


def test_validation_before_any_device_work(L):
    # rows not a multiple of rows_per_group
    assert L.dit_adaln_modulate(FAKE, FAKE, FAKE, FAKE, 10, 64, 3, 1e-6, 1.0, None) == 2
    # D not a multiple of 8
    assert L.dit_gated_residual(FAKE, FAKE, FAKE, FAKE, 4, 12, 4, None) == 2
    # NULL pointer
    assert L.dit_gated_residual(None, FAKE, FAKE, FAKE, 4, 16, 4, None) == 1
    # misaligned pointer
    assert L.dit_adaln_modulate(MISALIGNED, FAKE, FAKE, FAKE, 4, 64, 4, 1e-6, 1.0, None) == 3
    # head_dim 96 unsupported
    assert L.dit_attn_fwd(FAKE, FAKE, FAKE, FAKE, None, 10, 2, 96, 1, None, None, 0.0, None,
                          None) == 2
    # cu_seqlens on host only
    cu = (ctypes.c_int32 * 3)(0, 5, 10)
    assert L.dit_attn_fwd(FAKE, FAKE, FAKE, FAKE, None, 10, 2, 128, 2, None, cu, 0.0, None,
                          None) == 1
    # cu_seqlens not ending at rows / decreasing
    bad = (ctypes.c_int32 * 3)(0, 5, 9)
    assert L.dit_attn_fwd(FAKE, FAKE, FAKE, FAKE, None, 10, 2, 128, 2, FAKE, bad, 0.0, None,
                          None) == 4
    bad = (ctypes.c_int32 * 3)(0, 7, 5)
    assert L.dit_rope3d_qk(FAKE, None, FAKE, None, 5, 2, 128, 2, FAKE, bad,
                           ctypes.byref(dit3d.rope_desc(1, 1, (44, 42, 42))), None) == 4
    # RoPE bands that do not sum to head_dim, odd band, sequence not a whole number of frames
    assert L.dit_rope3d_qk(FAKE, None, FAKE, None, 16, 2, 128, 1, None, None,
                           ctypes.byref(dit3d.rope_desc(2, 2, (44, 42, 40))), None) == 2
    assert L.dit_rope3d_qk(FAKE, None, FAKE, None, 16, 2, 64, 1, None, None,
                           ctypes.byref(dit3d.rope_desc(2, 2, (15, 25, 24))), None) == 2
    assert L.dit_rope3d_qk(FAKE, None, FAKE, None, 18, 2, 64, 1, None, None,
                           ctypes.byref(dit3d.rope_desc(2, 2, (16, 24, 24))), None) == 2
    # RoPE with E4M3 output: codes overlapping a source, codes not 8-byte aligned, a
    # scale that is not finite (q [16, 2, 128] bf16 spans 8 KB from FAKE)
    rope = ctypes.byref(dit3d.rope_desc(2, 2, (44, 42, 42)))
    e4 = lambda qi, ki, qo, ko, qs=1.0, ks=1.0: L.dit_rope3d_qk_e4m3(
        qi, ki, qo, ko, 16, 2, 128, 1, None, None, rope, qs, ks, None)
    apart, apart2 = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    k_in = ctypes.c_void_p(0x40000)
    assert e4(FAKE, None, FAKE, None) == 2
    assert e4(FAKE, None, ctypes.c_void_p(0x10000 + 8192 - 8), None) == 2
    assert e4(FAKE, k_in, apart, ctypes.c_void_p(0x40000 + 4096)) == 2   # k codes on k
    assert e4(FAKE, k_in, apart, ctypes.c_void_p(0x20000 + 4088)) == 2   # codes on codes
    assert e4(FAKE, None, ctypes.c_void_p(0x20004), None) == 3
    assert e4(FAKE, None, apart, None, float("nan")) == 2
    assert e4(FAKE, k_in, apart, apart2, 1.0, float("inf")) == 2
    assert e4(FAKE, None, None, None) == 1
    assert e4(FAKE, k_in, apart, None) == 1


def test_tail_split_rule(L):
    # the split of a dense attention launch's last partial wave, on made-up residency
    def split(units, sms, nk, resident):
        arr = (ctypes.c_int32 * 9)(*resident)
        out = ctypes.c_int32(-7)
        assert L.dit_debug_tail_split(units, sms, nk, arr, ctypes.byref(out)) == 0
        return out.value
    fits = [0, 0, 74, 49, 37, 29, 24, 21, 18]          # every size fits its tail
    # image: 768 units on 148 SMs -> 28 left: 5 x 28 = 140 CTAs, or 4 when 5 does not fit
    assert split(768, 148, 32, fits) == 5
    assert split(768, 148, 32, [0, 0, 74, 49, 37, 24, 24, 21, 18]) == 4
    assert split(5120, 148, 256, fits) == 1               # 480P: 88 left, 2 x 88 > 148
    assert split(8560, 148, 214, fits) == 1               # 720P: 124 left
    assert split(740, 148, 32, fits) == 1                 # whole waves only
    assert split(16, 148, 32, [0, 0, 74, 49, 37, 29, 24, 21, 18]) == 8   # one small wave
    assert split(16, 148, 6, fits) == 3                   # two key tiles per share at least
    assert split(16, 148, 3, fits) == 1                   # too few key tiles to share
    assert split(24, 148, 8, fits) == 4                   # 6 fits the wave, not 8 key tiles
    assert split(28, 148, 32, [0, 0, -1, -1, -1, -1, -1, -1, -1]) == 1   # residency unknown
    out = ctypes.c_int32(0)
    assert L.dit_debug_tail_split(768, 148, 32, None, ctypes.byref(out)) == 1   # DIT_ERR_NULL


@pytest.mark.skipif(os.environ.get("CUDA_VISIBLE_DEVICES", None) is None and
                    not os.path.exists("/dev/nvidia0") is False, reason="GPU present")
def test_valid_call_without_gpu_reports_device_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L.dit_adaln_modulate(FAKE, FAKE, FAKE, FAKE, 4, 64, 4, 1e-6, 1.0, None) == 5
    assert L.dit_rope3d_qk_e4m3(FAKE, None, ctypes.c_void_p(0x20000), None, 16, 2, 128, 1,
                                None, None, ctypes.byref(dit3d.rope_desc(2, 2, (44, 42, 42))),
                                64.0, 1.0, None) == 5


def test_watchdog_poll_loop_with_a_fake_query(L):
    # dit_wait_device's polling loop, driven by a fake query instead of a CUDA event:
    # done after 3 "not yet" answers, failed after 2, never done within 20 ms
    import time
    n = ctypes.c_int64(0)
    assert L.dit_debug_poll_fake(3, 0, 1_000_000, ctypes.byref(n)) == 0 and n.value == 4
    assert L.dit_debug_poll_fake(2, 1, 1_000_000, ctypes.byref(n)) == 6 and n.value == 3
    t0 = time.perf_counter()
    assert L.dit_debug_poll_fake(1 << 60, 0, 20_000, ctypes.byref(n)) == 7
    waited = time.perf_counter() - t0
    assert 0.02 <= waited < 2.0 and n.value > 2
    assert L.dit_debug_poll_fake(0, 0, 0, None) == 0        # done at the first poll
    assert L.dit_debug_poll_fake(5, 0, 0, None) == 7        # no time allowed
    assert L.dit_wait_device(None, -1) == 2                 # rejected before any CUDA call


def test_every_declaration_has_its_own_doc_comment():
    # each function the header declares is directly preceded by its own /* ... */ block
    lines = open(os.path.join(ROOT, "include", "dit3d.h")).read().splitlines()
    for i, line in enumerate(lines):
        m = re.match(r"^(?:int|void|const char\*)\s+(dit_[a-z0-9_]+)\(", line)
        if not m:
            continue
        j = i - 1
        while j >= 0 and lines[j].strip() == "":
            j -= 1
        assert lines[j].rstrip().endswith("*/"), f"{m.group(1)} has no doc comment right above it"
