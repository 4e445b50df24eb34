"""Synthetic workloads and their seeded input generator.

This module holds shapes and random numbers only -- none of the method's
arithmetic -- so that the CUDA path and the fp64 oracle can be fed the same
bf16 bit patterns. Inputs are drawn with ``numpy.random.default_rng`` keyed by
(seed, workload id, tensor id), as float32 normals, then rounded to bf16 with
round-to-nearest-even; the arrays returned are the raw ``uint16`` bf16 bits.

The five workloads follow the clip sizes the source pages discuss:

* ``tiny``   -- a 4x8x8 latent with a 1x2x2 patch (64 tokens, 2 heads of 64).
* ``image``  -- a 128x128 latent (1024x1024 image), T=1, 2x2 patch, 4096 tokens, 24x128.
* ``480p``   -- 81 frames of 480x832 through a 4x8x8 VAE: latent 21x60x104, 1x2x2 patch,
  32760 tokens, 40 heads x 128 (Wan2.2 page: 480P/720P clips, 4x8x8 VAE).
* ``720p``   -- 121 frames of 704x1280 through a 16x16x4 VAE: latent 31x44x80, 27280
  tokens, batch 2, 24x128, with a high-noise and a low-noise parameter set (the
  two-expert split of the Wan2.2 page).
* ``varlen`` -- 8 packed sequences with T_i ~ U{3..21} latent frames of 30x52 patches each
  (Flowception page: variable-length frame insertion, a local time per frame), 24x128.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# tensor ids inside one workload (keep stable: they key the random streams)
TID = {"x": 0, "y": 1, "q": 2, "k": 3, "v": 4, "gamma": 5, "beta": 6, "alpha": 7,
       "frames": 100, "t_local": 101}


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int                 # workload id, part of the rng key
    batch: int               # dense batch (ignored for varlen)
    frames: tuple            # latent frames per sequence (one entry per sequence)
    grid_h: int              # patch-grid height  H_lat / p_h
    grid_w: int              # patch-grid width   W_lat / p_w
    heads: int
    head_dim: int
    bands: tuple             # (d_t, d_h, d_w)
    base: float = 10000.0
    varlen: bool = False
    param_sets: int = 1      # adaLN parameter sets run one after the other (experts)
    per_frame_params: bool = False
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def d_model(self) -> int:
        return self.heads * self.head_dim

    @property
    def frame_tokens(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def seqlens(self) -> list:
        if self.varlen:
            return [t * self.frame_tokens for t in self.frames]
        return [self.frames[0] * self.frame_tokens] * self.batch

    @property
    def n_seq(self) -> int:
        return len(self.seqlens)

    @property
    def rows(self) -> int:
        return int(sum(self.seqlens))

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seqlens))

    @property
    def rows_per_group(self) -> int:
        # one parameter group per sample, or one per latent frame
        return self.frame_tokens if self.per_frame_params else self.seqlens[0]

    @property
    def groups(self) -> int:
        return self.rows // self.rows_per_group

    def attn_flops(self) -> float:
        """Algorithmic attention FLOPs: two matmuls, 4 * L^2 * d per head and sequence."""
        return float(sum(4.0 * L * L * self.head_dim * self.heads for L in self.seqlens))

    def rope_desc(self, offsets=(0, 0, 0)) -> dict:
        return dict(grid_h=self.grid_h, grid_w=self.grid_w, bands=tuple(self.bands),
                    base=self.base, offsets=tuple(offsets))


def varlen_frames(seed: int = 0, n: int = 8, lo: int = 3, hi: int = 21) -> tuple:
    rng = np.random.default_rng([seed, 5, TID["frames"]])
    return tuple(int(t) for t in rng.integers(lo, hi + 1, n))


def get_workload(name: str, seed: int = 0) -> Workload:
    if name == "tiny":
        return Workload("tiny", 1, 1, (4,), 4, 4, 2, 64, (16, 24, 24),
                        note="latent C=16 T=4 H=8 W=8, patch 1x2x2")
    if name == "image":
        return Workload("image", 2, 2, (1,), 64, 64, 24, 128, (32, 48, 48),
                        note="latent 128x128 (1024x1024 image), T=1, patch 2x2")
    if name == "480p":
        return Workload("480p", 3, 1, (21,), 30, 52, 40, 128, (44, 42, 42),
                        note="81x480x832 video, 4x8x8 VAE -> 21x60x104 latent, patch 1x2x2")
    if name == "720p":
        return Workload("720p", 4, 2, (31,), 22, 40, 24, 128, (44, 42, 42), param_sets=2,
                        note="121x704x1280 video, 16x16x4 VAE -> 31x44x80 latent, patch 1x2x2; "
                             "high-noise then low-noise adaLN parameter set")
    if name == "varlen":
        return Workload("varlen", 5, 1, varlen_frames(seed), 30, 52, 24, 128, (44, 42, 42),
                        varlen=True, per_frame_params=True,
                        note="8 packed sequences, T_i ~ U{3..21} frames of 30x52 patches, "
                             "per-frame adaLN parameters")
    raise KeyError(name)


WORKLOADS = ("tiny", "image", "480p", "720p", "varlen")


# ----------------------------------------------------------------------------- random bits

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float64 (exact)."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def normal_bf16(shape, seed: int, wid: int, tid: int, std: float = 1.0,
                param_set: int = 0) -> np.ndarray:
    rng = np.random.default_rng([seed, wid, tid, param_set])
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return f32_to_bf16_bits(a)


def local_times(w: Workload, seed: int = 0) -> np.ndarray:
    """Per-frame local times t_i ~ U[0,1] (recorded only; no network maps them to parameters)."""
    rng = np.random.default_rng([seed, w.wid, TID["t_local"]])
    return rng.random(sum(w.frames) if w.varlen else w.batch * w.frames[0])


def make_inputs(w: Workload, seed: int = 0, which=("x", "y", "q", "k", "v", "gamma", "beta",
                                                   "alpha"), param_set: int = 0,
                alpha_zero: bool = False) -> dict:
    """Seeded bf16 inputs of workload ``w`` as uint16 bit arrays.

    x, y: [rows, D] ~ N(0,1) (block input and attention-branch output);
    q, k, v: [rows, H, d] ~ N(0,1);  gamma, beta, alpha: [G, D] ~ N(0, 0.1)
    (alpha all zero when ``alpha_zero``, the adaLN-Zero initial state).
    """
    rows, D, H, d, G = w.rows, w.d_model, w.heads, w.head_dim, w.groups
    out = {}
    for name in which:
        tid = TID[name]
        if name in ("x", "y"):
            out[name] = normal_bf16((rows, D), seed, w.wid, tid)
        elif name in ("q", "k", "v"):
            out[name] = normal_bf16((rows, H, d), seed, w.wid, tid)
        elif name == "alpha" and alpha_zero:
            out[name] = np.zeros((G, D), dtype=np.uint16)
        else:
            out[name] = normal_bf16((G, D), seed, w.wid, tid, std=0.1, param_set=param_set)
    return out


def sample_rows(w: Workload, per_seq: int = 256, seed: int = 0) -> np.ndarray:
    """Query rows for sampled parity: per sequence the first and last row, the whole
    last 128-row tile, and random rows up to ``per_seq``."""
    rng = np.random.default_rng([seed, w.wid, 999])
    rows = []
    cu = w.cu_seqlens
    for s in range(w.n_seq):
        a, b = int(cu[s]), int(cu[s + 1])
        L = b - a
        tail0 = a + (L - 1) // 128 * 128
        picks = {a, b - 1, *range(tail0, b)}
        extra = max(0, per_seq - len(picks))
        picks |= set(int(r) for r in rng.integers(a, b, extra))
        rows.extend(sorted(picks))
    return np.asarray(rows, dtype=np.int64)
