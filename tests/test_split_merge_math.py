"""The arithmetic of the attention kernel's key-range split, in fp64 on the CPU.

Each CTA of a split unit runs the online softmax over its share of the key tiles in
base 2 with a lazily raised running maximum (the maximum moves only when a tile's
exceeds it by more than 2^8, and O and l are rescaled then), and leaves the
unnormalised O, its maximum m and its row sum l; the cluster merges the shares with
M = max_s m_s, w_s = 2^(m_s - M), o = sum_s w_s O_s / sum_s w_s l_s. This test runs
that algorithm exactly as stated and checks it against softmax attention written
out directly (numpy), for every way of cutting the key tiles the kernel uses
(nk tiles into S shares of floor-divided bounds), including scores sharp enough that
the shares' maxima lie far apart.
"""
import numpy as np
import pytest

TILE = 128
THRESHOLD = 8.0  # log2 units


def _direct(q, k, v, scale):
    s = (q @ k.T) * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p / p.sum(axis=1, keepdims=True)) @ v


def _share(q, k, v, scale_log2, j0, j1, n_keys):
    """Online softmax over key tiles [j0, j1) (keys from n_keys on masked to -inf, as the
    kernel masks a ragged last tile): unnormalised O, lazy maximum m, row sum l."""
    n = q.shape[0]
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    o = np.zeros((n, v.shape[1]))
    for j in range(j0, j1):
        kt, vt = k[j * TILE:(j + 1) * TILE], v[j * TILE:(j + 1) * TILE]
        t = (q @ kt.T) * scale_log2
        t[:, np.arange(j * TILE, (j + 1) * TILE) >= n_keys] = -np.inf
        cand = t.max(axis=1)
        raise_ = cand > m + THRESHOLD
        if j > j0:
            f = np.where(raise_, np.exp2(m - cand), 1.0)
            o *= f[:, None]
            l *= f
        m = np.where(raise_, cand, m)
        p = np.exp2(t - m[:, None])
        l += p.sum(axis=1)
        o += p @ vt
    return o, m, l


def _merge(parts):
    M = np.max([m for _, m, _ in parts], axis=0)
    num = sum(np.exp2(m - M)[:, None] * o for o, m, _ in parts)
    den = sum(np.exp2(m - M) * l for _, m, l in parts)
    return num / den[:, None]


@pytest.mark.parametrize("n_keys,S,q_scale", [(1024, 4, 1.0), (1024, 4, 6.0), (700, 3, 1.0),
                                              (4096, 8, 3.0), (256, 2, 1.0), (2048, 5, 10.0)])
def test_split_merge_equals_softmax_attention(n_keys, S, q_scale):
    rng = np.random.default_rng(n_keys + S)
    d = 64
    q = rng.standard_normal((96, d)) * q_scale
    k = rng.standard_normal((n_keys, d))
    v = rng.standard_normal((n_keys, d))
    nk = -(-n_keys // TILE)
    # pad to whole tiles; the padded keys are masked
    kp = np.vstack([k, np.zeros((nk * TILE - n_keys, d))])
    vp = np.vstack([v, np.zeros((nk * TILE - n_keys, d))])
    scale = d ** -0.5
    parts = []
    for s in range(S):
        j0, j1 = s * nk // S, (s + 1) * nk // S
        parts.append(_share(q, kp, vp, scale * np.log2(np.e), j0, j1, n_keys))
    got = _merge(parts)
    np.testing.assert_allclose(got, _direct(q, k, v, scale), rtol=0, atol=1e-12)


def test_split_bounds_cover_every_tile_once():
    for nk in range(2, 70):
        for S in range(2, min(8, nk // 2) + 1):
            tiles = [j for s in range(S) for j in range(s * nk // S, (s + 1) * nk // S)]
            assert tiles == list(range(nk))
            assert min((s + 1) * nk // S - s * nk // S for s in range(S)) >= 2
