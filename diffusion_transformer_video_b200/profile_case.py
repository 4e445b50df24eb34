"""Runs one libdit3d call at a chosen size, a few times, for a profiler to capture.

    python -m diffusion_transformer_video_b200.profile_case --kernel modulate --rows 54560 --d-model 3072
    python -m diffusion_transformer_video_b200.profile_case --kernel attn --rows 32760 --heads 16

Inputs are seeded bf16 normals made on the device (torch's generator): the sizes are
those of a workload, held small enough (one call's operands) for a capture that ends
on its own. Each call is one launch of the kernel named by --kernel; --iters calls
follow --warmup untimed ones, and the script reports the mean time per call measured
with CUDA events (a figure taken under a profiler is not a benchmark number).
"""
from __future__ import annotations

import argparse
import statistics

import torch

from . import dit3d


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", required=True,
                    choices=["modulate", "residual", "rope", "attn", "attn_rope", "euler", "linear"])
    ap.add_argument("--rows", type=int, required=True)
    ap.add_argument("--d-model", type=int, default=0, help="activation width (modulate, residual, euler)")
    ap.add_argument("--heads", type=int, default=0)
    ap.add_argument("--head-dim", type=int, default=128)
    ap.add_argument("--n-seq", type=int, default=1, help="attention: equal dense sequences")
    ap.add_argument("--rows-per-group", type=int, default=0, help="default: every row one group")
    ap.add_argument("--grid", type=int, nargs=2, default=(30, 52), help="patch grid (RoPE)")
    ap.add_argument("--bands", type=int, nargs=3, default=(44, 42, 42))
    ap.add_argument("--n-out", type=int, default=0, help="linear: output features")
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args()

    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(a.seed)
    bf = lambda *s, std=1.0: (torch.randn(*s, device="cuda", generator=g) * std).to(torch.bfloat16)
    rows = a.rows
    D = a.d_model or a.heads * a.head_dim
    rpg = a.rows_per_group or rows
    if a.kernel in ("modulate", "residual", "euler"):
        x, y = bf(rows, D), bf(rows, D)
        prm = bf(rows // rpg, D, std=0.1), bf(rows // rpg, D, std=0.1)
        out = torch.empty_like(x)
        dt = torch.rand(rows // rpg, device="cuda", generator=g) * 0.1
        call = {"modulate": lambda: dit3d.dit_adaln_modulate(x, prm[0], prm[1], rpg, out=out),
                "residual": lambda: dit3d.dit_gated_residual(x, y, prm[0], rpg, out=out),
                "euler": lambda: dit3d.dit_flow_euler_step(x, y, dt, rpg, out=out)}[a.kernel]
    elif a.kernel in ("rope", "attn", "attn_rope"):
        H, d = a.heads, a.head_dim
        q, k, v = bf(rows, H, d), bf(rows, H, d), bf(rows, H, d)
        frame = a.grid[0] * a.grid[1]
        desc = dit3d.rope_desc(a.grid[0], a.grid[1], a.bands)
        if a.kernel == "rope":
            qo, ko = torch.empty_like(q), torch.empty_like(k)
            if rows % frame:
                raise SystemExit(f"rows must be whole frames of {frame} tokens")
            call = lambda: dit3d.dit_rope3d_qk(q, k, desc, q_out=qo, k_out=ko)
        else:
            o = torch.empty_like(q)
            # attn_rope: q and k rotated inside the attention kernel (fused 3D-RoPE)
            rope = desc if a.kernel == "attn_rope" else None
            if rows % a.n_seq:
                raise SystemExit(f"rows must split into {a.n_seq} equal sequences")
            call = lambda: dit3d.dit_attn_fwd(q, k, v, n_seq=a.n_seq, out=o, rope=rope)
    else:
        K, N = D, a.n_out or 3 * D
        x, w = bf(rows, K), bf(N, K, std=K ** -0.5)
        out = torch.empty(rows, N, dtype=torch.bfloat16, device="cuda")
        call = lambda: dit3d.dit_linear(x, w, out=out)

    for _ in range(a.warmup):
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(a.iters)]
    for e0, e1 in evs:
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    dit3d.dit_check_device()
    print(f"{a.kernel} rows={rows}: {statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs):.4f} ms "
          f"per call (mean of {a.iters})")


if __name__ == "__main__":
    main()
