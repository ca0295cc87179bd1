"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the
CPU oracle.  This module holds no attention arithmetic: it only draws random
tensors.

Recipe (per tensor, in this draw order: q noise, q offset, k noise, k offset,
v noise, v offset, all from one CPU torch.Generator seeded with `seed`):

    x[b, n, head, :] = a * N(0, 1)^d + offset[b, head, cube(n), :]
    offset ~ N(0, 1)^d, one vector per (batch, head, tt x th x tw cube of the
    grid), so that cube means carry information the coarse scores can find.

Values are drawn in fp32 and rounded to bf16 (round-to-nearest-even).
Layout: [B, N, heads, d] with token n = (t*H + h)*W + w.
"""
import torch


def _cube_offsets(gen, B, heads, d, T, H, W, tile):
    tt, th, tw = tile
    nT, nH, nW = -(-T // tt), -(-H // th), -(-W // tw)
    off = torch.randn((B, heads, nT, nH, nW, d), generator=gen, dtype=torch.float32)
    # nearest-neighbour upsample of the cube grid back onto the token grid
    off = off.repeat_interleave(tt, dim=2)[:, :, :T]
    off = off.repeat_interleave(th, dim=3)[:, :, :, :H]
    off = off.repeat_interleave(tw, dim=4)[:, :, :, :, :W]
    # [B, heads, T, H, W, d] -> [B, T*H*W, heads, d]
    return off.permute(0, 2, 3, 4, 1, 5).reshape(B, T * H * W, heads, d)


def make_qkv(B, heads, head_dim, T, H, W, tile=(4, 4, 4), amplitude=1.0, seed=0):
    """Return (q, k, v) bf16 CPU tensors of shape [B, T*H*W, heads, head_dim]."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    N = T * H * W
    out = []
    for _ in range(3):
        x = torch.randn((B, N, heads, head_dim), generator=gen, dtype=torch.float32)
        x.mul_(float(amplitude))
        x.add_(_cube_offsets(gen, B, heads, head_dim, T, H, W, tile))
        out.append(x.to(torch.bfloat16))
    return tuple(out)


def make_workload_inputs(w, seed=None):
    """Inputs of a named workload; the default seed is the workload's position
    in the standard list (so every workload has its own fixed stream)."""
    from .workloads import WORKLOADS
    if seed is None:
        seed = list(WORKLOADS).index(w.name)
    return make_qkv(w.B, w.heads, w.head_dim, w.T, w.H, w.W, w.tile, w.amplitude, seed)
