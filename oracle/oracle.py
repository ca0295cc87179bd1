"""ctypes front-end of the C oracle -- TEST INFRASTRUCTURE ONLY.

Inputs are bf16 tensors (torch, any device; copied to host) or uint16 numpy
arrays holding bf16 bit patterns, in the layout [B, N, heads, d].  Every result
is a numpy array in the oracle's precision (fp64 unless precision="f32").
"""
import ctypes
import functools

import numpy as np

from . import build as _build

_c_int, _c_i64, _p = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p


@functools.lru_cache(maxsize=None)
def lib(precision: str = "f64"):
    _build.build()
    L = ctypes.CDLL(_build.lib_path(precision))
    L.oracle_num_tiles.restype = _c_int
    L.oracle_num_threads.restype = _c_int
    return L


def _real(precision):
    return np.float64 if precision == "f64" else np.float32


def bits(x) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array of bit patterns."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16, x.dtype
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_p)


def _grid_args(T, H, W, tile):
    tt, th, tw = tile
    return [_c_int(T), _c_int(H), _c_int(W), _c_int(tt), _c_int(th), _c_int(tw)]


def num_tiles(T, H, W, tile=(4, 4, 4)) -> int:
    return lib().oracle_num_tiles(*_grid_args(T, H, W, tile))


def num_threads() -> int:
    return lib().oracle_num_threads()


def tile_slots(T, H, W, tile=(4, 4, 4)) -> np.ndarray:
    nt = num_tiles(T, H, W, tile)
    vol = tile[0] * tile[1] * tile[2]
    out = np.empty((nt, vol), np.int64)
    lib().oracle_tile_slots(*_grid_args(T, H, W, tile), _ptr(out))
    return out


def gather(x, B, heads, d, T, H, W, tile=(4, 4, 4)) -> np.ndarray:
    xb = bits(x)
    nt = num_tiles(T, H, W, tile)
    vol = tile[0] * tile[1] * tile[2]
    out = np.empty((B, heads, nt, vol, d), np.uint16)
    lib().oracle_gather(_ptr(xb), _ptr(out), _c_int(B), _c_int(heads), _c_int(d),
                        *_grid_args(T, H, W, tile))
    return out


def scatter(tiles, B, heads, d, T, H, W, tile=(4, 4, 4), fill=None) -> np.ndarray:
    tb = bits(tiles)
    out = np.zeros((B, T * H * W, heads, d), np.uint16) if fill is None else bits(fill).copy()
    lib().oracle_scatter(_ptr(tb), _ptr(out), _c_int(B), _c_int(heads), _c_int(d),
                         *_grid_args(T, H, W, tile))
    return out


def pool(x, B, heads, d, T, H, W, tile=(4, 4, 4), precision="f64") -> np.ndarray:
    xb = bits(x)
    nt = num_tiles(T, H, W, tile)
    out = np.empty((B, heads, nt, d), _real(precision))
    lib(precision).oracle_pool(_ptr(xb), _c_int(B), _c_int(heads), _c_int(d),
                               *_grid_args(T, H, W, tile), _ptr(out))
    return out


def coarse(qp: np.ndarray, kp: np.ndarray, precision="f64", with_probs=False):
    B, heads, nt, d = qp.shape
    R = _real(precision)
    qp = np.ascontiguousarray(qp, R)
    kp = np.ascontiguousarray(kp, R)
    sc = np.empty((B, heads, nt, nt), R)
    pr = np.empty((B, heads, nt, nt), R) if with_probs else None
    lib(precision).oracle_coarse(_ptr(qp), _ptr(kp), _c_int(B), _c_int(heads), _c_int(nt),
                                 _c_int(d), _ptr(sc), _ptr(pr) if with_probs else None)
    return (sc, pr) if with_probs else sc


def topk(scores: np.ndarray, k: int, precision="f64") -> np.ndarray:
    B, heads, nt, nk = scores.shape
    assert nt == nk, "scores must be [B, heads, nt, nt]"
    sc = np.ascontiguousarray(scores, _real(precision))
    idx = np.empty((B, heads, nt, k), np.int32)
    lib(precision).oracle_topk(_ptr(sc), _c_int(B), _c_int(heads), _c_int(nt), _c_int(k),
                               _ptr(idx))
    return idx


def select(q, k, B, heads, d, T, H, W, topk_, tile=(4, 4, 4), precision="f64",
           with_scores=False):
    qb, kb = bits(q), bits(k)
    nt = num_tiles(T, H, W, tile)
    idx = np.empty((B, heads, nt, topk_), np.int32)
    sc = np.empty((B, heads, nt, nt), _real(precision)) if with_scores else None
    lib(precision).oracle_select(_ptr(qb), _ptr(kb), _c_int(B), _c_int(heads), _c_int(d),
                                 *_grid_args(T, H, W, tile), _c_int(topk_), _ptr(idx),
                                 _ptr(sc) if with_scores else None)
    return (idx, sc) if with_scores else idx


def fine(q, k, v, idx, B, heads, d, T, H, W, tile=(4, 4, 4), precision="f64") -> np.ndarray:
    qb, kb, vb = bits(q), bits(k), bits(v)
    idx = np.ascontiguousarray(idx, np.int32)
    topk_ = idx.shape[-1]
    out = np.zeros((B, T * H * W, heads, d), _real(precision))
    lib(precision).oracle_fine(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(idx), _c_int(B),
                               _c_int(heads), _c_int(d), *_grid_args(T, H, W, tile),
                               _c_int(topk_), _ptr(out))
    return out


def fine_bwd(q, k, v, dout, idx, B, heads, d, T, H, W, tile=(4, 4, 4), precision="f64"):
    """Gradients (dq, dk, dv), each [B][N][heads][d], of the fine pass with the
    selection idx held fixed, for the output gradient dout (bf16 like q)."""
    qb, kb, vb, gb = bits(q), bits(k), bits(v), bits(dout)
    idx = np.ascontiguousarray(idx, np.int32)
    R = _real(precision)
    dq, dk, dv = (np.empty((B, T * H * W, heads, d), R) for _ in range(3))
    lib(precision).oracle_fine_bwd(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gb), _ptr(idx), _c_int(B),
                                   _c_int(heads), _c_int(d), *_grid_args(T, H, W, tile),
                                   _c_int(idx.shape[-1]), _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


def fine_tiles(q, k, v, idx, rows, B, heads, d, T, H, W, tile=(4, 4, 4),
               precision="f64") -> np.ndarray:
    """Fine pass for a sample of query tiles; rows[r] = (b*heads + head)*nt + i.
    Returns [len(rows), vol, d] in slot order (padded slots are 0)."""
    qb, kb, vb = bits(q), bits(k), bits(v)
    idx = np.ascontiguousarray(idx, np.int32)
    rows = np.ascontiguousarray(rows, np.int64)
    topk_ = idx.shape[-1]
    vol = tile[0] * tile[1] * tile[2]
    out = np.zeros((len(rows), vol, d), _real(precision))
    lib(precision).oracle_fine_tiles(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(idx), _c_int(B),
                                     _c_int(heads), _c_int(d), *_grid_args(T, H, W, tile),
                                     _c_int(topk_), _ptr(rows), _c_i64(len(rows)), _ptr(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    """float32 values -> FP8 E4M3 codes (uint8): nearest, ties to even,
    magnitudes above 448 saturated."""
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().oracle_e4m3_encode(_ptr(x), _c_i64(x.size), _ptr(out))
    return out


def e4m3_decode(codes, precision="f64") -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    out = np.empty(codes.shape, _real(precision))
    lib(precision).oracle_e4m3_decode(_ptr(codes), _c_i64(codes.size), _ptr(out))
    return out


def quant_e4m3_cubes(x, B, heads, d, T, H, W, tile=(4, 4, 4)):
    """Per-(b, head, cube) E4M3 quantisation of a bf16 tensor [B, N, heads, d]:
    (codes uint8 [B, N, heads, d], scales float32 [B, heads, nt])."""
    xb = bits(x)
    nt = num_tiles(T, H, W, tile)
    codes = np.zeros((B, T * H * W, heads, d), np.uint8)
    scales = np.empty((B, heads, nt), np.float32)
    lib().oracle_quant_e4m3_cubes(_ptr(xb), _c_int(B), _c_int(heads), _c_int(d),
                                  *_grid_args(T, H, W, tile), _ptr(codes), _ptr(scales))
    return codes, scales


def dequant_e4m3_cubes(codes, scales, T, H, W, tile=(4, 4, 4)) -> np.ndarray:
    """codes x their cube's scale, fp64, [B, N, heads, d]."""
    slots = tile_slots(T, H, W, tile)
    cube_of = np.empty(T * H * W, np.int64)
    for j, row in enumerate(slots):
        cube_of[row[row >= 0]] = j
    sc = scales.astype(np.float64)[:, :, cube_of]                 # [B, heads, N]
    return e4m3_decode(codes) * sc.transpose(0, 2, 1)[..., None]


def fine_tiles_real(qh, kh, v, idx, rows, B, heads, d, T, H, W, tile=(4, 4, 4)) -> np.ndarray:
    """fine_tiles with real-valued q, k ([B, N, heads, d] fp64) and bf16 v."""
    qh = np.ascontiguousarray(qh, np.float64)
    kh = np.ascontiguousarray(kh, np.float64)
    vb = bits(v)
    idx = np.ascontiguousarray(idx, np.int32)
    rows = np.ascontiguousarray(rows, np.int64)
    vol = tile[0] * tile[1] * tile[2]
    out = np.zeros((len(rows), vol, d), np.float64)
    lib().oracle_fine_tiles_real(_ptr(qh), _ptr(kh), _ptr(vb), _ptr(idx), _c_int(B), _c_int(heads),
                                 _c_int(d), *_grid_args(T, H, W, tile), _c_int(idx.shape[-1]),
                                 _ptr(rows), _c_i64(len(rows)), _ptr(out))
    return out


def fine_real(qh, kh, v, idx, B, heads, d, T, H, W, tile=(4, 4, 4)) -> np.ndarray:
    """Fine pass with real-valued q, k over every query tile, grid order."""
    nt = num_tiles(T, H, W, tile)
    rows = np.arange(B * heads * nt, dtype=np.int64)
    part = fine_tiles_real(qh, kh, v, idx, rows, B, heads, d, T, H, W, tile)
    slots = tile_slots(T, H, W, tile)
    out = np.zeros((B, T * H * W, heads, d), np.float64)
    for r in range(len(rows)):
        bh, i = divmod(r, nt)
        b, hd = divmod(bh, heads)
        ok = slots[i] >= 0
        out[b, slots[i][ok], hd] = part[r][ok]
    return out


def weights(q, k, idx, b, head, n, B, heads, d, T, H, W, tile=(4, 4, 4)) -> np.ndarray:
    qb, kb = bits(q), bits(k)
    idx = np.ascontiguousarray(idx, np.int32)
    out = np.empty((T * H * W,), np.float64)
    lib().oracle_weights(_ptr(qb), _ptr(kb), _ptr(idx), _c_int(B), _c_int(heads), _c_int(d),
                         *_grid_args(T, H, W, tile), _c_int(idx.shape[-1]), _c_int(b),
                         _c_int(head), _c_i64(n), _ptr(out))
    return out


def linear_state(k, v, B, heads, d, N, precision="f64"):
    kb, vb = bits(k), bits(v)
    R = _real(precision)
    S = np.empty((B, heads, d, d), R)
    z = np.empty((B, heads, d), R)
    lib(precision).oracle_linear_state(_ptr(kb), _ptr(vb), _c_int(B), _c_int(heads), _c_int(d),
                                       _c_i64(N), _ptr(S), _ptr(z))
    return S, z


def linear_apply(q, S, z, B, heads, d, N, precision="f64") -> np.ndarray:
    qb = bits(q)
    R = _real(precision)
    S = np.ascontiguousarray(S, R)
    z = np.ascontiguousarray(z, R)
    out = np.empty((B, N, heads, d), R)
    lib(precision).oracle_linear_apply(_ptr(qb), _ptr(S), _ptr(z), _c_int(B), _c_int(heads),
                                       _c_int(d), _c_i64(N), _ptr(out))
    return out


def linear_bwd(q, k, v, dout, B, heads, d, N, precision="f64"):
    """Gradients (dq, dk, dv) of the linear branch phi(q)S / (phi(q).z) for
    the output gradient dout (bf16), each [B][N][heads][d]."""
    qb, kb, vb, gb = bits(q), bits(k), bits(v), bits(dout)
    R = _real(precision)
    dq, dk, dv = (np.empty((B, N, heads, d), R) for _ in range(3))
    lib(precision).oracle_linear_bwd(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gb), _c_int(B), _c_int(heads),
                                     _c_int(d), _c_i64(N), _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


def dense(q, k, v, B, heads, d, N, precision="f64") -> np.ndarray:
    qb, kb, vb = bits(q), bits(k), bits(v)
    out = np.empty((B, N, heads, d), _real(precision))
    lib(precision).oracle_dense(_ptr(qb), _ptr(kb), _ptr(vb), _c_int(B), _c_int(heads),
                                _c_int(d), _c_i64(N), _ptr(out))
    return out


def forward(q, k, v, B, heads, d, T, H, W, topk_, tile=(4, 4, 4), linear=False,
            precision="f64"):
    """Whole path: select, fine (+ linear branch).  Returns (out, idx)."""
    idx = select(q, k, B, heads, d, T, H, W, topk_, tile, precision)
    out = fine(q, k, v, idx, B, heads, d, T, H, W, tile, precision)
    if linear:
        S, z = linear_state(k, v, B, heads, d, T * H * W, precision)
        out = out + linear_apply(q, S, z, B, heads, d, T * H * W, precision)
    return out, idx
