"""Second, independent writing of the oracle in NumPy for tiny grids --
TEST INFRASTRUCTURE ONLY.

It follows the same reading of the pages as the C oracle (FastVideo
sparse-distill article, section "2. 视频稀疏注意力VSA": keep the key blocks a
query block needs and evaluate only those attention weights) but is built
differently: cube membership comes from coordinate arithmetic on the whole
grid at once, selection from a full sort, and the fine pass from dense N x N
attention under an explicit block mask.  Agreement between the two writings is
one of the pins of the C oracle.
"""
import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def cube_of_token(T, H, W, tile):
    """cube id of every token n = (t*H + h)*W + w, and the cube grid size."""
    tt, th, tw = tile
    nh, nw = -(-H // th), -(-W // tw)
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    cube = ((t // tt) * nh + (h // th)) * nw + (w // tw)
    nT = -(-T // tt)
    return cube.reshape(-1), nT * nh * nw


def pool(x, T, H, W, tile):
    """x: float64 [B, N, heads, d] -> means [B, heads, nt, d] over each cube's tokens."""
    cube, nt = cube_of_token(T, H, W, tile)
    B, N, heads, d = x.shape
    onehot = np.zeros((nt, N))
    onehot[cube, np.arange(N)] = 1.0
    sums = np.einsum("jn,bnhd->bhjd", onehot, x)
    return sums / onehot.sum(1)[None, None, :, None]


def select(q, k, T, H, W, tile, topk):
    qp, kp = pool(q, T, H, W, tile), pool(k, T, H, W, tile)
    d = q.shape[-1]
    scores = np.einsum("bhid,bhjd->bhij", qp, kp) / np.sqrt(d)
    nt = scores.shape[-1]
    # sort by (-score, j): lexsort uses the last key as primary
    order = np.lexsort((np.broadcast_to(np.arange(nt), scores.shape), -scores), axis=-1)
    idx = np.sort(order[..., :topk], axis=-1).astype(np.int32)
    return idx, scores


def block_mask(idx, T, H, W, tile):
    """Boolean [B, heads, N, N]: query n may attend key m iff cube(m) is kept by cube(n)."""
    cube, nt = cube_of_token(T, H, W, tile)
    B, heads = idx.shape[:2]
    keep = np.zeros((B, heads, nt, nt), bool)
    bi, hi, ii, _ = np.indices(idx.shape)
    keep[bi, hi, ii, idx] = True
    return keep[:, :, cube][:, :, :, cube]


def masked_attention(q, k, v, mask):
    """Dense softmax attention restricted by mask; q,k,v float64 [B, N, heads, d]."""
    d = q.shape[-1]
    s = np.einsum("bnhd,bmhd->bhnm", q, k) / np.sqrt(d)
    s = np.where(mask, s, -np.inf)
    s = s - s.max(-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(-1, keepdims=True)
    return np.einsum("bhnm,bmhd->bnhd", p, v), p


def phi(x):
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def linear_branch(q, k, v):
    """O(N^2) form: sum_m (phi(q_n).phi(k_m)) v_m / sum_m phi(q_n).phi(k_m)."""
    a = np.einsum("bnhd,bmhd->bhnm", phi(q), phi(k))
    return np.einsum("bhnm,bmhd->bnhd", a, v) / a.sum(-1).transpose(0, 2, 1)[..., None]


def forward(q, k, v, T, H, W, tile, topk, linear=False):
    idx, _ = select(q, k, T, H, W, tile, topk)
    out, _ = masked_attention(q, k, v, block_mask(idx, T, H, W, tile))
    if linear:
        out = out + linear_branch(q, k, v)
    return out, idx
