"""Pins of the CPU oracle against facts that do not come from the oracle itself:
closed forms, invariants, library routines, brute force on tiny inputs and an
independent NumPy writing of the method.  CPU only."""
import itertools
import json
import os

import numpy as np
import pytest
import torch

from block_sparse_attention_30_b200 import synth
from oracle import numpy_twin as twin

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# (T, H, W, tile, heads, d, topk) -- tiny grids, incl. ragged ones
TINY = [
    (2, 4, 4, (2, 2, 2), 2, 8, 2),
    (4, 8, 8, (4, 4, 4), 2, 16, 2),
    (5, 6, 7, (4, 4, 4), 2, 16, 3),
    (4, 8, 8, (2, 2, 2), 1, 8, 5),
    (3, 5, 9, (2, 2, 2), 2, 8, 7),
]


def _inputs(T, H, W, tile, heads, d, seed=0, B=1, amplitude=1.0):
    return synth.make_qkv(B, heads, d, T, H, W, tile, amplitude, seed)


def _f64(x):
    return x.to(torch.float64).numpy()


# ------------------------------------------------------------------ tiling map

def test_tile_map_matches_coordinate_formula(oracle_mod):
    for T, H, W, tile, *_ in TINY:
        slots = oracle_mod.tile_slots(T, H, W, tile)
        cube, nt = twin.cube_of_token(T, H, W, tile)
        assert slots.shape[0] == nt
        valid = slots[slots >= 0]
        # bijection onto the grid's tokens
        assert np.array_equal(np.sort(valid), np.arange(T * H * W))
        # every token sits in the cube the coordinate formula names
        for j in range(nt):
            toks = slots[j][slots[j] >= 0]
            assert np.all(cube[toks] == j)


def test_ragged_720p_tile_classes_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "ragged_720p_tile_classes.json")))
    slots = oracle_mod.tile_slots(*g["grid"], tuple(g["tile"]))
    assert slots.shape[0] == g["num_tiles"]
    counts = (slots >= 0).sum(1)
    hist = {str(c): int((counts == c).sum()) for c in np.unique(counts)}
    assert hist == g["valid_count_histogram"]
    assert counts.sum() == g["total_valid_tokens"]


# ------------------------------------------------------------- gather/scatter

@pytest.mark.parametrize("case", TINY)
def test_gather_scatter_roundtrip_bit_exact(oracle_mod, case):
    T, H, W, tile, heads, d, _ = case
    q, _, _ = _inputs(T, H, W, tile, heads, d)
    tiles = oracle_mod.gather(q, 1, heads, d, T, H, W, tile)
    slots = oracle_mod.tile_slots(T, H, W, tile)
    # padded slots are zero, valid slots carry the token's row
    pad = slots < 0
    assert np.all(tiles[:, :, pad] == 0)
    back = oracle_mod.scatter(tiles, 1, heads, d, T, H, W, tile)
    assert np.array_equal(back, oracle_mod.bits(q))


# ------------------------------------------------------------------- pooling

def test_pool_tile_constant_is_exact(oracle_mod):
    """P6: a tile-constant input pools to that constant exactly (valid-count
    division; dividing by the full tile volume would fail on ragged cubes)."""
    T, H, W, tile, heads, d = 5, 6, 7, (4, 4, 4), 2, 4
    cube, nt = twin.cube_of_token(T, H, W, tile)
    vals = torch.arange(nt * heads * d, dtype=torch.float32).reshape(nt, heads, d) / 8 - 3
    x = vals[torch.as_tensor(cube)].unsqueeze(0).to(torch.bfloat16)   # [1,N,heads,d]
    p = oracle_mod.pool(x, 1, heads, d, T, H, W, tile)
    expect = vals.permute(1, 0, 2).to(torch.bfloat16).to(torch.float64).numpy()[None]
    assert np.array_equal(p, expect)


# ------------------------------------------------------------------ selection

@pytest.mark.parametrize("case", TINY)
def test_select_matches_numpy_twin(oracle_mod, case):
    T, H, W, tile, heads, d, k = case
    q, kk, _ = _inputs(T, H, W, tile, heads, d, seed=3)
    idx, sc = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile, with_scores=True)
    tidx, tsc = twin.select(_f64(q), _f64(kk), T, H, W, tile, k)
    np.testing.assert_allclose(sc, tsc, rtol=0, atol=1e-12)
    assert np.array_equal(idx, tidx)
    assert np.all(np.diff(idx, axis=-1) > 0)        # strictly ascending rows


def test_topk_is_brute_force_best_subset(oracle_mod):
    """P2: the kept set maximises the summed coarse score over all C(nt, k)
    subsets (unique when scores have no ties)."""
    T, H, W, tile, heads, d = 4, 8, 8, (2, 2, 2), 1, 8
    q, kk, _ = _inputs(T, H, W, tile, heads, d, seed=11)
    for k in (1, 2, 3):
        idx, sc = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile, with_scores=True)
        nt = sc.shape[-1]
        for i in range(0, nt, 5):
            row = sc[0, 0, i]
            best = max(itertools.combinations(range(nt), k), key=lambda s: row[list(s)].sum())
            assert tuple(idx[0, 0, i]) == tuple(sorted(best))


def test_topk_ties_go_to_lower_tile_id(oracle_mod):
    scores = np.zeros((1, 1, 6, 6))               # square: nt query x nt key tiles
    scores[0, 0, 0] = [1, 5, 5, 5, 0, 5]          # four-way tie for the top
    scores[0, 0, 1] = [2, 2, 2, 2, 2, 2]          # all equal
    scores[0, 0, 2] = [-1, -2, -3, -4, -5, -6]
    scores[0, 0, 3] = [0, 0, 0, 0, 0, 9]
    idx = oracle_mod.topk(scores, 2)
    assert idx[0, 0, :4].tolist() == [[1, 2], [0, 1], [0, 1], [0, 5]]


def test_coarse_probs_are_row_softmax(oracle_mod):
    rng = np.random.default_rng(0)
    qp, kp = rng.normal(size=(1, 2, 7, 16)), rng.normal(size=(1, 2, 7, 16))
    sc, pr = oracle_mod.coarse(qp, kp, with_probs=True)
    ref = torch.softmax(torch.from_numpy(qp @ kp.transpose(0, 1, 3, 2) / 4.0), -1).numpy()
    np.testing.assert_allclose(pr, ref, atol=1e-14)
    np.testing.assert_allclose(sc, qp @ kp.transpose(0, 1, 3, 2) / 4.0, atol=1e-13)


# ------------------------------------------------------------------ fine pass

@pytest.mark.parametrize("case", TINY)
def test_fine_matches_masked_dense_attention(oracle_mod, case):
    """P2 (fine half): equals dense attention under an explicit N x N block mask."""
    T, H, W, tile, heads, d, k = case
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=5)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile)
    out = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile)
    ref, _ = twin.masked_attention(_f64(q), _f64(kk), _f64(v),
                                   twin.block_mask(idx, T, H, W, tile))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", [(4, 8, 8, (4, 4, 4), 2, 16), (5, 6, 7, (4, 4, 4), 3, 8)])
def test_all_tiles_equals_dense_sdpa(oracle_mod, case):
    """P1: k = nt reduces to dense softmax attention (torch SDPA, fp64 CPU)."""
    T, H, W, tile, heads, d = case
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=7, amplitude=0.7)
    nt = oracle_mod.num_tiles(T, H, W, tile)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, nt, tile)
    assert np.array_equal(idx[0, 0, 0], np.arange(nt))
    out = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile)
    tq, tk, tv = (x.to(torch.float64).permute(0, 2, 1, 3) for x in (q, kk, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    dense = oracle_mod.dense(q, kk, v, 1, heads, d, T * H * W)
    np.testing.assert_allclose(dense, ref.numpy(), rtol=0, atol=1e-12)


def test_weights_sum_to_one_and_vanish_off_selection(oracle_mod):
    """P3: each query's weights sum to one, are zero outside the kept tiles
    (and hence on padded slots), and reproduce the fine output."""
    T, H, W, tile, heads, d, k = 5, 6, 7, (4, 4, 4), 2, 16, 3
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=9)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile)
    out = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile)
    cube, _ = twin.cube_of_token(T, H, W, tile)
    for head in range(heads):
        for n in (0, 17, 101, T * H * W - 1):
            w = oracle_mod.weights(q, kk, idx, 0, head, n, 1, heads, d, T, H, W, tile)
            assert abs(w.sum() - 1.0) < 1e-12
            kept = np.isin(cube, idx[0, head, cube[n]])
            assert np.all(w[~kept] == 0) and np.all(w[kept] > 0)
            np.testing.assert_allclose(w @ _f64(v)[0, :, head], out[0, n, head], atol=1e-12)


def test_permutation_invariance(oracle_mod):
    """P5: the order of a row's indices, and the order of tokens inside a key
    tile, do not change the output."""
    T, H, W, tile, heads, d, k = 4, 8, 8, (2, 2, 2), 2, 8, 4
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=13)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile)
    out = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile)
    rng = np.random.default_rng(1)
    shuffled = np.take_along_axis(idx, rng.permuted(np.broadcast_to(np.arange(k), idx.shape).copy(), axis=-1), -1)
    out2 = oracle_mod.fine(q, kk, v, shuffled, 1, heads, d, T, H, W, tile)
    np.testing.assert_allclose(out, out2, rtol=0, atol=1e-12)
    # swap two tokens of one cube in k and v: cube membership is unchanged
    cube, _ = twin.cube_of_token(T, H, W, tile)
    a, b = np.nonzero(cube == 3)[0][:2]
    k2, v2 = kk.clone(), v.clone()
    k2[:, [a, b]] = kk[:, [b, a]]
    v2[:, [a, b]] = v[:, [b, a]]
    out3 = oracle_mod.fine(q, k2, v2, idx, 1, heads, d, T, H, W, tile)
    np.testing.assert_allclose(out, out3, rtol=0, atol=1e-12)


def test_topk_one_is_single_tile_softmax(oracle_mod):
    """P6: with k = 1 each query attends one tile: an explicit small softmax."""
    T, H, W, tile, heads, d = 4, 8, 8, (4, 4, 4), 1, 16
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=2)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, 1, tile)
    out = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile)
    cube, _ = twin.cube_of_token(T, H, W, tile)
    qf, kf, vf = _f64(q)[0, :, 0], _f64(kk)[0, :, 0], _f64(v)[0, :, 0]
    for n in (0, 63, 200):
        keys = np.nonzero(cube == idx[0, 0, cube[n], 0])[0]
        s = kf[keys] @ qf[n] / 4.0
        p = np.exp(s - s.max()); p /= p.sum()
        np.testing.assert_allclose(out[0, n, 0], p @ vf[keys], atol=1e-12)


def test_fine_tiles_sample_matches_full(oracle_mod):
    T, H, W, tile, heads, d, k = 5, 6, 7, (4, 4, 4), 2, 16, 3
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=4)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile)
    out = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile)
    nt = oracle_mod.num_tiles(T, H, W, tile)
    rows = np.array([0, nt - 1, nt + 3])
    part = oracle_mod.fine_tiles(q, kk, v, idx, rows, 1, heads, d, T, H, W, tile)
    slots = oracle_mod.tile_slots(T, H, W, tile)
    for r, row in enumerate(rows):
        head, i = divmod(int(row), nt)
        for s, n in enumerate(slots[i]):
            if n >= 0:
                assert np.array_equal(part[r, s], out[0, n, head])
            else:
                assert np.all(part[r, s] == 0)


# -------------------------------------------------------------- linear branch

def test_linear_zero_keys_gives_mean_value(oracle_mod):
    """P7: K = 0 makes phi(k) = 1, so every query's linear output is the mean
    of V over all tokens."""
    B, heads, d, T, H, W = 1, 2, 8, 3, 4, 5
    q, _, v = _inputs(T, H, W, (4, 4, 4), heads, d, seed=6)
    kk = torch.zeros_like(q)
    N = T * H * W
    S, z = oracle_mod.linear_state(kk, v, B, heads, d, N)
    lin = oracle_mod.linear_apply(q, S, z, B, heads, d, N)
    mean_v = _f64(v).mean(axis=1)                     # [B, heads, d]
    np.testing.assert_allclose(lin, np.broadcast_to(mean_v[:, None], lin.shape), atol=1e-12)


def test_linear_state_form_matches_quadratic_form(oracle_mod):
    B, heads, d, T, H, W = 1, 2, 8, 3, 4, 5
    q, kk, v = _inputs(T, H, W, (4, 4, 4), heads, d, seed=8)
    N = T * H * W
    S, z = oracle_mod.linear_state(kk, v, B, heads, d, N)
    lin = oracle_mod.linear_apply(q, S, z, B, heads, d, N)
    ref = twin.linear_branch(_f64(q), _f64(kk), _f64(v))
    np.testing.assert_allclose(lin, ref, rtol=1e-12, atol=1e-12)
    # phi is elu + 1 (torch's elu is an independent library routine)
    x = torch.linspace(-5, 5, 101, dtype=torch.float64)
    np.testing.assert_allclose(twin.phi(x.numpy()), (torch.nn.functional.elu(x) + 1).numpy(),
                               atol=1e-15)


def test_linear_state_matches_torch_einsum(oracle_mod):
    B, heads, d, T, H, W = 1, 3, 8, 2, 4, 4
    _, kk, v = _inputs(T, H, W, (4, 4, 4), heads, d, seed=10)
    S, z = oracle_mod.linear_state(kk, v, B, heads, d, T * H * W)
    pk = torch.nn.functional.elu(kk.to(torch.float64)) + 1
    Sref = torch.einsum("bnha,bnhc->bhac", pk, v.to(torch.float64))
    np.testing.assert_allclose(S, Sref.numpy(), rtol=1e-12)
    np.testing.assert_allclose(z, pk.sum(1).numpy(), rtol=1e-12)


def test_whole_path_matches_numpy_twin(oracle_mod):
    T, H, W, tile, heads, d, k = 5, 6, 7, (4, 4, 4), 2, 16, 3
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=12)
    out, idx = oracle_mod.forward(q, kk, v, 1, heads, d, T, H, W, k, tile, linear=True)
    ref, tidx = twin.forward(_f64(q), _f64(kk), _f64(v), T, H, W, tile, k, linear=True)
    assert np.array_equal(idx, tidx)
    np.testing.assert_allclose(out, ref, atol=1e-12)


# ------------------------------------------------------------------ precision

def test_fp32_oracle_far_inside_tolerance(oracle_mod):
    """P8: the same oracle in fp32 differs from fp64 by far less than the
    fine-pass tolerance (max-abs 2e-2, relative Frobenius 1e-2)."""
    T, H, W, tile, heads, d, k = 4, 16, 16, (4, 4, 4), 2, 64, 4
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=1)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile)
    o64 = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile)
    o32 = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile, precision="f32")
    err = np.abs(o64 - o32).max()
    rel = np.linalg.norm(o64 - o32) / np.linalg.norm(o64)
    assert err < 1e-4 and rel < 1e-5


# ------------------------------------------------------------ fine backward

def _dout(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return (0.5 * torch.randn(shape, generator=g)).to(torch.bfloat16)


def _torch_masked_attention(q, k, v, mask):
    """Dense attention restricted by mask, in torch fp64 (autograd-able)."""
    d = q.shape[-1]
    s = torch.einsum("bnhd,bmhd->bhnm", q, k) / np.sqrt(d)
    s = s.masked_fill(~mask, float("-inf"))
    return torch.einsum("bhnm,bmhd->bnhd", torch.softmax(s, -1), v)


@pytest.mark.parametrize("case", TINY)
def test_fine_bwd_matches_autograd_of_masked_dense(oracle_mod, case):
    """P9: the backward equals torch autograd (fp64) of dense attention under
    the explicit N x N block mask -- an independent differentiation path."""
    T, H, W, tile, heads, d, k = case
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=11, amplitude=0.7)
    dout = _dout(q.shape, seed=12)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile)
    dq, dk, dv = oracle_mod.fine_bwd(q, kk, v, dout, idx, 1, heads, d, T, H, W, tile)
    tq, tk, tv = (x.to(torch.float64).requires_grad_() for x in (q, kk, v))
    mask = torch.as_tensor(twin.block_mask(idx, T, H, W, tile))
    out = _torch_masked_attention(tq, tk, tv, mask)
    out.backward(dout.to(torch.float64))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-11)


def test_fine_bwd_all_tiles_equals_sdpa_autograd(oracle_mod):
    """P9 (dense limit): k = nt gives the gradients of torch SDPA (fp64)."""
    T, H, W, tile, heads, d = 4, 8, 8, (4, 4, 4), 2, 16
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=13, amplitude=0.7)
    dout = _dout(q.shape, seed=14)
    nt = oracle_mod.num_tiles(T, H, W, tile)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, nt, tile)
    dq, dk, dv = oracle_mod.fine_bwd(q, kk, v, dout, idx, 1, heads, d, T, H, W, tile)
    tq, tk, tv = (x.to(torch.float64).permute(0, 2, 1, 3).contiguous().requires_grad_() for x in (q, kk, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    out.backward(dout.to(torch.float64).permute(0, 2, 1, 3))
    for mine, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, ref.grad.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-11)


def test_fine_bwd_dv_is_weights_times_dout(oracle_mod):
    """P9: dv_m = sum_n p(n, m) dO_n, with p from the oracle's per-query
    weights (a separate function) -- and keys of tiles nobody keeps get 0."""
    T, H, W, tile, heads, d, k = 5, 6, 7, (4, 4, 4), 1, 8, 2
    q, kk, v = _inputs(T, H, W, tile, heads, d, seed=15)
    dout = _dout(q.shape, seed=16)
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile)
    dq, dk, dv = oracle_mod.fine_bwd(q, kk, v, dout, idx, 1, heads, d, T, H, W, tile)
    N = T * H * W
    P = np.stack([oracle_mod.weights(q, kk, idx, 0, 0, n, 1, heads, d, T, H, W, tile) for n in range(N)])
    ref = P.T @ dout[0, :, 0].to(torch.float64).numpy()
    np.testing.assert_allclose(dv[0, :, 0], ref, rtol=0, atol=1e-12)
    never = P.sum(0) == 0
    assert never.any(), "case should leave some key tiles unselected"
    assert np.all(dk[0, never] == 0) and np.all(dv[0, never] == 0)


# ---------------------------------------------------- linear branch backward

def _torch_linear(q, k, v):
    """phi(q) S / (phi(q) . z) in torch fp64, phi = elu + 1 (autograd-able)."""
    pq, pk = torch.nn.functional.elu(q) + 1, torch.nn.functional.elu(k) + 1
    S = torch.einsum("bnhd,bnhe->bhde", pk, v)
    z = pk.sum(1)                                              # [B, heads, d]
    num = torch.einsum("bnhd,bhde->bnhe", pq, S)
    den = torch.einsum("bnhd,bhd->bnh", pq, z)
    return num / den[..., None]


@pytest.mark.parametrize("case", [(1, 2, 8, 40), (2, 1, 16, 24)])
def test_linear_bwd_matches_autograd(oracle_mod, case):
    """P10: the linear-branch backward equals torch autograd (fp64) of the
    branch written with torch's own elu -- an independent differentiation."""
    B, heads, d, N = case
    g = torch.Generator().manual_seed(sum(case))
    q, k, v = ((0.8 * torch.randn((B, N, heads, d), generator=g)).to(torch.bfloat16) for _ in range(3))
    dout = _dout(q.shape, seed=17)
    dq, dk, dv = oracle_mod.linear_bwd(q, k, v, dout, B, heads, d, N)
    tq, tk, tv = (x.to(torch.float64).requires_grad_() for x in (q, k, v))
    _torch_linear(tq, tk, tv).backward(dout.to(torch.float64))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-11)


def test_linear_bwd_constant_keys_closed_form(oracle_mod):
    """P10: with every key equal, lin_n = mean of v for any q (phi(q) cancels),
    so dq = 0 and dv_m = (sum_n dO_n) / N exactly."""
    B, heads, d, N = 1, 1, 8, 20
    g = torch.Generator().manual_seed(3)
    q, v = ((0.8 * torch.randn((B, N, heads, d), generator=g)).to(torch.bfloat16) for _ in range(2))
    k = (0.8 * torch.randn((1, 1, 1, d), generator=g)).to(torch.bfloat16).expand(B, N, heads, d).contiguous()
    dout = _dout(q.shape, seed=4)
    dq, dk, dv = oracle_mod.linear_bwd(q, k, v, dout, B, heads, d, N)
    np.testing.assert_allclose(dq, 0, atol=1e-12)
    ref = dout.to(torch.float64).sum(1, keepdim=True).numpy() / N
    np.testing.assert_allclose(dv, np.broadcast_to(ref, dv.shape), rtol=0, atol=1e-12)


# ------------------------------------------- low-precision (E4M3) fine pass

def _torch_e4m3(x: np.ndarray) -> np.ndarray:
    """torch's own float32 -> float8_e4m3fn conversion (in-range values)."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch_and_the_format(oracle_mod):
    """P11: every finite code decodes as torch's float8_e4m3fn does, and the
    format's landmarks hold: 1 = 0x38, 2^-9 = 0x01 (least subnormal), 2^-6 =
    0x08 (least normal), 448 = 0x7E (largest), 0x7F / 0xFF are NaN."""
    codes = np.arange(256, dtype=np.uint8)
    got = oracle_mod.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isin(codes, [0x7F, 0xFF])
    np.testing.assert_array_equal(got[finite], ref[finite])
    assert np.isnan(got[~finite]).all()
    assert got[0x38] == 1.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6
    assert got[0x7E] == 448.0 and got[0xFE] == -448.0


def test_e4m3_encode_rounds_to_nearest_even_and_saturates(oracle_mod):
    """P11: encoding equals torch's conversion on random magnitudes over the
    whole range and on every exact midpoint between neighbouring codes (ties
    to even); magnitudes above 448 saturate to the largest finite value."""
    rng = np.random.default_rng(3)
    mags = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000))
    x = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    vals = oracle_mod.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))       # 0 .. 448
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    for arr in (x, mids, -mids):
        np.testing.assert_array_equal(oracle_mod.e4m3_encode(arr), _torch_e4m3(arr))
    big = np.array([448.5, 464.0, 480.0, 1e4, -1e6], np.float32)
    np.testing.assert_array_equal(oracle_mod.e4m3_encode(big), [0x7E, 0x7E, 0x7E, 0x7E, 0xFE])


@pytest.mark.parametrize("case", [(5, 6, 7, (4, 4, 4), 2, 16), (3, 5, 9, (2, 2, 2), 2, 8)])
def test_cube_quantisation_matches_torch(oracle_mod, case):
    """P11: per-cube scale = amax / 448 (fp32) and codes = E4M3(x * (1 /
    scale)) equal the same steps done with torch (max, float32 reciprocal and
    product, float8_e4m3fn); every nonzero cube reaches the largest code."""
    T, H, W, tile, heads, d = case
    q, _, _ = _inputs(T, H, W, tile, heads, d, seed=5, amplitude=0.7)
    codes, scales = oracle_mod.quant_e4m3_cubes(q, 1, heads, d, T, H, W, tile)
    slots = oracle_mod.tile_slots(T, H, W, tile)
    qf = q.float()
    for j, row in enumerate(slots):
        toks = torch.as_tensor(row[row >= 0])
        for h in range(heads):
            blk = qf[0, toks, h]
            sc = (blk.abs().max() / torch.tensor(448.0)).to(torch.float32)
            assert scales[0, h, j] == sc.item()
            inv = (torch.tensor(1.0, dtype=torch.float32) / sc).to(torch.float32)
            ref = _torch_e4m3((blk * inv).numpy())
            np.testing.assert_array_equal(codes[0, row[row >= 0], h], ref)
            assert np.abs(oracle_mod.e4m3_decode(codes[0, row[row >= 0], h])).max() == 448.0


def test_fine_real_equals_fine_on_exactly_representable_inputs(oracle_mod):
    """P11: when every q, k value is an E4M3 value times a power of two and
    each cube holds a +-448 multiple, quantisation is lossless, so the fine
    pass on the dequantised q, k equals the pinned bf16 fine pass."""
    T, H, W, tile, heads, d, k = 5, 6, 7, (4, 4, 4), 2, 16, 3
    rng = np.random.default_rng(11)
    vals = oracle_mod.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    N = T * H * W
    slots = oracle_mod.tile_slots(T, H, W, tile)

    def exact_tensor(seed_shift):
        x = rng.choice(vals, size=(1, N, heads, d)) * rng.choice([-1.0, 1.0], size=(1, N, heads, d))
        for j, row in enumerate(slots):
            for h in range(heads):
                s = 2.0 ** int(rng.integers(-8, -3))
                x[0, row[row >= 0], h] *= s
                x[0, row[row >= 0][0], h, 0] = 448.0 * s             # the cube maximum
        return torch.from_numpy(x).to(torch.bfloat16)

    q, kk = exact_tensor(0), exact_tensor(1)
    _, _, v = _inputs(T, H, W, tile, heads, d, seed=2)
    assert torch.equal(q.double().to(torch.bfloat16), q)            # bf16-exact by construction
    idx = oracle_mod.select(q, kk, 1, heads, d, T, H, W, k, tile)
    cq, sq = oracle_mod.quant_e4m3_cubes(q, 1, heads, d, T, H, W, tile)
    ck, sk = oracle_mod.quant_e4m3_cubes(kk, 1, heads, d, T, H, W, tile)
    qh = oracle_mod.dequant_e4m3_cubes(cq, sq, T, H, W, tile)
    kh = oracle_mod.dequant_e4m3_cubes(ck, sk, T, H, W, tile)
    np.testing.assert_array_equal(qh, q.double().numpy())
    np.testing.assert_array_equal(kh, kk.double().numpy())
    got = oracle_mod.fine_real(qh, kh, v, idx, 1, heads, d, T, H, W, tile)
    ref = oracle_mod.fine(q, kk, v, idx, 1, heads, d, T, H, W, tile)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


# ------------------------------------------------------ property-based pins
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None)
@given(T=st.integers(1, 9), H=st.integers(1, 9), W=st.integers(1, 9),
       tile=st.sampled_from([(4, 4, 4), (2, 4, 8), (8, 2, 4), (1, 8, 8), (2, 2, 2)]))
def test_tile_map_is_a_bijection_for_any_grid(oracle_mod, T, H, W, tile):
    """P5 (any shape): the tiling map sends every token of the grid to exactly
    one slot, of the cube the coordinate formula names, and marks exactly the
    out-of-grid slots as padding."""
    slots = oracle_mod.tile_slots(T, H, W, tile)
    cube, nt = twin.cube_of_token(T, H, W, tile)
    assert slots.shape == (nt, tile[0] * tile[1] * tile[2])
    valid = slots[slots >= 0]
    assert np.array_equal(np.sort(valid), np.arange(T * H * W))
    for j in range(nt):
        assert np.all(cube[slots[j][slots[j] >= 0]] == j)


@settings(max_examples=60, deadline=None)
@given(st.lists(st.floats(-448.0, 448.0, allow_nan=False, width=32), min_size=1, max_size=64))
def test_e4m3_rounding_error_and_monotonicity(oracle_mod, xs):
    """P11 (any value in range): decoding the code of x is within half a step
    of x (a step is 2^(e-3) for 2^e <= |x| < 2^(e+1), 2^-9 below 2^-6), and
    encoding preserves order."""
    x = np.array(xs, np.float32)
    d = oracle_mod.e4m3_decode(oracle_mod.e4m3_encode(x))
    a = np.abs(x.astype(np.float64))
    step = np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -6))) - 3))
    assert np.all(np.abs(d - x) <= step / 2)
    order = np.argsort(x, kind="stable")
    assert np.all(np.diff(d[order]) >= 0)


@settings(max_examples=40, deadline=None)
@given(nt=st.integers(1, 40), k=st.integers(1, 40), levels=st.integers(1, 6), seed=st.integers(0, 2**31 - 1))
def test_topk_matches_a_sort_with_ties_to_the_lower_id(oracle_mod, nt, k, levels, seed):
    """P4 (any row, heavy ties): the kept cubes are the first k of the order
    (score descending, cube id ascending), emitted ascending.  Scores drawn
    from a few levels force ties."""
    k = min(k, nt)
    rng = np.random.default_rng(seed)
    scores = rng.integers(0, levels, size=(1, 2, nt, nt)).astype(np.float64) / levels
    got = oracle_mod.topk(scores, k)
    for h in range(2):
        for i in range(nt):
            row = scores[0, h, i]
            order = np.lexsort((np.arange(nt), -row))
            assert got[0, h, i].tolist() == sorted(order[:k].tolist())
