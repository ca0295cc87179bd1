"""The selection kernel forms coarse scores in fp32 and trusts every score
whose distance from the k-th one exceeds twice a bound on the fp32 error;
only the rest are recomputed in fp64.  That bound (doubled once more in the
kernel) is the forward error of a d-term dot product evaluated with fused
multiply-adds on fp32-rounded inputs and scaled by an fp32 1/sqrt(d), with
|k| taken as the largest key norm of the row:

    |C32 - C64| <= (d + 8) * 2^-24 * |q| * |k| / sqrt(d).

These CPU checks emulate that evaluation order exactly (one rounding per FMA,
via fp64 arithmetic rounded to fp32 at every step) on cube-mean-like inputs
and on inputs built for cancellation, and check the bound against the fp64
value.  No GPU is involved."""
import numpy as np
import pytest


def fp32_fma_dot(q32, k32):
    """sum_c q[c] k[c] in feature order, one fp32 rounding per FMA (an fp64
    product plus an fp32 addend is exact before the one rounding)."""
    acc = np.zeros(q32.shape[0], np.float32)
    for c in range(q32.shape[1]):
        acc = (q32[:, c].astype(np.float64) * k32[:, c].astype(np.float64) + acc.astype(np.float64)).astype(np.float32)
    return acc


def kernel_order_score(q32, k32, d):
    """The selection kernel's order: each half of the features summed in
    feature order by its own warp, the halves added in fp32, the sum scaled
    by the fp32 1/sqrt(d)."""
    h = d // 2
    s = fp32_fma_dot(q32[:, :h], k32[:, :h]) + fp32_fma_dot(q32[:, h:], k32[:, h:])
    return s * np.float32(1.0 / np.sqrt(d))


def check(q, k, d):
    q32, k32 = q.astype(np.float32), k.astype(np.float32)
    c32 = kernel_order_score(q32, k32, d)
    c64 = np.einsum("nc,nc->n", q, k) / np.sqrt(d)
    bound = (d + 8) * 2.0 ** -24 * np.linalg.norm(q32, axis=1) * np.linalg.norm(k32, axis=1) / np.sqrt(d)
    err = np.abs(c32.astype(np.float64) - c64)
    assert np.all(err <= bound), float((err / bound).max())
    # the sequential order obeys the same bound
    seq = fp32_fma_dot(q32, k32) * np.float32(1.0 / np.sqrt(d))
    assert np.all(np.abs(seq.astype(np.float64) - c64) <= bound)
    return float((err / bound).max())


@pytest.mark.parametrize("d", [64, 128])
def test_bound_on_cube_mean_like_inputs(d):
    rng = np.random.default_rng(d)
    n = 4000
    # a per-cube offset plus the mean of 64 noisy tokens (the synthetic recipe)
    q = rng.standard_normal((n, d)) + 0.7 * rng.standard_normal((n, d)) / 8
    k = rng.standard_normal((n, d)) + 0.7 * rng.standard_normal((n, d)) / 8
    assert check(q, k, d) < 0.1          # the bound is far from tight on such data


@pytest.mark.parametrize("d", [64, 128])
def test_bound_under_cancellation(d):
    """Large terms that cancel: the result is tiny against |q||k|, where a
    relative bound on the result alone would fail."""
    rng = np.random.default_rng(7 + d)
    n = 2000
    q = rng.standard_normal((n, d)) * 1e3
    k = rng.standard_normal((n, d))
    # make k nearly orthogonal to q, row by row
    k -= (np.einsum("nc,nc->n", q, k) / np.einsum("nc,nc->n", q, q))[:, None] * q
    k += 1e-6 * rng.standard_normal((n, d))
    check(q, k, d)


def test_bound_with_wide_exponent_range():
    rng = np.random.default_rng(3)
    d, n = 128, 2000
    scale = 2.0 ** rng.integers(-20, 20, size=(n, d))
    q = rng.standard_normal((n, d)) * scale
    k = rng.standard_normal((n, d)) / scale
    check(q, k, d)


@pytest.mark.parametrize("d,nt,topk", [(128, 455, 46), (64, 300, 9), (128, 64, 63)])
def test_band_rule_gives_the_fp64_set(d, nt, topk):
    """The kernel's rule end to end on the CPU: fp32 scores in the kernel's
    order, eps = twice the bound with the row's largest key norm, every
    score above the k-th fp32 score + 2 eps kept, every one below it - 2 eps
    dropped, the band ranked by fp64 score (ties to the lower cube).  The
    kept set must equal the fp64 top-k, here on rows built with many
    near-ties around the k-th score."""
    rng = np.random.default_rng(nt + topk)
    for row in range(20):
        q = rng.standard_normal((1, d))
        k = rng.standard_normal((nt, d))
        # pull a third of the keys to within a few fp32 ulps of the k-th score
        s64 = (k @ q[0]) / np.sqrt(d)
        kth = np.sort(s64)[::-1][topk - 1]
        near = rng.choice(nt, nt // 3, replace=False)
        qq = q[0] / np.dot(q[0], q[0])
        k[near] += ((kth * np.sqrt(d) - k[near] @ q[0]) * (1 + 1e-7 * rng.standard_normal(len(near))))[:, None] * qq
        q32, k32 = q.astype(np.float32), k.astype(np.float32)
        c32 = kernel_order_score(np.repeat(q32, nt, 0), k32, d).astype(np.float64)
        c64 = (k @ q[0]) / np.sqrt(d)
        eps = 2 * (d + 8) * 2.0 ** -24 * np.linalg.norm(q32) * np.linalg.norm(k32, axis=1).max() / np.sqrt(d)
        t = np.sort(c32)[::-1][topk - 1]
        above = np.nonzero(c32 > t + 2 * eps)[0]
        band = np.nonzero((c32 <= t + 2 * eps) & (c32 >= t - 2 * eps))[0]
        need = topk - len(above)
        assert 1 <= need <= len(band)
        ranked = sorted(band, key=lambda j: (-c64[j], j))[:need]
        kept = set(above.tolist()) | set(ranked)
        want = set(sorted(range(nt), key=lambda j: (-c64[j], j))[:topk])
        assert kept == want
