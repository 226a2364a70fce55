"""Pins of the oracle's caller-supplied dual transform pair.

Source: Dual-QK summary Sec. 1 and Sec. 3.1 -- queries take an invertible
matrix T and keys its inverse transpose, fixed per KV head, so that query-key
dot products are unchanged before quantization and pruning.  Both matrices
come from the caller.

The pins do not go through the oracle's own product: a permutation scaled by
powers of two transforms exactly (one nonzero per row), so the oracle's cache
and mask must equal those of the untransformed oracle fed numpy's exact
transform; a dense pair must leave the scores of bf16 window tokens at q.k up
to the bf16 rounding of the transformed keys, which the transposed pairing
does not.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc

D = 128


def scaled_cycle(seed, H):
    """T = diag(2^e) P with P a cyclic shift (not symmetric) and T^{-T} = diag(2^-e) P."""
    rng = np.random.default_rng(seed)
    tq = np.zeros((H, D, D), np.float32)
    tk = np.zeros((H, D, D), np.float32)
    for h in range(H):
        shift = 1 + 7 * h
        e = rng.integers(-3, 4, D)
        for i in range(D):
            j = (i + shift) % D
            tq[h, i, j] = 2.0 ** e[i]
            tk[h, i, j] = 2.0 ** -e[i]
    return tq, tk


def dense_pair(seed, H):
    rng = np.random.default_rng(seed)
    tq = np.empty((H, D, D), np.float32)
    tk = np.empty((H, D, D), np.float32)
    for h in range(H):
        t = np.eye(D) + 0.35 * rng.standard_normal((D, D)) / np.sqrt(D)
        t[:, : D // 2] *= 2.0  # anisotropic: the pair is not orthogonal
        tq[h] = t
        tk[h] = np.linalg.inv(t).T
    return tq, tk


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def test_transform_is_the_matrix_vector_product():
    rng = np.random.default_rng(2)
    for _ in range(20):
        A = rng.standard_normal((D, D)).astype(np.float32)
        x = (rng.standard_normal(D) * rng.uniform(0.1, 10)).astype(np.float32)
        want = A.astype(np.float64) @ x.astype(np.float64)
        got = orc.transform(A, x).astype(np.float64)
        # fp32 rounding of an fp64 sum: half an fp32 ulp plus the fp64 rounding of 128 terms
        bound = np.abs(want) * 2.0 ** -24 + (np.abs(A).astype(np.float64) @ np.abs(x)) * 128 * 2.0 ** -53
        assert np.all(np.abs(got - want) <= bound)


@pytest.mark.parametrize("kb,vb,ch0", [(4, 2, 0), (2, 2, 1), (4, 4, 1)])
def test_exact_pair_equals_plain_cache_on_transformed_inputs(kb, vb, ch0):
    B, H, T, G = 2, 2, 70, 3
    rng = np.random.default_rng(40 + kb + ch0)
    k = rng.standard_normal((B, H, T, D)).astype(np.float32)
    v = rng.standard_normal((B, H, T, D)).astype(np.float32)
    q = rng.standard_normal((B, H * G, D)).astype(np.float32)
    tq, tk = scaled_cycle(5, H)
    kt = np.einsum("hij,bhtj->bhti", tk.astype(np.float64), k.astype(np.float64)).astype(np.float32)
    qt = np.stack([np.einsum("ij,bj->bi", tq[hq // G].astype(np.float64), q[:, hq].astype(np.float64))
                   for hq in range(H * G)], 1).astype(np.float32)
    a = orc.Cache(B, H, D, 200, kb, vb, 2, ch0, 0, 1.0, 4, 8, tq, tk)
    b = orc.Cache(B, H, D, 200, kb, vb, 0, ch0, 0, 1.0, 4, 8)
    a.append(k[:, :, :33], v[:, :, :33], 0)
    a.append(k[:, :, 33:], v[:, :, 33:], 33)
    b.append(kt[:, :, :33], v[:, :, :33], 0)
    b.append(kt[:, :, 33:], v[:, :, 33:], 33)
    for name in ("k_codes", "k_scales", "k_ch0", "v_codes", "v_scales", "k_win", "v_win"):
        x, y = getattr(a, name), getattr(b, name)
        assert (x is None) == (y is None)
        if x is not None:
            assert np.array_equal(x, y), name
    ma, _ = orc.select(q, H, 2, 19, tq)
    mb, _ = orc.select(qt, H, 0, 19)
    assert np.array_equal(ma, mb)
    lens = np.array([T, 41], np.int32)
    np.testing.assert_array_equal(a.attention(q, lens, ma, 0.09), b.attention(qt, lens, mb, 0.09))


def test_identity_pair_is_the_untransformed_cache():
    H, T = 2, 40
    rng = np.random.default_rng(9)
    k = rng.standard_normal((1, H, T, D)).astype(np.float32)
    v = rng.standard_normal((1, H, T, D)).astype(np.float32)
    q = rng.standard_normal((1, 2 * H, D)).astype(np.float32)
    eye = np.broadcast_to(np.eye(D, dtype=np.float32), (H, D, D))
    a = orc.Cache(1, H, D, 64, 2, 2, 2, 1, 0, 1.0, 0, 0, eye, eye)
    b = orc.Cache(1, H, D, 64, 2, 2, 0, 1)
    a.append(k, v, 0)
    b.append(k, v, 0)
    assert np.array_equal(a.k_codes, b.k_codes) and np.array_equal(a.k_scales, b.k_scales)
    lens = np.array([T], np.int32)
    np.testing.assert_array_equal(a.attention(q, lens, None, 0.1), b.attention(q, lens, None, 0.1))


def test_dense_pair_keeps_scores_of_window_tokens():
    # every token in the bf16 sink: the scores are (T q).bf16(T^{-T} k), which
    # equal q.k up to the bf16 rounding of the transformed keys
    H, T, G = 2, 48, 2
    rng = np.random.default_rng(17)
    k = rng.standard_normal((1, H, T, D)).astype(np.float32)
    v = rng.standard_normal((1, H, T, D)).astype(np.float32)
    q = (rng.standard_normal((1, H * G, D)) * 2).astype(np.float32)
    tq, tk = dense_pair(3, H)
    c = orc.Cache(1, H, D, 64, 4, 4, 2, 0, 0, 1.0, 64, 0, tq, tk)
    c.append(k, v, 0)
    scale = 1.0 / np.sqrt(D)
    out = c.attention(q, np.array([T], np.int32), None, scale)
    for hq in range(H * G):
        h = hq // G
        qt = tq[h].astype(np.float64) @ q[0, hq]
        kt = k[0, h].astype(np.float64) @ tk[h].T.astype(np.float64)
        s_true = scale * (k[0, h].astype(np.float64) @ q[0, hq])
        # the oracle rounds transformed rows to fp32, keys then to bf16
        s_bf = scale * (bf16(kt.astype(np.float32)) @ qt.astype(np.float32).astype(np.float64))
        s_transposed = scale * (kt @ (tq[h].T.astype(np.float64) @ q[0, hq]))
        tol = 2.0 ** -8 * scale * (np.abs(kt) @ np.abs(qt)) + 1e-6
        assert np.all(np.abs(s_bf - s_true) <= tol)
        assert np.max(np.abs(s_transposed - s_true)) > 20 * np.max(tol)
        p = np.exp(s_bf - s_bf.max())
        np.testing.assert_allclose(out[hq], (p / p.sum()) @ bf16(v[0, h]), rtol=1e-6, atol=1e-9)
