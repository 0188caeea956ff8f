"""Pins of the oracle's routing, permutation, SwiGLU and combine steps."""
import numpy as np
import scipy.special

import oracle
from oracle import moe
from bit_linear_moe_b200 import synth


def test_topk_equals_stable_full_sort():
    rng = np.random.default_rng(0)
    l = rng.standard_normal((64, 512))
    l[3, 100] = l[3, 7] = 9.0                  # a tie at the top: index 7 first
    l[4, :] = 0.0                              # all equal: indices 0..9
    idx, w = moe.topk(l, 10)
    ref = np.argsort(-l, axis=1, kind="stable")[:, :10]
    assert np.array_equal(idx, ref)
    assert list(idx[3, :2]) == [7, 100]
    assert list(idx[4]) == list(range(10))


def test_topk_weights_are_renormalised_softmax():
    rng = np.random.default_rng(1)
    l = 3 * rng.standard_normal((32, 512))
    idx, w = moe.topk(l, 10)
    p = scipy.special.softmax(l, axis=1)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    assert np.allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-12)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-12)
    assert (np.diff(w, axis=1) <= 0).all()     # slots in descending weight


def test_topk_with_k_equal_E_is_full_softmax():
    l = np.random.default_rng(2).standard_normal((4, 16))
    idx, w = moe.topk(l, 16)
    full = scipy.special.softmax(l, axis=1)
    assert np.allclose(np.take_along_axis(full, idx.astype(np.int64), axis=1), w, rtol=1e-12)


def test_router_logits_hand_computed():
    """l[t, e] = sum_h h[t, h] * Wr[e, h] + bias[e], worked by hand: a one-hot
    token reads one column of Wr, a token of ones the row sums, and the bias is
    added per expert (not per token).  A transposed Wr, a bias broadcast along
    the wrong axis or a dropped bias gives other numbers."""
    H, E = 4, 3
    wr = np.array([[1.0, 2.0, 3.0, 4.0],
                   [-1.0, 0.5, 0.0, 2.0],
                   [0.25, 0.0, -2.0, 1.0]], dtype=np.float32)   # [E, H]
    bias = np.array([10.0, 20.0, 30.0], dtype=np.float32)
    h = np.array([[0.0, 1.0, 0.0, 0.0],                          # selects column 1 of Wr
                  [1.0, 1.0, 1.0, 1.0],                          # row sums of Wr
                  [2.0, 0.0, 0.0, -1.0]], dtype=np.float32)
    l = moe.router_logits(h, wr, bias)
    expected = np.array([[2.0 + 10, 0.5 + 20, 0.0 + 30],
                         [10.0 + 10, 1.5 + 20, -0.75 + 30],
                         [-2.0 + 10, -4.0 + 20, -0.5 + 30]])
    assert l.shape == (3, E)
    assert np.array_equal(l, expected)
    assert np.array_equal(moe.router_logits(h, wr), expected - bias[None, :].astype(np.float64))


def test_router_logits_exact_in_fp64():
    """bf16 x bf16 products have at most 16 significant bits, so at H = 2048 the
    fp64 sum is exact: it equals the exact rational sum (brute force with
    Fractions on a few tokens and experts)."""
    from fractions import Fraction
    h = synth.moe_hidden(2)
    wr = synth.moe_router()
    l = moe.router_logits(h, wr)
    for t in range(2):
        for e in (0, 17, 511):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(h[t], wr[e]))
            assert Fraction(l[t, e]) == exact


def test_zipf_bias_is_log_prior():
    b = synth.moe_zipf_bias()
    ranks = np.rint(np.exp(-b.astype(np.float64) / 1.1)).astype(int)
    assert sorted(ranks) == list(range(1, 513))


def test_permutation_is_stable_argsort_and_inverse():
    rng = np.random.default_rng(3)
    T, E, k = 50, 16, 4
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, perm_tok, perm_slot, row_of = moe.permute(idx, E)
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.array_equal(np.diff(offsets), np.bincount(idx.ravel(), minlength=E))
    key = idx.astype(np.int64) * T + np.arange(T)[:, None]
    order = np.argsort(key.ravel(), kind="stable")
    assert np.array_equal(perm_tok, order // k) and np.array_equal(perm_slot, order % k)
    assert np.array_equal(row_of[perm_tok, perm_slot], np.arange(T * k))
    for e in range(E):
        assert (idx[perm_tok[offsets[e]:offsets[e + 1]], perm_slot[offsets[e]:offsets[e + 1]]] == e).all()


def test_swiglu_matches_library_sigmoid():
    gu = 4 * np.random.default_rng(4).standard_normal((7, 64))
    a = moe.swiglu(gu)
    assert np.allclose(a, gu[:, :32] * scipy.special.expit(gu[:, :32]) * gu[:, 32:], rtol=1e-13, atol=1e-15)


def test_combine_matches_einsum():
    rng = np.random.default_rng(5)
    T, k, H = 6, 3, 8
    d = rng.standard_normal((T * k, H))
    w = rng.random((T, k))
    row_of = rng.permutation(T * k).reshape(T, k).astype(np.int32)
    y, b = moe.combine(d, w, row_of)
    assert np.allclose(y, np.einsum("tj,tjh->th", w, d[row_of]), rtol=1e-13)
    assert np.allclose(b, np.einsum("tj,tjh->th", w, np.abs(d[row_of])), rtol=1e-13)


def test_grouped_linear_equals_per_row_linear():
    rng = np.random.default_rng(6)
    E, T, k, K, N = 4, 5, 2, 64, 32
    x = synth.activations(rng, T, K)
    qs = [oracle.quantize(synth.weight(rng, N, K)) for _ in range(E)]
    wc = np.stack([q[0] for q in qs]); ws = np.stack([q[1] for q in qs])
    gs = np.array([q[2] for q in qs], np.float32)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, perm_tok, perm_slot, row_of = moe.permute(idx, E)
    y, _ = moe.grouped_linear_w4a16(x, offsets, perm_tok, wc, ws, gs, gather=True)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            ref, _ = oracle.linear_w4a16(x[t:t + 1], wc[e], ws[e], gs[e])
            assert np.array_equal(y[row_of[t, j]], ref[0])
