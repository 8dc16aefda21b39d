"""Property tests of the oracle on random small problems (hypothesis): bounds and
invariances that hold for any exact softmax attention, whatever the shapes, masks
and scales (convex combinations, lse bounds, row shifts, the bottom-right suffix,
key permutations, linearity in V and in dO, the gate as a post-normalisation
factor, the scale as a factor on the scores)."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import sdpa_forward

SHAPES = st.tuples(st.integers(1, 2), st.integers(1, 2), st.integers(1, 9), st.integers(1, 9), st.integers(1, 5))


@settings(max_examples=60, deadline=None)
@given(shape=SHAPES, causal=st.booleans(), scale=st.floats(0.0, 3.0), seed=st.integers(0, 2**31 - 1))
def test_output_rows_are_convex_combinations_of_visible_values(shape, causal, scale, seed):
    B, H, nq, nk, d = shape
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal(s) for s in ((B, H, nq, d), (B, H, nk, d), (B, H, nk, d)))
    o, lse = sdpa_forward(q, k, v, causal=causal, scale=scale)
    off = nk - nq
    for i in range(nq):
        vis = np.arange(nk) if not causal else np.arange(min(nk, max(0, i + off + 1)))
        if len(vis) == 0:                      # dead row
            assert np.all(o[:, :, i] == 0) and np.all(lse[:, :, i] == -np.inf)
            continue
        lo = v[:, :, vis].min(axis=2) - 1e-12
        hi = v[:, :, vis].max(axis=2) + 1e-12
        assert np.all(o[:, :, i] >= lo) and np.all(o[:, :, i] <= hi)
        s = scale * np.einsum("bhd,bhjd->bhj", q[:, :, i], k[:, :, vis])
        m = s.max(axis=2)
        assert np.all(lse[:, :, i] >= m - 1e-12)
        assert np.all(lse[:, :, i] <= m + np.log(len(vis)) + 1e-12)


@settings(max_examples=40, deadline=None)
@given(shape=SHAPES, shift=st.floats(-50.0, 50.0), seed=st.integers(0, 2**31 - 1))
def test_a_constant_row_shift_moves_only_lse(shape, shift, seed):
    B, H, nq, nk, d = shape
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal(s) for s in ((B, H, nq, d), (B, H, nk, d), (B, H, nk, d)))
    bias = rng.standard_normal((H, nq, nk))
    o0, l0 = sdpa_forward(q, k, v, bias=bias, scale=0.5)
    o1, l1 = sdpa_forward(q, k, v, bias=bias + shift, scale=0.5)
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    np.testing.assert_allclose(l1, l0 + shift, atol=1e-11)


@settings(max_examples=40, deadline=None)
@given(n=st.integers(1, 12), drop=st.integers(0, 11), d=st.integers(1, 4), seed=st.integers(0, 2**31 - 1))
def test_fewer_queries_are_the_last_rows_of_the_square_problem(n, drop, d, seed):
    drop = min(drop, n - 1)
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, 2, n, d)) for _ in range(3))
    o_sq, l_sq = sdpa_forward(q, k, v, causal=True, scale=0.7)
    o, l = sdpa_forward(q[:, :, drop:], k, v, causal=True, scale=0.7)
    np.testing.assert_allclose(o, o_sq[:, :, drop:], atol=1e-14)
    np.testing.assert_allclose(l, l_sq[:, :, drop:], atol=1e-14)


@settings(max_examples=40, deadline=None)
@given(shape=SHAPES, seed=st.integers(0, 2**31 - 1))
def test_permuting_keys_with_their_values_and_bias_columns_changes_nothing(shape, seed):
    # without causal masking the keys form a set: one permutation applied to the rows of K and V
    # and to the bias columns leaves O and lse unchanged (catches K/V or bias index mix-ups)
    B, H, nq, nk, d = shape
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((B, H, nq, d)), rng.standard_normal((B, H, nk, d)), rng.standard_normal((B, H, nk, d))
    bias = rng.standard_normal((B, H, nq, nk))
    perm = rng.permutation(nk)
    o, lse = sdpa_forward(q, k, v, bias=bias, scale=0.6)
    o2, l2 = sdpa_forward(q, k[:, :, perm], v[:, :, perm], bias=bias[..., perm], scale=0.6)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(l2, lse, atol=1e-12)


@settings(max_examples=40, deadline=None)
@given(shape=SHAPES, causal=st.booleans(), a=st.floats(-3, 3), b=st.floats(-3, 3), seed=st.integers(0, 2**31 - 1))
def test_output_is_linear_in_the_values_and_lse_ignores_them(shape, causal, a, b, seed):
    B, H, nq, nk, d = shape
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal((B, H, nq, d)), rng.standard_normal((B, H, nk, d))
    v1, v2 = rng.standard_normal((B, H, nk, d)), rng.standard_normal((B, H, nk, d))
    o1, l1 = sdpa_forward(q, k, v1, causal=causal, scale=0.9)
    o2, _ = sdpa_forward(q, k, v2, causal=causal, scale=0.9)
    o3, l3 = sdpa_forward(q, k, a * v1 + b * v2, causal=causal, scale=0.9)
    np.testing.assert_allclose(o3, a * o1 + b * o2, atol=1e-11)
    np.testing.assert_array_equal(l3, l1)


@settings(max_examples=30, deadline=None)
@given(shape=SHAPES, causal=st.booleans(), seed=st.integers(0, 2**31 - 1))
def test_gate_multiplies_the_normalised_output_only(shape, causal, seed):
    B, H, nq, nk, d = shape
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((B, H, nq, d)), rng.standard_normal((B, H, nk, d)), rng.standard_normal((B, H, nk, d))
    g = 3.0 * rng.standard_normal((B, H, nq, d))
    o, lse = sdpa_forward(q, k, v, causal=causal, scale=0.5)
    og, lg = sdpa_forward(q, k, v, gate=g, causal=causal, scale=0.5)
    np.testing.assert_allclose(og, o / (1.0 + np.exp(-g)), atol=1e-13)
    np.testing.assert_array_equal(lg, lse)


@settings(max_examples=30, deadline=None)
@given(shape=SHAPES, causal=st.booleans(), s=st.floats(0.05, 4.0), seed=st.integers(0, 2**31 - 1))
def test_the_scale_acts_on_the_scores_only(shape, causal, s, seed):
    # scale * (Q K^T) == (s Q) K^T with scale 1: the scale is a factor on the scores, not on V or O
    B, H, nq, nk, d = shape
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((B, H, nq, d)), rng.standard_normal((B, H, nk, d)), rng.standard_normal((B, H, nk, d))
    o, lse = sdpa_forward(q, k, v, causal=causal, scale=s)
    o2, l2 = sdpa_forward(s * q, k, v, causal=causal, scale=1.0)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(l2, lse, atol=1e-12)


@settings(max_examples=25, deadline=None)
@given(shape=SHAPES, causal=st.booleans(), a=st.floats(-2, 2), b=st.floats(-2, 2), seed=st.integers(0, 2**31 - 1))
def test_gradients_are_linear_in_the_upstream_gradient(shape, causal, a, b, seed):
    from oracle import sdpa_backward
    B, H, nq, nk, d = shape
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((B, H, nq, d)), rng.standard_normal((B, H, nk, d)), rng.standard_normal((B, H, nk, d))
    d1, d2 = rng.standard_normal((B, H, nq, d)), rng.standard_normal((B, H, nq, d))
    g1 = sdpa_backward(q, k, v, d1, causal=causal, scale=0.7)
    g2 = sdpa_backward(q, k, v, d2, causal=causal, scale=0.7)
    g3 = sdpa_backward(q, k, v, a * d1 + b * d2, causal=causal, scale=0.7)
    for x1, x2, x3 in zip(g1, g2, g3):
        np.testing.assert_allclose(x3, a * x1 + b * x2, atol=1e-10)
