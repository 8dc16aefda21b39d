"""Property tests of the oracle on random small problems (hypothesis): bounds that
hold for any exact softmax attention, whatever the shapes, masks and scales."""
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
