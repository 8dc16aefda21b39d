"""Pins for the oracle's ragged-batch forward: a single sequence is the plain
forward; equal lengths are the batched forward; sequences do not interact
(changing one leaves the others' rows unchanged); empty sequences and a
brute-force tiny case."""
import math

import numpy as np

from oracle import sdpa_forward, sdpa_varlen_forward

RNG = np.random.default_rng


def _rand(shape, seed):
    return RNG(seed).standard_normal(shape)


def test_single_sequence_is_the_plain_forward():
    q, k, v = _rand((37, 3, 8), 400), _rand((37, 3, 8), 401), _rand((37, 3, 8), 402)
    o, lse = sdpa_varlen_forward(q, k, v, [0, 37], [0, 37], causal=True, scale=0.4)
    o2, l2 = sdpa_forward(q.transpose(1, 0, 2)[None], k.transpose(1, 0, 2)[None], v.transpose(1, 0, 2)[None],
                          causal=True, scale=0.4)
    np.testing.assert_array_equal(o, o2[0].transpose(1, 0, 2))
    np.testing.assert_array_equal(lse, l2[0])


def test_equal_lengths_are_the_batched_forward():
    B, n, H, d = 3, 11, 2, 4
    q, k, v = _rand((B * n, H, d), 410), _rand((B * n, H, d), 411), _rand((B * n, H, d), 412)
    cu = [0, n, 2 * n, 3 * n]
    o, lse = sdpa_varlen_forward(q, k, v, cu, cu, causal=False, scale=0.7)
    to4 = lambda x: x.reshape(B, n, H, d).transpose(0, 2, 1, 3)
    o2, l2 = sdpa_forward(to4(q), to4(k), to4(v), scale=0.7)
    np.testing.assert_allclose(o, o2.transpose(0, 2, 1, 3).reshape(B * n, H, d), atol=1e-15)
    np.testing.assert_allclose(lse, l2.transpose(1, 0, 2).reshape(H, B * n), atol=1e-15)


def test_sequences_do_not_interact():
    cu_q, cu_k = [0, 5, 5, 12, 20], [0, 9, 12, 19, 20]          # an empty query sequence, a 1-key one
    q, k, v = _rand((20, 2, 4), 420), _rand((20, 2, 4), 421), _rand((20, 2, 4), 422)
    o, lse = sdpa_varlen_forward(q, k, v, cu_q, cu_k, causal=True, scale=0.5)
    k2, v2 = k.copy(), v.copy()
    k2[12:19] += 3.0                                                   # change sequence 2's keys only
    v2[12:19] -= 1.0
    o2, l2 = sdpa_varlen_forward(q, k2, v2, cu_q, cu_k, causal=True, scale=0.5)
    same = np.r_[0:5, 12:20]
    np.testing.assert_array_equal(o[same], o2[same])
    assert not np.allclose(o[5:12], o2[5:12])                          # rows of sequence 2 changed


def test_brute_force_tiny():
    cu_q, cu_k = [0, 2, 5], [0, 3, 4]
    q, k, v = _rand((5, 1, 2), 430), _rand((4, 1, 2), 431), _rand((4, 1, 2), 432)
    o, lse = sdpa_varlen_forward(q, k, v, cu_q, cu_k, causal=True, scale=1.0)
    for b in range(2):
        nq, nk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for i in range(nq):
            sc = []
            for j in range(nk):
                if j > i + nk - nq:
                    continue
                sc.append((j, float(q[cu_q[b] + i, 0] @ k[cu_k[b] + j, 0])))
            if not sc:
                assert np.all(o[cu_q[b] + i] == 0) and lse[0, cu_q[b] + i] == -np.inf
                continue
            mx = max(s for _, s in sc)
            den = sum(math.exp(s - mx) for _, s in sc)
            ref = sum(math.exp(s - mx) * v[cu_k[b] + j, 0] for j, s in sc) / den
            np.testing.assert_allclose(o[cu_q[b] + i, 0], ref, atol=1e-14)
            assert abs(lse[0, cu_q[b] + i] - (mx + math.log(den))) < 1e-14
