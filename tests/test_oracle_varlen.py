"""Pins for the oracle's ragged-batch forward: a single sequence is the plain
forward; equal lengths are the batched forward; sequences do not interact
(changing one leaves the others' rows unchanged); a sequence with queries but no
keys has dead rows (closed form); empty sequences and a brute-force tiny case.
The last test plants mistakes in the packing logic and checks that a pin fails."""
import math

import numpy as np
import pytest

import oracle.sdpa as osdpa
from oracle import sdpa_forward, sdpa_varlen_forward

RNG = np.random.default_rng


def _rand(shape, seed):
    return RNG(seed).standard_normal(shape)


def pin_single_sequence_is_the_plain_forward(fn):
    q, k, v = _rand((37, 3, 8), 400), _rand((37, 3, 8), 401), _rand((37, 3, 8), 402)
    o, lse = fn(q, k, v, [0, 37], [0, 37], causal=True, scale=0.4)
    o2, l2 = sdpa_forward(q.transpose(1, 0, 2)[None], k.transpose(1, 0, 2)[None], v.transpose(1, 0, 2)[None],
                          causal=True, scale=0.4)
    np.testing.assert_array_equal(o, o2[0].transpose(1, 0, 2))
    np.testing.assert_array_equal(lse, l2[0])


def pin_equal_lengths_are_the_batched_forward(fn):
    B, n, H, d = 3, 11, 2, 4
    q, k, v = _rand((B * n, H, d), 410), _rand((B * n, H, d), 411), _rand((B * n, H, d), 412)
    cu = [0, n, 2 * n, 3 * n]
    o, lse = fn(q, k, v, cu, cu, causal=False, scale=0.7)
    to4 = lambda x: x.reshape(B, n, H, d).transpose(0, 2, 1, 3)
    o2, l2 = sdpa_forward(to4(q), to4(k), to4(v), scale=0.7)
    np.testing.assert_allclose(o, o2.transpose(0, 2, 1, 3).reshape(B * n, H, d), atol=1e-15)
    np.testing.assert_allclose(lse, l2.transpose(1, 0, 2).reshape(H, B * n), atol=1e-15)


def pin_sequences_do_not_interact(fn):
    cu_q, cu_k = [0, 5, 5, 12, 20], [0, 9, 12, 19, 20]          # an empty query sequence, a 1-key one
    q, k, v = _rand((20, 2, 4), 420), _rand((20, 2, 4), 421), _rand((20, 2, 4), 422)
    o, lse = fn(q, k, v, cu_q, cu_k, causal=True, scale=0.5)
    k2, v2 = k.copy(), v.copy()
    k2[12:19] += 3.0                                                   # change sequence 2's keys only
    v2[12:19] -= 1.0
    o2, l2 = fn(q, k2, v2, cu_q, cu_k, causal=True, scale=0.5)
    same = np.r_[0:5, 12:20]
    np.testing.assert_array_equal(o[same], o2[same])
    assert not np.allclose(o[5:12], o2[5:12])                          # rows of sequence 2 changed


def pin_queries_without_keys_are_dead_rows(fn):
    # sequence 1 has three queries and no keys: O = 0, lse = -inf there; the others are untouched
    cu_q, cu_k = [0, 4, 7, 9], [0, 5, 5, 8]
    q, k, v = _rand((9, 2, 4), 440), _rand((8, 2, 4), 441), _rand((8, 2, 4), 442)
    for causal in (False, True):
        o, lse = fn(q, k, v, cu_q, cu_k, causal=causal, scale=0.6)
        assert np.all(o[4:7] == 0.0) and np.all(lse[:, 4:7] == -np.inf)
        assert np.all(np.isfinite(lse[:, 0:4])) and np.all(np.isfinite(lse[:, 7:9]))


def pin_brute_force_tiny(fn):
    cu_q, cu_k = [0, 2, 5], [0, 3, 4]
    q, k, v = _rand((5, 1, 2), 430), _rand((4, 1, 2), 431), _rand((4, 1, 2), 432)
    o, lse = fn(q, k, v, cu_q, cu_k, causal=True, scale=1.0)
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


PINS = [pin_single_sequence_is_the_plain_forward, pin_equal_lengths_are_the_batched_forward,
        pin_sequences_do_not_interact, pin_queries_without_keys_are_dead_rows, pin_brute_force_tiny]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__[4:])
def test_varlen_pin(pin):
    pin(sdpa_varlen_forward)


def _mutant(kind):
    """sdpa_varlen_forward with one plausible mistake in its packing logic."""
    def fn(q, k, v, cu_q, cu_k, causal=False, scale=None):
        q, k, v = (osdpa.to_f64(t) for t in (q, k, v))
        Tq, H, d = q.shape
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        O = np.zeros((Tq, H, d))
        L = np.zeros((H, Tq)) if kind == "dead_rows_lse_zero" else np.full((H, Tq), -np.inf)
        if kind == "one_sequence":                    # sequence boundaries ignored
            cu_q, cu_k = [0, cu_q[-1]], [0, cu_k[-1]]
        for b in range(len(cu_q) - 1):
            q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
            k0, k1 = (int(cu_q[b]), int(cu_q[b + 1])) if kind == "keys_from_cu_q" else (int(cu_k[b]), int(cu_k[b + 1]))
            k1 = min(k1, k.shape[0])
            if q1 == q0 or k1 <= k0:
                continue
            qs = q[q0:q1].transpose(1, 0, 2)[None]
            ks = k[k0:k1].transpose(1, 0, 2)[None]
            vs = v[k0:k1].transpose(1, 0, 2)[None]
            if kind == "top_left_alignment" and causal and k1 - k0 > q1 - q0:
                ks, vs = ks[:, :, : q1 - q0], vs[:, :, : q1 - q0]      # queries read as the first positions
            o, lse = sdpa_forward(qs, ks, vs, causal=causal, scale=scale)
            O[q0:q1] = o[0].transpose(1, 0, 2)
            L[:, q0:q1] = lse[0]
        return O, L
    return fn


@pytest.mark.parametrize("kind", ["dead_rows_lse_zero", "one_sequence", "keys_from_cu_q", "top_left_alignment"])
def test_varlen_pins_catch_planted_mistake(kind):
    caught = 0
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(_mutant(kind))
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {kind!r}"


def test_the_mutant_without_a_mistake_passes_every_pin():
    # the mutant scaffold itself is faithful: with no mistake planted it passes all pins
    for pin in PINS:
        pin(_mutant("none"))
