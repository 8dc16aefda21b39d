"""Pins for the fp64 oracle: values the pages print, closed forms, invariants,
a library routine and brute force on tiny inputs.

Each pin is a function of the oracle under test, so that the mutation test at
the end can run every pin against deliberately broken copies of the oracle
(planted on the CPU) and show that each plausible mistake is caught.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.sdpa as osdpa
from oracle import sdpa_forward, sdpa_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")
RNG = np.random.default_rng


def _rand(shape, seed, scale=1.0):
    return RNG(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------------------
# pins, each written against an oracle ``fwd`` with sdpa_forward's signature
# ---------------------------------------------------------------------------

def pin_hand_2x2(fwd):
    g = json.load(open(GOLDEN))["hand_softmax_2x2"]
    q = np.array(g["q"])[None, None]
    k = np.array(g["k"])[None, None]
    v = np.array(g["v"])[None, None]
    o, lse = fwd(q, k, v, scale=g["scale"])
    np.testing.assert_allclose(o[0, 0], g["o"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], g["lse"], rtol=0, atol=1e-15)


def pin_hand_causal(fwd):
    g = json.load(open(GOLDEN))["hand_causal_3x1"]
    v = np.array(g["v"])[None, None]
    q = _rand((1, 1, 3, 1), 1)
    k = _rand((1, 1, 3, 1), 2)
    o, lse = fwd(q, k, v, causal=True, scale=0.0)
    np.testing.assert_allclose(o[0, 0], g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], g["lse"], rtol=0, atol=1e-14)


def pin_rows_sum_to_one(fwd):
    # V = identity makes O the weight matrix itself: every row must sum to 1
    for causal in (False, True):
        n = 9
        q = _rand((2, 2, n, n), 3)
        k = _rand((2, 2, n, n), 4)
        v = np.broadcast_to(np.eye(n), (2, 2, n, n)).copy()
        bias = _rand((2, n, n), 5)
        o, _ = fwd(q, k, v, bias=bias, causal=causal, scale=0.7)
        np.testing.assert_allclose(o.sum(-1), 1.0, rtol=0, atol=1e-14)
        assert (o >= 0).all()
        if causal:
            assert np.all(np.triu(o, 1) == 0.0)    # weight of any key j > i is exactly zero


def pin_identical_v_rows(fwd):
    u = _rand((7,), 6)
    v = np.broadcast_to(u, (1, 3, 33, 7)).copy()
    q = _rand((1, 3, 33, 7), 7, 3.0)
    k = _rand((1, 3, 33, 7), 8, 3.0)
    for causal in (False, True):
        o, _ = fwd(q, k, v, causal=causal)
        np.testing.assert_allclose(o, np.broadcast_to(u, o.shape), rtol=0, atol=1e-13)


def pin_dominant_key(fwd):
    n, d = 20, 5
    q = _rand((1, 1, n, d), 9)
    k = _rand((1, 1, n, d), 10)
    v = _rand((1, 1, n, d), 11)
    jstar = 13
    bias = np.zeros((1, n, n))
    bias[0, :, jstar] = 1.0e4
    scale = 0.5
    o, lse = fwd(q, k, v, bias=bias, scale=scale)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0, jstar], (n, d)), rtol=0, atol=1e-12)
    s_star = scale * q[0, 0] @ k[0, 0, jstar] + 1.0e4
    np.testing.assert_allclose(lse[0, 0], s_star, rtol=1e-15, atol=1e-9)


def pin_causal_row0(fwd):
    q = _rand((2, 3, 17, 8), 12)
    k = _rand((2, 3, 17, 8), 13)
    v = _rand((2, 3, 17, 8), 14)
    scale = 0.3
    o, lse = fwd(q, k, v, causal=True, scale=scale)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=0, atol=1e-15)
    s00 = scale * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], s00, rtol=0, atol=1e-14)


def pin_scale_zero_closed_form(fwd):
    n = 11
    q = _rand((1, 2, n, 4), 15)
    k = _rand((1, 2, n, 4), 16)
    v = _rand((1, 2, n, 4), 17)
    o, lse = fwd(q, k, v, scale=0.0)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(n), atol=1e-14)
    o, lse = fwd(q, k, v, causal=True, scale=0.0)
    cmean = np.cumsum(v, axis=2) / np.arange(1, n + 1)[None, None, :, None]
    np.testing.assert_allclose(o, cmean, atol=1e-14)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(np.arange(1, n + 1)), lse.shape), atol=1e-14)


def pin_bias_shift(fwd):
    n = 12
    q = _rand((2, 2, n, 6), 18)
    k = _rand((2, 2, n, 6), 19)
    v = _rand((2, 2, n, 6), 20)
    bias = _rand((2, n, n), 21)
    c = _rand((2, n, 1), 22, 5.0)                   # a per-(h, row) constant
    o1, l1 = fwd(q, k, v, bias=bias, scale=0.4)
    o2, l2 = fwd(q, k, v, bias=bias + c, scale=0.4)
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + c[None, :, :, 0], atol=1e-12)


def pin_key_permutation(fwd):
    n = 14
    q = _rand((1, 2, n, 5), 23)
    k = _rand((1, 2, n, 5), 24)
    v = _rand((1, 2, n, 5), 25)
    perm = RNG(26).permutation(n)
    o1, l1 = fwd(q, k, v)
    o2, l2 = fwd(q, k[:, :, perm], v[:, :, perm])
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_allclose(l2, l1, atol=1e-13)


def pin_gate(fwd):
    q = _rand((1, 1, 6, 3), 27)
    k = _rand((1, 1, 6, 3), 28)
    v = _rand((1, 1, 6, 3), 29)
    o0, l0 = fwd(q, k, v)
    o_half, l_half = fwd(q, k, v, gate=np.zeros_like(q))       # sigmoid(0) = 1/2
    np.testing.assert_allclose(o_half, 0.5 * o0, atol=1e-15)
    np.testing.assert_allclose(l_half, l0, atol=0)              # the gate does not enter lse
    g = _rand(q.shape, 30)
    o_g, _ = fwd(q, k, v, gate=g)
    np.testing.assert_allclose(o_g, o0 * np.exp(g) / (1.0 + np.exp(g)), atol=1e-14)


def _brute_force(q, k, v, bias, gate, causal, scale):
    """Per-element pure-Python loops, no BLAS, written from Equation (1)."""
    B, H, N, d = q.shape
    O = np.zeros(q.shape)
    L = np.zeros(q.shape[:3])
    for b in range(B):
        for h in range(H):
            for i in range(N):
                scores = []
                for j in range(k.shape[2]):
                    if causal and j > i:
                        continue
                    s = 0.0
                    for t in range(d):
                        s += float(q[b, h, i, t]) * float(k[b, h, j, t])
                    s *= scale
                    if bias is not None:
                        s += float(bias[h, i, j])
                    scores.append((j, s))
                mx = max(s for _, s in scores)
                den = sum(math.exp(s - mx) for _, s in scores)
                for t in range(d):
                    acc = sum(math.exp(s - mx) * float(v[b, h, j, t]) for j, s in scores)
                    val = acc / den
                    if gate is not None:
                        val *= 1.0 / (1.0 + math.exp(-float(gate[b, h, i, t])))
                    O[b, h, i, t] = val
                L[b, h, i] = mx + math.log(den)
    return O, L


def pin_brute_force(fwd):
    for causal, with_bias, with_gate, n in [(False, False, False, 5), (True, False, False, 16),
                                            (False, True, True, 9), (True, True, False, 13)]:
        q = _rand((1, 2, n, 4), 31 + n)
        k = _rand((1, 2, n, 4), 32 + n)
        v = _rand((1, 2, n, 4), 33 + n)
        bias = _rand((2, n, n), 34 + n) if with_bias else None
        gate = _rand((1, 2, n, 4), 35 + n) if with_gate else None
        o, lse = fwd(q, k, v, bias=bias, gate=gate, causal=causal, scale=0.45)
        ob, lb = _brute_force(q, k, v, bias, gate, causal, 0.45)
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-13)


def pin_torch_sdpa(fwd):
    # an independent library implementation of the same definition, in float64 on the CPU
    for causal, with_bias in [(False, False), (True, False), (False, True)]:
        q = _rand((2, 3, 40, 16), 40)
        k = _rand((2, 3, 40, 16), 41)
        v = _rand((2, 3, 40, 16), 42)
        bias = _rand((3, 40, 40), 43) if with_bias else None
        o, _ = fwd(q, k, v, bias=bias, causal=causal, scale=0.25)
        t = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
            attn_mask=None if bias is None else torch.from_numpy(bias)[None],
            is_causal=causal, scale=0.25)
        np.testing.assert_allclose(o, t.numpy(), rtol=0, atol=1e-12)


def _online_softmax_attention(q, k, v, causal, scale, block):
    """A second, independent fp64 routine: the single-pass online softmax of the
    gist.science FLASHLIGHT summary (Methodology, item 3): a running max and a
    running sum, the sum rescaled by e^(m_old - m_new) when the max grows,
    walked over keys ``block`` at a time."""
    B, H, N, d = q.shape
    O = np.zeros(q.shape)
    L = np.zeros(q.shape[:3])
    for b in range(B):
        for h in range(H):
            for i in range(N):
                m, l, acc = -np.inf, 0.0, np.zeros(d)
                last = i if causal else k.shape[2] - 1
                for j0 in range(0, last + 1, block):
                    js = list(range(j0, min(last + 1, j0 + block)))
                    s = np.array([scale * float(np.dot(q[b, h, i], k[b, h, j])) for j in js])
                    m_new = max(m, s.max())
                    alpha = math.exp(m - m_new) if np.isfinite(m) else 0.0
                    p = np.exp(s - m_new)
                    l = alpha * l + p.sum()
                    acc = alpha * acc + p @ v[b, h, js]
                    m = m_new
                O[b, h, i] = acc / l
                L[b, h, i] = m + math.log(l)
    return O, L


def pin_online_equals_two_pass(fwd):
    q = _rand((1, 2, 10, 6), 50, 2.0)
    k = _rand((1, 2, 10, 6), 51, 2.0)
    v = _rand((1, 2, 10, 6), 52)
    for causal in (False, True):
        o, lse = fwd(q, k, v, causal=causal, scale=0.6)
        for block in (1, 3):
            oo, lo = _online_softmax_attention(q, k, v, causal, 0.6, block)
            np.testing.assert_allclose(o, oo, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse, lo, rtol=0, atol=1e-12)


def pin_large_scores_stable(fwd):
    # scores near 1e3 overflow exp() unless the row max is subtracted first
    q = _rand((1, 1, 8, 4), 60, 30.0)
    k = _rand((1, 1, 8, 4), 61, 30.0)
    v = _rand((1, 1, 8, 4), 62)
    o, lse = fwd(q, k, v, scale=1.0)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    ob, lb = _brute_force(q, k, v, None, None, False, 1.0)
    np.testing.assert_allclose(o, ob, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=1e-14)


def pin_causal_suffix_alignment(fwd):
    # fewer queries than keys: the queries are the last Nq positions, so their rows must equal
    # the last Nq rows of the square causal problem over the same keys (bottom-right alignment)
    n, nq = 12, 5
    q = _rand((2, 2, n, 6), 100)
    k = _rand((2, 2, n, 6), 101)
    v = _rand((2, 2, n, 6), 102)
    bias = _rand((2, n, n), 103)
    o_sq, l_sq = fwd(q, k, v, bias=bias, causal=True, scale=0.45)
    o, lse = fwd(q[:, :, n - nq:], k, v, bias=bias[:, n - nq:], causal=True, scale=0.45)
    np.testing.assert_allclose(o, o_sq[:, :, n - nq:], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, l_sq[:, :, n - nq:], rtol=0, atol=1e-14)


def pin_decode_single_query(fwd):
    # one query after all the keys sees every key: causal or not makes no difference
    q = _rand((1, 3, 1, 8), 104)
    k = _rand((1, 3, 9, 8), 105)
    v = _rand((1, 3, 9, 8), 106)
    o_c, l_c = fwd(q, k, v, causal=True, scale=0.3)
    o_n, l_n = fwd(q, k, v, causal=False, scale=0.3)
    np.testing.assert_allclose(o_c, o_n, rtol=0, atol=0)
    np.testing.assert_allclose(l_c, l_n, rtol=0, atol=0)
    ob, lb = _brute_force(q, k, v, None, None, False, 0.3)
    np.testing.assert_allclose(o_c, ob, atol=1e-14)


def pin_more_queries_than_keys(fwd):
    # Nq > Nk, causal: the first Nq - Nk queries precede every key (dead rows: O = 0,
    # lse = -inf); the others are the square problem on the last Nk queries
    q = _rand((1, 2, 7, 4), 107)
    k = _rand((1, 2, 4, 4), 108)
    v = _rand((1, 2, 4, 4), 109)
    o, lse = fwd(q, k, v, causal=True, scale=0.8)
    assert np.all(o[:, :, :3] == 0.0) and np.all(lse[:, :, :3] == -np.inf)
    o_sq, l_sq = fwd(q[:, :, 3:], k, v, causal=True, scale=0.8)
    np.testing.assert_allclose(o[:, :, 3:], o_sq, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 3:], l_sq, rtol=0, atol=1e-15)
    ob, lb = _brute_force(q[:, :, 3:], k, v, None, None, True, 0.8)
    np.testing.assert_allclose(o_sq, ob, atol=1e-14)


PINS = [pin_hand_2x2, pin_hand_causal, pin_rows_sum_to_one, pin_identical_v_rows, pin_dominant_key,
        pin_causal_row0, pin_scale_zero_closed_form, pin_bias_shift, pin_key_permutation, pin_gate,
        pin_brute_force, pin_torch_sdpa, pin_online_equals_two_pass, pin_large_scores_stable,
        pin_causal_suffix_alignment, pin_decode_single_query, pin_more_queries_than_keys]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(sdpa_forward)


# ---------------------------------------------------------------------------
# other oracle properties
# ---------------------------------------------------------------------------

def test_worked_sizing_closed_form():
    g = json.load(open(GOLDEN))["naive_weights_bytes"]
    b = g["bytes_per_element"] * g["B"] * g["h"] * g["n"] * g["n"]
    assert b == g["bytes"] == 6_442_450_944
    assert round(b / 1e9, 2) == g["printed_gb_one_layer"]
    assert round(b * g["layers"] / 1e9) == g["printed_gb_32_layers"]


def test_output_shape_contract():
    g = json.load(open(GOLDEN))["output_shape"]
    small = [2, 3, 16, 8]   # same rule on a small case: out shape == Q shape
    q = _rand(small, 70)
    o, lse = sdpa_forward(q, _rand(small, 71), _rand(small, 72), causal=True)
    assert list(o.shape) == small and list(lse.shape) == small[:3]
    assert g["out_shape"] == g["q_shape"]


def test_fully_masked_row_convention():
    q = _rand((1, 1, 4, 3), 80)
    k = _rand((1, 1, 4, 3), 81)
    v = _rand((1, 1, 4, 3), 82)
    bias = np.zeros((1, 4, 4))
    bias[0, 2, :] = -np.inf
    o, lse = sdpa_forward(q, k, v, bias=bias)
    assert np.all(o[0, 0, 2] == 0.0) and lse[0, 0, 2] == -np.inf
    assert np.isfinite(o[0, 0, [0, 1, 3]]).all()


def test_rows_match_forward():
    q = _rand((2, 2, 300, 16), 90)
    k = _rand((2, 2, 300, 16), 91)
    v = _rand((2, 2, 300, 16), 92)
    bias = _rand((2, 300, 300), 93)
    gate = _rand((2, 2, 300, 16), 94)
    for causal in (False, True):
        o, lse = sdpa_forward(q, k, v, bias=bias, gate=gate, causal=causal, block_rows=128)
        picks = [(0, 0, 0), (1, 1, 299), (0, 1, 128), (1, 0, 77), (1, 1, 0)]
        ro, rl = sdpa_rows(q, k, v, picks, bias=bias, gate=gate, causal=causal)
        for n, (b, h, i) in enumerate(picks):
            np.testing.assert_allclose(ro[n], o[b, h, i], atol=1e-14)
            np.testing.assert_allclose(rl[n], lse[b, h, i], atol=1e-14)


def test_exact_upcast_of_half_inputs():
    t = torch.randn(3, 5, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    a = osdpa.to_f64(t)
    assert a.dtype == np.float64
    assert np.array_equal(a, t.double().numpy())


# ---------------------------------------------------------------------------
# mutation test: plausible mistakes planted in copies of the oracle are caught
# ---------------------------------------------------------------------------

def _mutant(kind):
    real = osdpa._attend_rows

    def attend(qr, k, v, bias_r, gate_r, rows, causal, scale, offset=0, mods=None):
        if kind == "no_scale":
            scale = 1.0
        if kind == "bias_sign" and bias_r is not None:
            bias_r = -bias_r
        if kind == "causal_off_by_one" and causal:
            # reveal key i+1 as well (j <= i+1 instead of j <= i)
            keys = np.arange(k.shape[0])
            s = scale * (qr @ k.T) + (0 if bias_r is None else bias_r)
            s = np.where(keys[None, :] > rows[:, None] + offset + 1, -np.inf, s)
            m = s.max(1)
            w = np.exp(s - m[:, None])
            o = (w @ v) / w.sum(1)[:, None]
            if gate_r is not None:
                o = o / (1 + np.exp(-gate_r))
            return o, m + np.log(w.sum(1))
        if kind == "k_for_v":
            v = k
        if kind == "no_max_shift":
            s = scale * (qr @ k.T) + (0 if bias_r is None else bias_r)
            if causal:
                keys = np.arange(k.shape[0])
                s = np.where(keys[None, :] > rows[:, None] + offset, -np.inf, s)
            with np.errstate(over="ignore", invalid="ignore"):
                w = np.exp(s)
                o = (w @ v) / w.sum(1)[:, None]
                lse = np.log(w.sum(1))
            if gate_r is not None:
                o = o / (1 + np.exp(-gate_r))
            return o, lse
        if kind == "lse_log2":
            o, lse = real(qr, k, v, bias_r, gate_r, rows, causal, scale, offset, mods)
            return o, lse / math.log(2.0)
        if kind == "gate_not_sigmoid" and gate_r is not None:
            o, lse = real(qr, k, v, bias_r, None, rows, causal, scale, offset, mods)
            return o * gate_r, lse
        if kind == "transposed_q":
            qr = qr[::-1]
        if kind == "top_left_alignment":
            offset = 0
        return real(qr, k, v, bias_r, gate_r, rows, causal, scale, offset, mods)

    return attend


@pytest.mark.parametrize("kind", ["no_scale", "bias_sign", "causal_off_by_one", "k_for_v",
                                  "no_max_shift", "lse_log2", "gate_not_sigmoid", "transposed_q",
                                  "top_left_alignment"])
def test_pins_catch_planted_mistake(kind, monkeypatch):
    monkeypatch.setattr(osdpa, "_attend_rows", _mutant(kind))
    caught = 0
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(osdpa.sdpa_forward)
        except (AssertionError, FloatingPointError, ValueError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {kind!r}"
