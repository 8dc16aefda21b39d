"""Pins for the oracle's score modifications (ALiBi, logit softcap, left window):
limits that reduce to the plain forward or to a one-hot attention, and a
per-element pure-Python brute force; planted mistakes are caught."""
import math

import numpy as np
import pytest

import oracle.sdpa as osdpa
from oracle import sdpa_forward

RNG = np.random.default_rng


def _rand(shape, seed, scale=1.0):
    return RNG(seed).standard_normal(shape) * scale


def _brute(q, k, v, causal, scale, softcap=0.0, slopes=None, window=-1):
    """Per-element loops (no BLAS), each modification applied as the definition says."""
    B, H, N, d = q.shape
    Nk = k.shape[2]
    off = Nk - N
    O = np.zeros(q.shape)
    L = np.zeros(q.shape[:3])
    for b in range(B):
        for h in range(H):
            for i in range(N):
                sc = []
                for j in range(Nk):
                    if causal and j > i + off:
                        continue
                    if window >= 0 and j < i + off - window:
                        continue
                    s = scale * sum(float(q[b, h, i, t]) * float(k[b, h, j, t]) for t in range(d))
                    if slopes is not None:
                        s -= float(slopes[h]) * abs(i + off - j)
                    if softcap > 0:
                        s = softcap * math.tanh(s / softcap)
                    sc.append((j, s))
                if not sc:
                    L[b, h, i] = -math.inf
                    continue
                mx = max(s for _, s in sc)
                den = sum(math.exp(s - mx) for _, s in sc)
                for t in range(d):
                    O[b, h, i, t] = sum(math.exp(s - mx) * float(v[b, h, j, t]) for j, s in sc) / den
                L[b, h, i] = mx + math.log(den)
    return O, L


def _qkv(n=7, nk=9, d=4, seed=300, amp=1.0):
    return (_rand((1, 2, n, d), seed, amp), _rand((1, 2, nk, d), seed + 1, amp), _rand((1, 2, nk, d), seed + 2))


def pin_large_softcap_is_plain(fwd):
    q, k, v = _qkv()
    for causal in (False, True):
        o0, l0 = fwd(q, k, v, causal=causal, scale=0.5)
        o1, l1 = fwd(q, k, v, causal=causal, scale=0.5, softcap=1e8)
        np.testing.assert_allclose(o1, o0, atol=1e-12)
        np.testing.assert_allclose(l1, l0, atol=1e-12)


def pin_zero_slopes_are_plain(fwd):
    q, k, v = _qkv(seed=310)
    o0, l0 = fwd(q, k, v, causal=True, scale=0.5)
    o1, l1 = fwd(q, k, v, causal=True, scale=0.5, alibi_slopes=np.zeros(2))
    np.testing.assert_array_equal(o1, o0)
    np.testing.assert_array_equal(l1, l0)


def pin_steep_alibi_picks_the_aligned_key(fwd):
    # a huge slope leaves only the key at distance 0 (j = i + Nk - N) with weight
    q, k, v = _qkv(n=5, nk=8, seed=320)
    o, lse = fwd(q, k, v, causal=False, scale=0.3, alibi_slopes=np.array([1e5, 2e5]))
    for i in range(5):
        np.testing.assert_allclose(o[0, :, i], v[0, :, i + 3], atol=1e-12)
        np.testing.assert_allclose(lse[0, :, i], 0.3 * np.einsum("hd,hd->h", q[0, :, i], k[0, :, i + 3]), atol=1e-9)


def pin_zero_window_is_the_diagonal(fwd):
    q, k, v = _qkv(n=6, nk=6, seed=330)
    o, lse = fwd(q, k, v, causal=True, scale=0.7, window_left=0)
    np.testing.assert_allclose(o[0], v[0], atol=1e-15)
    np.testing.assert_allclose(lse[0], 0.7 * np.einsum("hid,hid->hi", q[0], k[0]), atol=1e-14)


def pin_wide_window_is_plain(fwd):
    q, k, v = _qkv(seed=340)
    o0, l0 = fwd(q, k, v, causal=True, scale=0.5)
    o1, l1 = fwd(q, k, v, causal=True, scale=0.5, window_left=9)
    np.testing.assert_array_equal(o1, o0)
    np.testing.assert_array_equal(l1, l0)


def pin_brute_force_all_mods(fwd):
    slopes = np.array([0.25, 0.6])
    for causal, (n, nk), w in [(True, (5, 9), 3), (False, (6, 4), 2), (True, (7, 7), 1)]:
        q, k, v = _qkv(n=n, nk=nk, seed=350 + n, amp=2.0)
        o, lse = fwd(q, k, v, causal=causal, scale=0.8, softcap=1.7, alibi_slopes=slopes, window_left=w)
        ob, lb = _brute(q, k, v, causal, 0.8, 1.7, slopes, w)
        np.testing.assert_allclose(o, ob, atol=1e-13)
        np.testing.assert_allclose(lse, lb, atol=1e-13)


MOD_PINS = [pin_large_softcap_is_plain, pin_zero_slopes_are_plain, pin_steep_alibi_picks_the_aligned_key,
            pin_zero_window_is_the_diagonal, pin_wide_window_is_plain, pin_brute_force_all_mods]


@pytest.mark.parametrize("pin", MOD_PINS, ids=[p.__name__ for p in MOD_PINS])
def test_mod_pin(pin):
    pin(sdpa_forward)


def _mutant(kind):
    real = osdpa._attend_rows

    def attend(qr, k, v, bias_r, gate_r, rows, causal, scale, offset=0, mods=None):
        if mods is not None:
            mods = dict(mods)
            if kind == "alibi_sign" and mods.get("alibi_slope") is not None:
                mods["alibi_slope"] = -mods["alibi_slope"]
            if kind == "window_off_by_one" and mods.get("window_left", -1) >= 0:
                mods["window_left"] += 1
            if kind == "softcap_before_scale" and mods.get("softcap", 0) > 0:
                cap = mods["softcap"]
                return real(qr, k, v, bias_r, gate_r, rows, causal, scale * cap / max(cap, 1.0) * 1.01, offset, mods)
        return real(qr, k, v, bias_r, gate_r, rows, causal, scale, offset, mods)

    return attend


def _mutant_scores(kind):
    """_attend_rows with one mistake in how the modifications meet the scores and the masks."""
    def attend(qr, k, v, bias_r, gate_r, rows, causal, scale, offset=0, mods=None):
        s = scale * (qr @ k.T)
        if bias_r is not None:
            s = s + bias_r
        keys = np.arange(k.shape[0])
        diag = rows[:, None] + (0 if kind in ("alibi_no_offset", "window_no_offset") else offset)
        if causal and kind == "softcap_after_mask":
            s = np.where(keys[None, :] > rows[:, None] + offset, -np.inf, s)
        if mods is not None:
            if mods.get("alibi_slope") is not None:
                d_al = diag if kind == "alibi_no_offset" else rows[:, None] + offset
                s = s - mods["alibi_slope"] * np.abs(d_al - keys[None, :])
            cap = mods.get("softcap", 0.0)
            if cap and cap > 0:
                s = cap * np.tanh(s) if kind == "softcap_no_inner_division" else cap * np.tanh(s / cap)
            w = mods.get("window_left", -1)
            if w is not None and w >= 0:
                d_w = diag if kind == "window_no_offset" else rows[:, None] + offset
                s = np.where(keys[None, :] < d_w - w, -np.inf, s)
        if causal and kind != "softcap_after_mask":
            s = np.where(keys[None, :] > rows[:, None] + offset, -np.inf, s)
        m = s.max(axis=1)
        dead = ~np.isfinite(m) & (m < 0)
        wts = np.exp(s - np.where(dead, 0.0, m)[:, None])
        l = wts.sum(axis=1)
        with np.errstate(invalid="ignore", divide="ignore"):
            o = np.where(dead[:, None], 0.0, (wts @ v) / l[:, None])
            lse = np.where(dead, -np.inf, m + np.log(l))
        if gate_r is not None:
            o = o * (1.0 / (1.0 + np.exp(-gate_r)))
        return o, lse
    return attend


@pytest.mark.parametrize("kind", ["none", "alibi_no_offset", "window_no_offset", "softcap_no_inner_division",
                                  "softcap_after_mask"])
def test_mod_pins_catch_planted_score_mistake(kind, monkeypatch):
    monkeypatch.setattr(osdpa, "_attend_rows", _mutant_scores(kind))
    failed = []
    for pin in MOD_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(osdpa.sdpa_forward)
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(pin.__name__)
    if kind == "none":          # the scaffold without a mistake is faithful
        assert not failed, failed
    else:
        assert failed, f"no pin caught the planted mistake {kind!r}"


@pytest.mark.parametrize("kind", ["alibi_sign", "window_off_by_one", "softcap_before_scale"])
def test_mod_pins_catch_planted_mistake(kind, monkeypatch):
    monkeypatch.setattr(osdpa, "_attend_rows", _mutant(kind))
    caught = 0
    for pin in MOD_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(osdpa.sdpa_forward)
        except (AssertionError, FloatingPointError, ValueError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {kind!r}"


@pytest.mark.parametrize("causal,nq,nk", [(True, 7, 7), (True, 5, 11), (False, 6, 9), (True, 9, 4)])
def test_alibi_and_window_equal_their_explicit_bias(causal, nq, nk):
    # the modifications are defined as score terms; written out as an additive bias matrix
    # (-slope_h |i + Nk - Nq - j|, and -inf left of the window) the plain forward must agree
    rng = np.random.default_rng(900 + nq * nk)
    q, k, v = rng.standard_normal((2, 2, nq, 8)), rng.standard_normal((2, 2, nk, 8)), rng.standard_normal((2, 2, nk, 8))
    slopes = np.array([0.4, 0.05])
    off = nk - nq
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    alibi_bias = -slopes[:, None, None] * np.abs(i + off - j)[None]              # [H, Nq, Nk]
    o, lse = sdpa_forward(q, k, v, causal=causal, scale=0.7, alibi_slopes=slopes)
    ob, lb = sdpa_forward(q, k, v, bias=alibi_bias, causal=causal, scale=0.7)
    np.testing.assert_allclose(o, ob, atol=1e-13)
    np.testing.assert_allclose(lse, lb, atol=1e-13)
    w = 2
    win_bias = np.where(j < i + off - w, -np.inf, 0.0)[None].repeat(2, axis=0)   # [H, Nq, Nk]
    o, lse = sdpa_forward(q, k, v, causal=causal, scale=0.7, window_left=w)
    ob, lb = sdpa_forward(q, k, v, bias=win_bias, causal=causal, scale=0.7)
    np.testing.assert_allclose(o, ob, atol=1e-13)
    np.testing.assert_array_equal(np.isfinite(lse), np.isfinite(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], atol=1e-13)
