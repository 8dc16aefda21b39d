"""Pins of the FP8 (e4m3) oracle (oracle/fp8.py) against things other than itself.

* the codec: every one of the 256 codes against torch's float8_e4m3fn, rounding against
  torch's conversion on random values and on every midpoint between neighbours (ties), the
  saturation the format's finite variant needs (closed forms);
* the forward on e4m3 inputs: closed forms (zero queries give the mean of the values) and the
  invariances the per-tensor scales must have;
* the P-rounding bound: a brute-force simulation of a kernel that rounds each tile's
  probabilities to e4m3 against its own, lagging reference maximum never exceeds it, and
  comes within a small factor of it (the bound is not vacuous).
"""
import math

import numpy as np
import pytest
import torch

from oracle.fp8 import (E4M3_MAX, e4m3_decode, e4m3_encode, e4m3_round, p_rounding_bound,
                        sdpa_forward_fp8)


def torch_e4m3(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_decode_closed_forms():
    assert e4m3_decode(np.uint8(0x7E)) == E4M3_MAX == 448.0
    assert e4m3_decode(np.uint8(0x01)) == 2.0 ** -9
    assert e4m3_decode(np.uint8(0x08)) == 2.0 ** -6          # smallest normal
    assert e4m3_decode(np.uint8(0x38)) == 1.0
    assert e4m3_decode(np.uint8(0xB8)) == -1.0
    assert np.isnan(e4m3_decode(np.uint8(0x7F))) and np.isnan(e4m3_decode(np.uint8(0xFF)))


def test_round_matches_torch_on_random_values():
    rng = np.random.default_rng(0)
    mags = np.exp2(rng.uniform(-12, 8.85, 20000))              # 2^8.85 < 464: torch does not overflow
    x = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32).astype(np.float64)
    assert np.array_equal(e4m3_round(x), torch_e4m3(x))


def test_round_ties_go_to_the_even_code():
    vals = e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2                            # exact in fp32
    got = e4m3_round(mids)
    assert np.array_equal(got, torch_e4m3(mids))
    codes = e4m3_encode(mids)
    assert np.all(codes % 2 == 0)


def test_round_saturates_at_448():
    x = np.array([448.0, 449.0, 463.9, 464.0, 1e9, -500.0])
    assert np.array_equal(e4m3_round(x), [448.0, 448.0, 448.0, 448.0, 448.0, -448.0])


def test_encode_decode_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = e4m3_decode(codes)
    back = e4m3_encode(vals)
    # +0 and -0 keep their codes; every other value maps back to its own code
    assert np.array_equal(back, codes)


def _codes(rng, shape, amp=1.0):
    return e4m3_encode(amp * rng.standard_normal(shape))


def test_fp8_forward_with_zero_queries_is_the_mean_of_the_values():
    rng = np.random.default_rng(1)
    q = np.zeros((1, 1, 3, 16), dtype=np.uint8)                  # code 0 = +0.0
    k = _codes(rng, (1, 1, 5, 16))
    v = _codes(rng, (1, 1, 5, 16))
    o, lse = sdpa_forward_fp8(q, k, v, 1.0, 1.0, 0.5)
    assert np.allclose(o[0, 0], np.broadcast_to(0.5 * e4m3_decode(v[0, 0]).mean(axis=0), (3, 16)), atol=1e-15)
    assert np.allclose(lse, math.log(5.0), atol=1e-15)
    # causal with 3 queries over 5 keys (bottom-right): query i sees keys 0..i+2
    o, lse = sdpa_forward_fp8(q, k, v, 1.0, 1.0, 1.0, causal=True)
    for i in range(3):
        assert np.allclose(o[0, 0, i], e4m3_decode(v[0, 0, : i + 3]).mean(axis=0), atol=1e-15)
        assert abs(lse[0, 0, i] - math.log(i + 3)) < 1e-14


def test_fp8_forward_scale_invariances():
    rng = np.random.default_rng(2)
    q, k, v = (_codes(rng, (1, 2, n, 32)) for n in (7, 9, 9))
    o1, l1 = sdpa_forward_fp8(q, k, v, 1.0, 1.0, 1.0, scale=0.2)
    # only the product of the query and key scales and the score scale matters
    o2, l2 = sdpa_forward_fp8(q, k, v, 4.0, 0.125, 1.0, scale=0.4)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)
    # the value scale multiplies O and leaves lse alone
    o3, l3 = sdpa_forward_fp8(q, k, v, 1.0, 1.0, 3.0, scale=0.2)
    assert np.allclose(o3, 3.0 * o1, atol=1e-13) and np.array_equal(l3, l1)


def _simulate_rounded_p(qc, kc, vc, sq, sk, sv, causal, scale, prescale, threshold, rng, tile=16):
    """O with P rounded to e4m3 as a tiled kernel would: per key tile, p against a reference
    maximum at or below the true one (random lag, keeping every rounded p <= 2^threshold)."""
    q = e4m3_decode(qc) * sq
    k = e4m3_decode(kc) * sk
    v = e4m3_decode(vc) * sv
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    out = np.zeros((B, H, Nq, d))
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h].T)
            if causal:
                s = np.where(np.arange(Nk)[None, :] <= np.arange(Nq)[:, None] + Nk - Nq, s, -np.inf)
            m = s.max(axis=1)
            for i in range(Nq):
                p = np.exp(s[i] - m[i])
                l = p.sum()
                pr = np.zeros_like(p)
                for t0 in range(0, Nk, tile):
                    pt = p[t0:t0 + tile]
                    top = pt.max()
                    if top == 0:
                        continue
                    # c = prescale * 2^delta, delta >= 0, and c * max(pt) <= prescale * 2^threshold
                    room = threshold - math.log2(top)
                    delta = rng.uniform(0.0, max(room, 0.0))
                    c = prescale * 2.0 ** delta
                    pr[t0:t0 + tile] = e4m3_round(c * pt) / c
                out[b, h, i] = (pr @ v[b, h]) / l
    return out


@pytest.mark.parametrize("amp,causal,prescale,threshold", [
    (1.0, False, 1.0, 8.0),
    (4.0, True, 1.0, 8.0),          # wide score spread: many subnormal p
    (4.0, False, 256.0, 0.0),       # pre-scaled P with an always-rescaling kernel
    (0.25, True, 1.0, 8.0),         # narrow spread: every p normal
])
def test_p_rounding_bound_holds_and_is_tight(amp, causal, prescale, threshold):
    rng = np.random.default_rng(3)
    worst = 0.0
    for rep in range(4):
        qc = _codes(rng, (1, 1, 24, 32), amp)
        kc = _codes(rng, (1, 1, 40, 32), amp)
        vc = _codes(rng, (1, 1, 40, 32))
        sq, sk, sv, scale = 0.5, 2.0, 1.5, 1 / math.sqrt(32)
        exact, _ = sdpa_forward_fp8(qc, kc, vc, sq, sk, sv, causal=causal, scale=scale)
        bound = p_rounding_bound(qc, kc, vc, sq, sk, sv, causal=causal, scale=scale, p_prescale=prescale,
                                 threshold_log2=threshold)
        for _ in range(3):
            got = _simulate_rounded_p(qc, kc, vc, sq, sk, sv, causal, scale, prescale, threshold, rng)
            err = np.abs(got - exact)
            assert np.all(err <= bound + 1e-12), float((err - bound).max())
            worst = max(worst, float((err / np.maximum(bound, 1e-300)).max()))
    assert worst > 0.4, worst      # rounding reaches a good part of the bound: it is not loose


def test_bound_rejects_a_saturating_configuration():
    rng = np.random.default_rng(4)
    qc, kc, vc = (_codes(rng, (1, 1, 4, 16)) for _ in range(3))
    with pytest.raises(AssertionError):
        p_rounding_bound(qc, kc, vc, 1.0, 1.0, 1.0, p_prescale=256.0, threshold_log2=8.0)


def _codec_mutant(kind):
    """e4m3_decode / e4m3_round with one plausible mistake."""
    import oracle.fp8 as f8
    real_decode, real_round = f8.e4m3_decode, f8.e4m3_round

    def decode(codes):
        c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
        out = real_decode(codes)
        if kind == "exponent_bias_8":
            out = out / 2.0
        if kind == "subnormal_scale":
            sub = ((c >> 3) & 0xF) == 0
            out = np.where(sub, out * 2.0, out)
        if kind == "no_nan":
            out = np.where(np.isnan(out), np.copysign(480.0, np.where(c & 0x80, -1.0, 1.0)), out)
        return out

    def rnd(x):
        r = real_round(x)
        if kind == "ties_away":
            vals = real_decode(np.arange(0x7F, dtype=np.uint8))
            a = np.abs(np.asarray(x, dtype=np.float64))
            mids = (vals[:-1] + vals[1:]) / 2
            hit = np.isin(a, mids)
            up = vals[np.clip(np.searchsorted(vals, a), 0, len(vals) - 1)]
            r = np.where(hit, np.copysign(up, x), r)
        if kind == "no_saturation":
            r = np.where(np.abs(np.asarray(x)) > E4M3_MAX, np.nan, r)
        return r
    return decode, rnd


CODEC_PINS = [test_decode_matches_torch_on_every_code, test_decode_closed_forms, test_round_matches_torch_on_random_values,
              test_round_ties_go_to_the_even_code, test_round_saturates_at_448]


@pytest.mark.parametrize("kind", ["exponent_bias_8", "subnormal_scale", "no_nan", "ties_away", "no_saturation"])
def test_codec_pins_catch_planted_mistake(kind, monkeypatch):
    decode, rnd = _codec_mutant(kind)
    monkeypatch.setitem(globals(), "e4m3_decode", decode)
    monkeypatch.setitem(globals(), "e4m3_round", rnd)
    caught = 0
    for pin in CODEC_PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {kind!r}"
