"""fp64 oracle for the FP8 (e4m3) forward: the e4m3 codec, the forward on e4m3 inputs with
per-tensor scales, and the error bound that rounding P to e4m3 allows.

TEST INFRASTRUCTURE ONLY (the same rule as oracle/sdpa.py: only the test suite, smoke() and
bench.py's oracle legs may import it; it shares no code with the CUDA path).

What the pages fix: hamidun.com's FlashAttention-3 article (the low-precision section) runs
the attention in FP8 for about twice the FP16 throughput and states that its error stays
close to that of plain FP8 attention.  It gives no format, scaling or accumulation rule.
Readings taken here (each the plainest one the rest supports):

* the 8-bit format is e4m3 in its finite variant: 1 sign bit, 4 exponent bits (bias 7), 3
  mantissa bits, subnormals, no infinities, the two all-ones codes are NaN, largest finite
  value 448;
* Q, K and V arrive as e4m3 codes with one fp32 scale per tensor: the value of element x is
  decode(x) * scale_x;
* the attention itself is exact (the fused method is exact, oracle/sdpa.py): O and lse are
  those of the plain forward on the decoded, scaled values, in fp64;
* the only rounding the method adds is P's: a kernel that multiplies P by V on the FP8 tensor
  core rounds each p to e4m3 (round to nearest even, saturating at 448) after multiplying it
  by a power-of-two pre-scale, and divides the pre-scale back out of the accumulator; the
  row sum l is taken over the unrounded p.  ``p_rounding_bound`` gives, per output element,
  the largest difference that rounding can make, whatever the reference maximum each key
  tile was exponentiated against (the online softmax's running maximum, at or below the true
  row maximum; the kernel keeps every p it rounds at most 2^threshold, threshold being its
  rescale threshold in log2 units).

e4m3 values: code c = s eeee mmm; e = 0 gives (m / 8) * 2^-6 (subnormal), e > 0 gives
(1 + m / 8) * 2^(e - 7); c & 0x7f == 0x7f is NaN.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .sdpa import sdpa_forward

E4M3_MAX = 448.0
E4M3_MIN_SUBNORMAL = 2.0 ** -9


def e4m3_decode(codes) -> np.ndarray:
    """float64 value of each e4m3 code (uint8 array); NaN for the two NaN codes."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    out = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


def _positive_values() -> np.ndarray:
    """The 127 finite non-negative e4m3 values in increasing order (codes 0x00..0x7e)."""
    return e4m3_decode(np.arange(0x7F, dtype=np.uint8))


def e4m3_round(x) -> np.ndarray:
    """x rounded to the nearest e4m3 value, ties to the even code, magnitudes above 448 to 448."""
    x = np.asarray(x, dtype=np.float64)
    vals = _positive_values()
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, len(vals) - 1)   # first value >= a
    lo = np.maximum(hi - 1, 0)
    v_hi, v_lo = vals[hi], vals[lo]
    exact = v_hi == a
    d_lo, d_hi = a - v_lo, v_hi - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))      # even code on a tie
    r = np.where(exact, a, np.where(pick_hi, v_hi, v_lo))
    return np.copysign(r, x)


def e4m3_encode(x) -> np.ndarray:
    """uint8 code of e4m3_round(x) (the code with the same sign as x)."""
    r = e4m3_round(x)
    vals = _positive_values()
    idx = np.searchsorted(vals, np.abs(r), side="left").astype(np.uint8)
    return np.where(np.signbit(r), idx | np.uint8(0x80), idx).astype(np.uint8)


def sdpa_forward_fp8(q_codes, k_codes, v_codes, q_scale: float, k_scale: float, v_scale: float,
                     causal: bool = False, scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """(O, lse) in fp64 of the exact forward on the decoded, per-tensor scaled e4m3 inputs."""
    q = e4m3_decode(q_codes) * float(q_scale)
    k = e4m3_decode(k_codes) * float(k_scale)
    v = e4m3_decode(v_codes) * float(v_scale)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    return sdpa_forward(q, k, v, causal=causal, scale=scale)


def p_rounding_bound(q_codes, k_codes, v_codes, q_scale: float, k_scale: float, v_scale: float,
                     causal: bool = False, scale: Optional[float] = None, p_prescale: float = 1.0,
                     threshold_log2: float = 8.0) -> np.ndarray:
    """Per output element [B, H, Nq, d], an upper bound on |O_P-rounded - O_exact|.

    With p_ij = exp(s_ij - m_i) (m_i the true row maximum, 0 < p <= 1) a kernel rounds
    c * p_ij to e4m3, where c = p_prescale * 2^delta and delta >= 0 is how far the reference
    maximum of key j's tile lies below m_i (in log2 units).  A normal result is off by at most
    2^-4 of c * p, a subnormal one (below 2^-6) by at most half the subnormal step, 2^-10;
    after dividing c back out the error in p_ij is at most max(2^-4 p_ij, 2^-10 / p_prescale)
    (c >= p_prescale).  With l_i the sum of the unrounded p:
        |dO_ic| <= sum_j max(2^-4 p_ij, 2^-10 / p_prescale) |v_jc| / l_i.
    No value saturates as long as p_prescale * 2^threshold_log2 <= 448 (each rounded value is
    at most that).
    """
    q = e4m3_decode(q_codes) * float(q_scale)
    k = e4m3_decode(k_codes) * float(k_scale)
    v = e4m3_decode(v_codes) * float(v_scale)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    assert p_prescale * 2.0 ** threshold_log2 <= E4M3_MAX, "rounded values would saturate"
    off = Nk - Nq
    out = np.zeros((B, H, Nq, d))
    keys = np.arange(Nk)
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h].T)
            if causal:
                s = np.where(keys[None, :] <= np.arange(Nq)[:, None] + off, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            err = np.where(p > 0, np.maximum(2.0 ** -4 * p, 2.0 ** -10 / p_prescale), 0.0)
            out[b, h] = (err @ np.abs(v[b, h])) / np.where(l > 0, l, 1.0)
    return out
