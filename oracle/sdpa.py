"""fp64 CPU oracle for the exact scaled-dot-product attention: the forward
(sdpa_forward, sdpa_rows), ragged batches (sdpa_varlen_forward) and the
gradients (sdpa_backward).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may
import or run this module.  It shares no code with the CUDA path and imports
nothing from the ``exact_attention_sdpa_b200`` package.

What it computes is the plain definition, because the fused method is exact
(inskillml Module 9, "FlashAttention is not an approximation"; aiinarabic.com
"flash-attention", the exactness remark beside the O(N^2) -> O(N) memory
claim).  The definition is Equation (1) of aiinarabic.com "flash-attention",

    Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V,

evaluated row by row with the two-pass stable softmax that the gist.science
FLASHLIGHT summary (Methodology, item 3, semantic fusion) names as the thing
the online softmax replaces: pass 1 finds the row maximum, pass 2 sums the
exponentials shifted by it.  Readings of points the pages leave open:

* the explicit ``scale`` multiplies Q K^T, and the additive bias enters after
  scaling: s = scale * q.k + bias;
* causal: key j is visible to query i iff j <= i + (Nk - Nq).  For square
  problems (Nq = Nk, every workload the pages size) this is j <= i.  With
  fewer queries than keys the queries are read as the last Nq positions of the
  Nk-long sequence (the KV-cache reading of inskillml Module 9's general
  ``scaled_dot_product_attention`` use: a prefill chunk or a decode step
  attends to everything before and including itself), so the alignment is at
  the bottom right; with more queries than keys the first Nq - Nk rows see no
  key and are dead rows (below);
* lse_i = m_i + ln(l_i) in natural log, of the scaled, biased, masked scores;
  the gate does not enter it;
* the gate multiplies the normalised output elementwise by 1/(1+exp(-g));
* a row whose every score is -inf has O = 0 and lse = -inf;
* score modifications (inskillml Module 9's list of attention variants and
  patterns; FLASHLIGHT's named variants), all optional and applied in this
  order to s = scale * q.k + bias: ALiBi adds -slope_h * |i + (Nk - Nq) - j|
  (a per-head linear distance penalty); a logit softcap c > 0 replaces s by
  c * tanh(s / c); a left window w >= 0 masks keys j < i + (Nk - Nq) - w (a
  sliding window, together with the causal mask a band of w + 1 keys).

* the gradients with score modifications follow from the chain rule: the ALiBi
  shift and the window mask do not depend on Q or K, and the softcap multiplies
  dS by its derivative 1 - tanh(s / c)^2.

Inputs of any float dtype are upcast exactly to float64 before any arithmetic.
Parity: every function is pinned (tests/test_oracle.py, test_oracle_mods.py,
test_oracle_varlen.py, test_oracle_backward.py, test_oracle_properties.py).
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = ["sdpa_forward", "sdpa_rows", "sdpa_backward", "sdpa_varlen_forward", "to_f64"]


def to_f64(x) -> Optional[np.ndarray]:
    """Exact upcast of a torch tensor (fp16/bf16/fp32/fp64) or array to float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):                       # torch tensor, without importing torch here
        x = x.detach().cpu()
        if str(x.dtype) in ("torch.bfloat16", "torch.float16"):
            x = x.float()                          # exact widening
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _bias_rows(bias: Optional[np.ndarray], b: int, h: int, rows: np.ndarray) -> Optional[np.ndarray]:
    if bias is None:
        return None
    if bias.ndim == 3:                             # [H, Nq, Nk], shared over the batch (Evoformer pair bias)
        return bias[h, rows, :]
    return bias[b, h, rows, :]                     # [B, H, Nq, Nk]


def _attend_rows(qr, k, v, bias_r, gate_r, rows, causal, scale, offset=0, mods=None) -> Tuple[np.ndarray, np.ndarray]:
    """Two-pass stable softmax attention for a block of query rows of one (b, h).

    qr: [r, d] queries; k, v: [Nk, d]; bias_r: [r, Nk] or None; rows: the
    query indices of qr (for the causal mask); offset = Nk - Nq; mods: None or
    a dict with "alibi_slope" (this head's slope), "softcap", "window_left".
    """
    # step 1: scores s_ij = scale * q_i . k_j (+ bias_ij), causal keys j > i + offset masked to -inf
    s = scale * (qr @ k.T)
    if bias_r is not None:
        s = s + bias_r
    keys = np.arange(k.shape[0])
    if mods is not None:
        slope = mods.get("alibi_slope")
        if slope is not None:
            s = s - slope * np.abs(rows[:, None] + offset - keys[None, :])
        cap = mods.get("softcap", 0.0)
        if cap and cap > 0:
            s = cap * np.tanh(s / cap)
        w = mods.get("window_left", -1)
        if w is not None and w >= 0:
            s = np.where(keys[None, :] < rows[:, None] + offset - w, -np.inf, s)
    if causal:
        s = np.where(keys[None, :] > rows[:, None] + offset, -np.inf, s)
    # pass 1: row maximum
    m = s.max(axis=1)
    dead = ~np.isfinite(m) & (m < 0)               # every score of the row is -inf
    m_safe = np.where(dead, 0.0, m)
    # pass 2: shifted exponentials and their sum
    w = np.exp(s - m_safe[:, None])
    l = w.sum(axis=1)
    # output = weighted mean of the value rows; logsumexp of the scores
    with np.errstate(invalid="ignore", divide="ignore"):
        o = (w @ v) / l[:, None]
        lse = m + np.log(l)
    o = np.where(dead[:, None], 0.0, o)
    lse = np.where(dead, -np.inf, lse)
    if gate_r is not None:
        o = o * (1.0 / (1.0 + np.exp(-gate_r)))
    return o, lse


def _check(q, k, v, causal):
    assert q.ndim == 4 and k.ndim == 4 and v.ndim == 4, "q, k, v must be [B, H, N, d]"
    assert k.shape == v.shape and q.shape[:2] == k.shape[:2] and q.shape[3] == k.shape[3]
    assert k.shape[2] >= 1, "at least one key"


def _head_mods(softcap, alibi_slopes, window_left, h):
    if not softcap and alibi_slopes is None and (window_left is None or window_left < 0):
        return None
    return {"softcap": softcap or 0.0, "window_left": -1 if window_left is None else window_left,
            "alibi_slope": None if alibi_slopes is None else float(alibi_slopes[h])}


def sdpa_forward(q, k, v, bias=None, gate=None, causal: bool = False, scale: Optional[float] = None,
                 block_rows: int = 1024, softcap: float = 0.0, alibi_slopes=None,
                 window_left: int = -1) -> Tuple[np.ndarray, np.ndarray]:
    """Full forward: returns (O [B,H,Nq,d], lse [B,H,Nq]) in float64.

    q: [B,H,Nq,d]; k, v: [B,H,Nk,d]; bias: [H,Nq,Nk] or [B,H,Nq,Nk] or None;
    gate: [B,H,Nq,d] or None; scale defaults to 1/sqrt(d); softcap, alibi_slopes
    ([H]) and window_left as in the module docstring (off by default).
    Query rows are processed in blocks of ``block_rows`` only to bound memory.
    """
    alibi_slopes = None if alibi_slopes is None else to_f64(alibi_slopes)
    q, k, v, bias, gate = (to_f64(t) for t in (q, k, v, bias, gate))
    _check(q, k, v, causal)
    B, H, Nq, d = q.shape
    offset = k.shape[2] - Nq
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    O = np.zeros((B, H, Nq, d))
    L = np.zeros((B, H, Nq))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, Nq, block_rows):
                rows = np.arange(r0, min(Nq, r0 + block_rows))
                o, lse = _attend_rows(q[b, h, rows], k[b, h], v[b, h], _bias_rows(bias, b, h, rows),
                                      None if gate is None else gate[b, h, rows], rows, causal, scale, offset,
                                      _head_mods(softcap, alibi_slopes, window_left, h))
                O[b, h, rows] = o
                L[b, h, rows] = lse
    return O, L


def sdpa_rows(q, k, v, picks: Sequence[Tuple[int, int, int]], bias=None, gate=None, causal: bool = False,
              scale: Optional[float] = None, softcap: float = 0.0, alibi_slopes=None,
              window_left: int = -1) -> Tuple[np.ndarray, np.ndarray]:
    """Selected output rows only: picks = [(b, h, i), ...]; returns (O [n,d], lse [n]) in float64.

    Used to check full-size problems on a sample of rows; each row is computed
    from the whole of its K, V exactly as in ``sdpa_forward``.
    """
    d = q.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out_o = np.zeros((len(picks), d))
    out_l = np.zeros(len(picks))
    by_bh = {}
    for n, (b, h, i) in enumerate(picks):
        by_bh.setdefault((b, h), []).append((n, i))
    for (b, h), lst in by_bh.items():
        idx = np.array([i for _, i in lst])
        qr = to_f64(q[b, h][idx])
        kb, vb = to_f64(k[b, h]), to_f64(v[b, h])
        br = None
        if bias is not None:
            bsel = bias[h] if bias.ndim == 3 else bias[b, h]
            br = to_f64(bsel[idx])
        gr = None if gate is None else to_f64(gate[b, h][idx])
        slopes = None if alibi_slopes is None else to_f64(alibi_slopes)
        o, lse = _attend_rows(qr, kb, vb, br, gr, idx, causal, scale, k.shape[2] - q.shape[2],
                              _head_mods(softcap, slopes, window_left, h))
        for t, (n, _) in enumerate(lst):
            out_o[n] = o[t]
            out_l[n] = lse[t]
    return out_o, out_l


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def _grad_rows(q, k, v, do, causal, scale, offset, mods=None):
    """Gradients of one (b, h) head without bias or gate, from the definition.

    These are the derivatives of Equation (1) of aiinarabic.com
    "flash-attention" (S = scale Q K^T, masked; P = softmax_rows(S); O = P V)
    with respect to Q, K and V, given an upstream gradient dO.  (The same
    page's recomputation section is why a fused backward rebuilds S and P from
    Q, K and the saved normaliser; the oracle simply forms them.)

        dV = P^T dO
        dP = dO V^T
        dS = P * (dP - rowsum(P * dP))        (softmax Jacobian, row by row)
        dQ = scale dS K,   dK = scale dS^T Q

    P is formed here with the two-pass softmax of the forward definition (not
    from a saved lse), so the oracle does not depend on the forward under test.

    Score modifications (``mods`` as in _attend_rows, applied in the forward's
    order): the ALiBi shift and the window mask do not depend on Q or K, so they
    change only P; the softcap t = c tanh(s / c) has the derivative 1 - tanh(s / c)^2,
    by which dS is multiplied before dQ and dK are formed (the chain rule).
    """
    s = scale * (q @ k.T)
    rows = np.arange(q.shape[0])
    keys = np.arange(k.shape[0])
    dcap = None
    if mods is not None:
        slope = mods.get("alibi_slope")
        if slope is not None:
            s = s - slope * np.abs(rows[:, None] + offset - keys[None, :])
        cap = mods.get("softcap", 0.0)
        if cap and cap > 0:
            t = np.tanh(s / cap)
            s = cap * t
            dcap = 1.0 - t * t
        w = mods.get("window_left", -1)
        if w is not None and w >= 0:
            s = np.where(keys[None, :] < rows[:, None] + offset - w, -np.inf, s)
    if causal:
        s = np.where(keys[None, :] > rows[:, None] + offset, -np.inf, s)
    m = s.max(axis=1)
    dead = ~np.isfinite(m)
    m_safe = np.where(dead, 0.0, m)
    w = np.exp(s - m_safe[:, None])
    l = w.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        p = w / l[:, None]
    p = np.where(dead[:, None], 0.0, p)
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    if dcap is not None:
        ds = ds * dcap
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def sdpa_backward(q, k, v, do, causal: bool = False, scale: Optional[float] = None, softcap: float = 0.0,
                  alibi_slopes=None, window_left: int = -1) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(dQ, dK, dV) in float64 for O = softmax(scale Q K^T [causal]) V and upstream dO.

    q, do: [B,H,Nq,d]; k, v: [B,H,Nk,d]; causal masking aligned as in the forward
    (key j visible to query i iff j <= i + Nk - Nq).  No bias or gate.  softcap,
    alibi_slopes ([H]) and window_left as in sdpa_forward (off by default).
    """
    alibi_slopes = None if alibi_slopes is None else to_f64(alibi_slopes)
    q, k, v, do = (to_f64(t) for t in (q, k, v, do))
    _check(q, k, v, causal)
    assert do.shape == q.shape
    B, H, Nq, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dQ, dK, dV = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            dQ[b, h], dK[b, h], dV[b, h] = _grad_rows(q[b, h], k[b, h], v[b, h], do[b, h], causal, scale,
                                                      k.shape[2] - Nq,
                                                      mods=_head_mods(softcap, alibi_slopes, window_left, h))
    return dQ, dK, dV


# ---------------------------------------------------------------------------
# ragged batches
# ---------------------------------------------------------------------------

def sdpa_varlen_forward(q, k, v, cu_q: Sequence[int], cu_k: Sequence[int], causal: bool = False,
                        scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Sequences of different lengths packed along the token axis.

    q: [Tq, H, d] with sequence b in rows cu_q[b] .. cu_q[b+1]; k, v: [Tk, H, d]
    likewise with cu_k.  Each sequence is its own attention problem (no token
    attends across a sequence boundary), with the bottom-right causal alignment
    of sdpa_forward when its query and key counts differ.  Returns O [Tq, H, d]
    and lse [H, Tq] in float64; a sequence with no query rows contributes nothing,
    one with queries but no keys has dead rows (O = 0, lse = -inf).
    """
    q, k, v = (to_f64(t) for t in (q, k, v))
    Tq, H, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    O = np.zeros((Tq, H, d))
    L = np.full((H, Tq), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0 or k1 == k0:
            continue
        qs = q[q0:q1].transpose(1, 0, 2)[None]        # [1, H, n, d]
        ks = k[k0:k1].transpose(1, 0, 2)[None]
        vs = v[k0:k1].transpose(1, 0, 2)[None]
        o, lse = sdpa_forward(qs, ks, vs, causal=causal, scale=scale)
        O[q0:q1] = o[0].transpose(1, 0, 2)
        L[:, q0:q1] = lse[0]
    return O, L
