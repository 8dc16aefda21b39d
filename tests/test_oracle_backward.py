"""Pins for the fp64 oracle's backward: central finite differences of the
forward oracle (itself pinned in test_oracle.py), autograd of torch's own
scaled_dot_product_attention in float64, closed forms, an invariant, and a
mutation test showing that plausible mistakes are caught."""
import numpy as np
import pytest
import torch

import oracle.sdpa as osdpa
from oracle import sdpa_backward, sdpa_forward

RNG = np.random.default_rng


def _rand(shape, seed, scale=1.0):
    return RNG(seed).standard_normal(shape) * scale


def _fd_grads(q, k, v, do, causal, scale, eps=1e-6):
    """Central differences of L = sum(dO * O) with respect to every input element."""
    def loss(q_, k_, v_):
        o, _ = sdpa_forward(q_, k_, v_, causal=causal, scale=scale)
        return float((o * do).sum())
    grads = []
    for which in range(3):
        xs = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(xs[which])
        it = np.nditer(g, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = [x.copy() for x in xs]
            xm = [x.copy() for x in xs]
            xp[which][idx] += eps
            xm[which][idx] -= eps
            g[idx] = (loss(*xp) - loss(*xm)) / (2 * eps)
        grads.append(g)
    return grads


def pin_finite_differences(bwd):
    for causal, (nq, nk) in [(False, (5, 7)), (True, (5, 5)), (True, (3, 7)), (True, (6, 4))]:
        q = _rand((1, 2, nq, 3), 200 + nq)
        k = _rand((1, 2, nk, 3), 210 + nk)
        v = _rand((1, 2, nk, 3), 220 + nk)
        do = _rand((1, 2, nq, 3), 230 + nq)
        dq, dk, dv = bwd(q, k, v, do, causal=causal, scale=0.7)
        fq, fk, fv = _fd_grads(q, k, v, do, causal, 0.7)
        for a, b in ((dq, fq), (dk, fk), (dv, fv)):
            np.testing.assert_allclose(a, b, rtol=0, atol=2e-8)


def pin_torch_autograd(bwd):
    for causal, (nq, nk) in [(False, (9, 13)), (True, (11, 11)), (True, (4, 12))]:
        q = _rand((2, 2, nq, 8), 240)
        k = _rand((2, 2, nk, 8), 241)
        v = _rand((2, 2, nk, 8), 242)
        do = _rand((2, 2, nq, 8), 243)
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
        mask = None
        if causal:   # bottom-right alignment written as an explicit boolean mask
            mask = torch.ones(nq, nk, dtype=torch.bool).tril(diagonal=nk - nq)
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.5)
        o.backward(torch.tensor(do))
        dq, dk, dv = bwd(q, k, v, do, causal=causal, scale=0.5)
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-12)


def pin_scale_zero_closed_form(bwd):
    # scale 0: P is uniform over the visible keys and does not depend on Q or K
    q = _rand((1, 1, 6, 4), 250)
    k = _rand((1, 1, 6, 4), 251)
    v = _rand((1, 1, 6, 4), 252)
    do = _rand((1, 1, 6, 4), 253)
    dq, dk, dv = bwd(q, k, v, do, causal=True, scale=0.0)
    assert np.all(dq == 0.0) and np.all(dk == 0.0)
    ref = np.zeros((6, 4))
    for i in range(6):
        ref[: i + 1] += do[0, 0, i] / (i + 1)
    np.testing.assert_allclose(dv[0, 0], ref, rtol=0, atol=1e-15)


def pin_identical_values_give_no_score_gradient(bwd):
    # all value rows equal: O does not depend on P, so dQ = dK = 0 and dV sums dO
    q = _rand((1, 2, 5, 4), 260)
    k = _rand((1, 2, 5, 4), 261)
    v = np.broadcast_to(_rand((4,), 262), (1, 2, 5, 4)).copy()
    do = _rand((1, 2, 5, 4), 263)
    dq, dk, dv = bwd(q, k, v, do, causal=False, scale=0.9)
    np.testing.assert_allclose(dq, 0.0, atol=1e-14)
    np.testing.assert_allclose(dk, 0.0, atol=1e-14)
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-13)


BWD_PINS = [pin_finite_differences, pin_torch_autograd, pin_scale_zero_closed_form,
            pin_identical_values_give_no_score_gradient]


@pytest.mark.parametrize("pin", BWD_PINS, ids=[p.__name__ for p in BWD_PINS])
def test_backward_pin(pin):
    pin(sdpa_backward)


def _mutant(kind):
    real = osdpa._grad_rows

    def grad(q, k, v, do, causal, scale, offset, mods=None):
        if kind == "dq_without_scale":
            dq, dk, dv = real(q, k, v, do, causal, scale, offset, mods)
            return dq / scale if scale != 0 else dq, dk, dv
        if kind == "softmax_jacobian_sign":
            s = scale * (q @ k.T)
            if causal:
                rows, keys = np.arange(q.shape[0]), np.arange(k.shape[0])
                s = np.where(keys[None, :] > rows[:, None] + offset, -np.inf, s)
            p = np.exp(s - s.max(1, keepdims=True))
            p /= p.sum(1, keepdims=True)
            dp = do @ v.T
            ds = p * (dp + (p * dp).sum(1, keepdims=True))
            return scale * ds @ k, scale * ds.T @ q, p.T @ do
        if kind == "dk_from_k":
            dq, dk, dv = real(q, k, v, do, causal, scale, offset, mods)
            return dq, dk * 0 + scale * (q.T @ q)[:1].repeat(k.shape[0], 0)[:, : k.shape[1]], dv
        if kind == "dv_untransposed":
            dq, dk, dv = real(q, k, v, do, causal, scale, offset, mods)
            s = scale * (q @ k.T)
            p = np.exp(s - s.max(1, keepdims=True))
            p /= p.sum(1, keepdims=True)
            if p.shape[0] == p.shape[1]:
                return dq, dk, p @ do
            return dq, dk, dv[::-1]
        if kind == "no_causal_mask":
            return real(q, k, v, do, False, scale, offset, mods)
        if kind == "top_left_alignment":
            return real(q, k, v, do, causal, scale, 0, mods)
        return real(q, k, v, do, causal, scale, offset, mods)

    return grad


@pytest.mark.parametrize("kind", ["dq_without_scale", "softmax_jacobian_sign", "dk_from_k", "dv_untransposed",
                                  "no_causal_mask", "top_left_alignment"])
def test_backward_pins_catch_planted_mistake(kind, monkeypatch):
    monkeypatch.setattr(osdpa, "_grad_rows", _mutant(kind))
    caught = 0
    for pin in BWD_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(osdpa.sdpa_backward)
        except (AssertionError, FloatingPointError, ValueError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {kind!r}"



# ---------------------------------------------------------------------------- score modifications
def _fd_grads_mods(q, k, v, do, causal, scale, mods, eps=1e-6):
    def loss(q_, k_, v_):
        o, _ = sdpa_forward(q_, k_, v_, causal=causal, scale=scale, **mods)
        return float((o * do).sum())
    grads = []
    for which in range(3):
        xs = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(xs[which])
        it = np.nditer(g, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = [x.copy() for x in xs]
            xm = [x.copy() for x in xs]
            xp[which][idx] += eps
            xm[which][idx] -= eps
            g[idx] = (loss(*xp) - loss(*xm)) / (2 * eps)
        grads.append(g)
    return grads


MOD_CASES = [  # (causal, nq, nk, softcap, alibi, window)
    (False, 5, 7, 1.3, True, -1),
    (True, 6, 6, 0.9, False, 2),
    (True, 4, 7, 2.0, True, 3),
    (True, 6, 4, 0.0, True, 1),     # more queries than keys: dead rows
]


def pin_mods_finite_differences(bwd):
    for causal, nq, nk, cap, alibi, win in MOD_CASES:
        q = _rand((1, 2, nq, 3), 500 + nq, 2.0)
        k = _rand((1, 2, nk, 3), 510 + nk, 2.0)
        v = _rand((1, 2, nk, 3), 520 + nk)
        do = _rand((1, 2, nq, 3), 530 + nq)
        mods = {"softcap": cap, "alibi_slopes": np.array([0.5, 0.125]) if alibi else None, "window_left": win}
        dq, dk, dv = bwd(q, k, v, do, causal=causal, scale=0.7, **mods)
        fq, fk, fv = _fd_grads_mods(q, k, v, do, causal, 0.7, mods)
        for a, b in ((dq, fq), (dk, fk), (dv, fv)):
            np.testing.assert_allclose(a, b, rtol=0, atol=5e-8)


def pin_mods_limits_are_the_plain_backward(bwd):
    q, k, v, do = (_rand((1, 2, 6, 4), 540 + i) for i in range(4))
    plain = bwd(q, k, v, do, causal=True, scale=0.5)
    for mods in ({"softcap": 1e7}, {"alibi_slopes": np.zeros(2)}, {"window_left": 100}):
        got = bwd(q, k, v, do, causal=True, scale=0.5, **mods)
        for a, b in zip(got, plain):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-9)


MOD_BWD_PINS = [pin_mods_finite_differences, pin_mods_limits_are_the_plain_backward]


@pytest.mark.parametrize("pin", MOD_BWD_PINS, ids=[p.__name__ for p in MOD_BWD_PINS])
def test_backward_mods_pin(pin):
    pin(sdpa_backward)


def _mods_mutant(kind):
    real = osdpa._grad_rows

    def grad(q, k, v, do, causal, scale, offset, mods=None):
        if mods is not None:
            mods = dict(mods)
            if kind == "no_softcap_derivative" and mods.get("softcap", 0) > 0:
                # P with the softcap, but dS not multiplied by its derivative
                cap = mods.pop("softcap")
                s = scale * (q @ k.T)
                rows, keys = np.arange(q.shape[0]), np.arange(k.shape[0])
                if mods.get("alibi_slope") is not None:
                    s = s - mods["alibi_slope"] * np.abs(rows[:, None] + offset - keys[None, :])
                s = cap * np.tanh(s / cap)
                w = mods.get("window_left", -1)
                if w is not None and w >= 0:
                    s = np.where(keys[None, :] < rows[:, None] + offset - w, -np.inf, s)
                if causal:
                    s = np.where(keys[None, :] > rows[:, None] + offset, -np.inf, s)
                m = s.max(1, keepdims=True)
                m = np.where(np.isfinite(m), m, 0.0)
                p = np.exp(s - m)
                l = p.sum(1, keepdims=True)
                p = np.where(l > 0, p / np.where(l > 0, l, 1.0), 0.0)
                dp = do @ v.T
                ds = p * (dp - (p * dp).sum(1, keepdims=True))
                return scale * ds @ k, scale * ds.T @ q, p.T @ do
            if kind == "alibi_ignored":
                mods["alibi_slope"] = None
            if kind == "window_ignored":
                mods["window_left"] = -1
        return real(q, k, v, do, causal, scale, offset, mods)
    return grad


@pytest.mark.parametrize("kind", ["no_softcap_derivative", "alibi_ignored", "window_ignored"])
def test_backward_mods_pins_catch_planted_mistake(kind, monkeypatch):
    monkeypatch.setattr(osdpa, "_grad_rows", _mods_mutant(kind))
    caught = 0
    for pin in MOD_BWD_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(osdpa.sdpa_backward)
        except (AssertionError, FloatingPointError, ValueError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {kind!r}"
