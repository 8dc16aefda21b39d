"""Host-side checks of the seeded input recipe and the metric's FLOP and byte
counts (no GPU): the counts are written from the definitions the bench states."""
import torch

from exact_attention_sdpa_b200.workloads import (WORKLOADS, Workload, algorithmic_bytes, alibi_slopes,
                                                 attention_flops, make_e4m3_inputs, make_grad_output, make_inputs,
                                                 make_varlen_inputs)


def test_square_counts_match_the_metric():
    w = WORKLOADS["n8192_causal"]
    assert attention_flops(w) == 4.0 * 4 * 12 * 8192 * 8192 * 64 / 2
    assert algorithmic_bytes(w) == 4 * (4 * 12 * 8192 * 64 * 2) + 4 * 12 * 8192 * 4
    e = WORKLOADS["evoformer_row"]
    assert algorithmic_bytes(e) == 5 * (256 * 8 * 256 * 32 * 2) + 8 * 256 * 256 * 2 + 256 * 8 * 256 * 4


def test_rectangular_causal_counts_visible_pairs():
    w = Workload("r", B=1, H=1, N=3, d=8, dtype="fp16", causal=True, seed=0, Nk=5)
    assert attention_flops(w) == 4.0 * 8 * (3 + 4 + 5)          # query i sees i + 3 keys
    w2 = w.with_(N=5, Nk=3)
    assert attention_flops(w2) == 4.0 * 8 * (0 + 0 + 1 + 2 + 3)  # the first two rows see none
    w3 = w.with_(causal=False)
    assert attention_flops(w3) == 4.0 * 8 * 3 * 5


def test_inputs_are_seeded_and_shaped():
    w = Workload("s", B=2, H=3, N=17, d=32, dtype="bf16", causal=False, seed=11, Nk=29, bias=True, gate=True)
    a, b = make_inputs(w), make_inputs(w)
    for k in ("q", "k", "v", "bias", "gate"):
        assert torch.equal(a[k], b[k])
    assert a["q"].shape == (2, 3, 17, 32) and a["k"].shape == (2, 3, 29, 32) and a["bias"].shape == (3, 17, 29)
    assert a["q"].dtype == torch.bfloat16
    g = make_grad_output(w)
    assert g.shape == a["q"].shape and not torch.equal(g, a["q"])


def test_varlen_inputs_and_counts():
    w = WORKLOADS["varlen_mix"]
    inp = make_varlen_inputs(w)
    T = sum(w.lengths)
    assert inp["q"].shape == (T, w.H, w.d) and inp["cu_seqlens"][-1].item() == T
    assert inp["cu_seqlens"].dtype == torch.int32 and inp["cu_seqlens"][0].item() == 0
    assert attention_flops(w) == sum(4.0 * w.H * n * n * w.d for n in w.lengths) / 2


def test_alibi_slopes():
    assert alibi_slopes(WORKLOADS["n8192_causal"]) is None
    s = alibi_slopes(WORKLOADS["n8192_alibi_softcap"])
    assert s.shape == (12,) and abs(s[0].item() - 2 ** (-8 / 12)) < 1e-7 and abs(s[-1].item() - 2 ** -8) < 1e-9


def test_window_counts_visible_pairs_by_brute_force():
    for n, nk, causal, wl in [(7, 7, True, 2), (5, 9, True, 3), (9, 4, True, 1), (6, 8, False, 2), (300, 300, True, 63)]:
        w = Workload("win", B=2, H=3, N=n, d=8, dtype="fp16", causal=causal, seed=0, Nk=nk, window_left=wl)
        off = nk - n
        pairs = sum(1 for i in range(n) for j in range(nk)
                    if j >= i + off - wl and (not causal or j <= i + off))
        assert attention_flops(w) == 4.0 * 2 * 3 * 8 * pairs
    big = WORKLOADS["n8192_window"]
    assert attention_flops(big) == 4.0 * 4 * 12 * 64 * sum(min(i, 1023) + 1 for i in range(8192))


def test_e4m3_inputs_are_seeded_scaled_codes_of_the_same_draws():
    import math
    w = Workload("f8", B=1, H=2, N=40, d=64, dtype="bf16", causal=True, seed=21, Nk=72)
    a, b = make_e4m3_inputs(w), make_e4m3_inputs(w)
    g = torch.Generator().manual_seed(21)
    for name, n in (("q", 40), ("k", 72), ("v", 72)):
        c = a[name]
        assert c.dtype == torch.float8_e4m3fn and c.shape == (1, 2, n, 64)
        assert torch.equal(c.view(torch.uint8), b[name].view(torch.uint8))
        s = a[name + "_scale"]
        assert s > 0 and math.log2(s) == round(math.log2(s))             # a power of two
        x = torch.randn(1, 2, n, 64, generator=g, dtype=torch.float32).double()   # the same draws
        y = c.to(torch.float64) * s
        assert not torch.isnan(y).any() and float(y.abs().max()) <= 448 * s
        # e4m3 rounding: within 2^-4 relative for normal values, 2^-10 * s absolute below 2^-6 * s
        err = (y - x).abs()
        assert bool((err <= torch.maximum(x.abs() * 2.0 ** -4, torch.full_like(x, 2.0 ** -10 * s))).all())
