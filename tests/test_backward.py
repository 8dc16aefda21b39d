"""GPU parity of the backward (attn_bwd) against the fp64 oracle's sdpa_backward
on the same seeded inputs and upstream gradient, element by element.

Tolerance (a reading: the pages state none for gradients): the forward's O
tolerances relative to the gradient's own scale, max |dX - dX_ref| <=
2e-2 (bf16) or 5e-3 (fp16) times max(1, max |dX_ref|), for X in Q, K, V.  The
kernel accumulates in fp32 and rounds once into the dtype; the forward O it is
given (for D = rowsum(dO * O)) is itself rounded to the dtype."""
import pytest
import torch

from exact_attention_sdpa_b200 import attn_bwd, attn_fwd, last_device_status
from exact_attention_sdpa_b200.workloads import Workload, make_grad_output, make_inputs
from oracle import sdpa_backward

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float16: 5e-3}

CASES = [  # B, H, N, Nk, d, causal, dtype
    (1, 2, 64, 64, 64, False, "fp16"),
    (2, 3, 200, 200, 64, True, "bf16"),
    (1, 2, 129, 300, 32, True, "fp16"),
    (2, 2, 300, 100, 128, True, "bf16"),
    (1, 4, 257, 257, 128, False, "fp16"),
    (1, 1, 1, 500, 64, True, "bf16"),
    (2, 2, 384, 384, 32, False, "bf16"),
    # fewer column blocks than TMEM column sets: dK/dV sees 2 query blocks and dQ 3 key blocks
    # (three sets at d=64), then 3 and 2 at d=128 (two sets)
    (1, 2, 128, 192, 64, False, "fp16"),
    (1, 2, 192, 128, 128, False, "bf16"),
]


def _check(g, ref, dtype, what):
    ref = torch.as_tensor(ref)
    err = (g.double().cpu() - ref).abs().max().item()
    bound = TOL[dtype] * max(1.0, ref.abs().max().item())
    assert torch.isfinite(g).all(), what
    assert err <= bound, f"{what}: max err {err:.3e} > {bound:.3e}"
    return err


@pytest.mark.parametrize("B,H,N,Nk,d,causal,dtype", CASES)
def test_backward_matches_oracle(B, H, N, Nk, d, causal, dtype):
    w = Workload("bwd", B=B, H=H, N=N, d=d, dtype=dtype, causal=causal, seed=70 + N % 13, Nk=Nk)
    inp = make_inputs(w)
    do = make_grad_output(w)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    out, lse = attn_fwd(q, k, v, causal=causal, scale=w.scale)
    dq, dk, dv = attn_bwd(q, k, v, out, lse, do.to(dev), causal=causal, scale=w.scale)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    rq, rk, rv = sdpa_backward(inp["q"], inp["k"], inp["v"], do, causal=causal, scale=w.scale)
    for g, r, name in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
        _check(g, r, w.torch_dtype, f"{name} {B}x{H}x{N}x{Nk}x{d} causal={causal}")


def test_backward_deterministic():
    w = Workload("bwdd", B=2, H=2, N=300, d=64, dtype="bf16", causal=True, seed=77)
    inp = make_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    do = make_grad_output(w).to(dev)
    out, lse = attn_fwd(q, k, v, causal=True, scale=w.scale)
    first = attn_bwd(q, k, v, out, lse, do, causal=True, scale=w.scale)
    for _ in range(3):
        again = attn_bwd(q, k, v, out, lse, do, causal=True, scale=w.scale)
        assert all(torch.equal(a, b) for a, b in zip(first, again))


MOD_CASES = [  # N, Nk, d, causal, dtype, softcap, alibi, window
    (300, 300, 64, True, "fp16", 2.0, False, -1),
    (257, 400, 128, True, "bf16", 0.0, True, -1),
    (400, 400, 32, True, "bf16", 0.0, False, 100),
    (300, 700, 64, True, "bf16", 1.5, True, 200),
    (200, 200, 64, False, "fp16", 3.0, True, 50),
]


@pytest.mark.parametrize("N,Nk,d,causal,dtype,softcap,alibi,window", MOD_CASES)
def test_backward_with_score_modifications(N, Nk, d, causal, dtype, softcap, alibi, window):
    H = 3
    w = Workload("bwdm", B=2, H=H, N=N, d=d, dtype=dtype, causal=causal, seed=150 + N % 11, Nk=Nk)
    inp = make_inputs(w)
    do = make_grad_output(w)
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32) if alibi else None
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    sd = None if slopes is None else slopes.to(dev)
    out, lse = attn_fwd(q, k, v, causal=causal, scale=w.scale, softcap=softcap, alibi_slopes=sd, window_left=window)
    dq, dk, dv = attn_bwd(q, k, v, out, lse, do.to(dev), causal=causal, scale=w.scale, softcap=softcap,
                          alibi_slopes=sd, window_left=window)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    rq, rk, rv = sdpa_backward(inp["q"], inp["k"], inp["v"], do, causal=causal, scale=w.scale, softcap=softcap,
                               alibi_slopes=slopes, window_left=window)
    for g, r, name in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
        _check(g, r, w.torch_dtype, f"{name} mods N={N} Nk={Nk} d={d}")


def test_backward_full_size_two_heads():
    """The N=8192 causal fp16 workload in the launch configuration the benchmark times; the
    oracle's gradients of two whole (b, h) heads are compared element by element."""
    from exact_attention_sdpa_b200.workloads import WORKLOADS
    w = WORKLOADS["n8192_causal"]
    inp = make_inputs(w)
    do = make_grad_output(w)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    out, lse = attn_fwd(q, k, v, causal=True, scale=w.scale)
    dq, dk, dv = attn_bwd(q, k, v, out, lse, do.to(dev), causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv = sdpa_backward(inp["q"][sl], inp["k"][sl], inp["v"][sl], do[sl], causal=True, scale=w.scale)
        for g, r, name in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
            _check(g[sl], r, w.torch_dtype, f"{name} n8192 head ({b},{h})")
