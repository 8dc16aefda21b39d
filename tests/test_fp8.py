"""GPU parity of the FP8 (e4m3) forward (attn_fwd_fp8) against the fp64 oracle on the decoded,
scaled e4m3 inputs (oracle.fp8.sdpa_forward_fp8), element by element.

Tolerance per output element: the bound oracle.fp8.p_rounding_bound derives for rounding P to
e4m3 (the kernel's one added rounding), plus the output's rounding into its dtype (half an
ulp: 2^-9 relative for bf16, 2^-11 for fp16), plus 2e-3 of max|V| for the fp32 accumulation
order and the approximate exponentials.  lse involves no rounding of P (the row sum adds the
unrounded values): |lse - lse_ref| <= 1e-3 * max(1, |lse_ref|), as for the 16-bit forward."""
import math

import numpy as np
import pytest
import torch

from exact_attention_sdpa_b200 import attn_fwd_fp8, last_device_status
from exact_attention_sdpa_b200.workloads import WORKLOADS, Workload, make_e4m3_inputs
from oracle.fp8 import p_rounding_bound, sdpa_forward_fp8

pytestmark = pytest.mark.gpu


def transposed_padded(v: torch.Tensor, dev) -> torch.Tensor:
    """V [B, H, Nk, d] -> V^T [B, H, d, Nk] on the device, rows padded to 16 bytes."""
    B, H, Nk, d = v.shape
    buf = torch.zeros(B, H, d, (Nk + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    buf[..., :Nk] = v.view(torch.uint8).transpose(-1, -2).to(dev)
    return buf[..., :Nk].view(torch.float8_e4m3fn)


def run_fp8(inp, causal, scale, out_dtype):
    dev = torch.device("cuda")
    q, k = inp["q"].to(dev), inp["k"].to(dev)
    vt = transposed_padded(inp["v"], dev)
    o, lse = attn_fwd_fp8(q, k, vt, inp["q_scale"], inp["k_scale"], inp["v_scale"], causal=causal, scale=scale,
                          out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    return o, lse


def check(inp, o, lse, causal, scale, out_dtype, what):
    codes = {n: inp[n].view(torch.uint8).numpy() for n in "qkv"}
    args = (codes["q"], codes["k"], codes["v"], inp["q_scale"], inp["k_scale"], inp["v_scale"])
    o_ref, l_ref = sdpa_forward_fp8(*args, causal=causal, scale=scale)
    bound = p_rounding_bound(*args, causal=causal, scale=scale)
    half_ulp = 2.0 ** -9 if out_dtype == torch.bfloat16 else 2.0 ** -11
    vmax = float(np.nanmax(np.abs(inp["v"].float().numpy()))) * inp["v_scale"]
    tol = bound + half_ulp * np.abs(o_ref) + 2e-3 * vmax
    err = np.abs(o.double().cpu().numpy() - o_ref)
    worst = float((err / tol).max())
    assert worst <= 1.0, f"{what}: max |dO| / tolerance = {worst:.3f} (max |dO| {float(err.max()):.3e})"
    l = lse.double().cpu().numpy()
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l), fin)
    assert np.all(np.abs(l[fin] - l_ref[fin]) <= 1e-3 * np.maximum(1.0, np.abs(l_ref[fin]))), what
    return worst


CASES = [  # B, H, N, Nk, d, causal, out dtype
    (1, 2, 256, 256, 64, False, torch.bfloat16),
    (1, 2, 300, 300, 64, True, torch.float16),
    (1, 1, 200, 520, 128, True, torch.bfloat16),
    (2, 1, 129, 129, 128, False, torch.float16),
    (2, 3, 1000, 1000, 64, True, torch.bfloat16),      # several key tiles, ragged tail
    (1, 2, 640, 2048, 128, True, torch.bfloat16),      # prefill chunk against a longer key sequence
]


@pytest.mark.parametrize("B,H,N,Nk,d,causal,out_dtype", CASES)
def test_fp8_forward_matches_oracle(B, H, N, Nk, d, causal, out_dtype):
    w = Workload("fp8", B=B, H=H, N=N, d=d, dtype="bf16", causal=causal, seed=200 + N % 17, Nk=Nk)
    inp = make_e4m3_inputs(w)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_fp8(inp, causal, scale, out_dtype)
    check(inp, o, lse, causal, scale, out_dtype, f"fp8 {B}x{H}x{N}x{Nk}x{d}")


def test_fp8_full_size_heads():
    """The N=8192 causal d=64 shape of the benchmarked workload on e4m3 inputs, in the launch
    configuration the benchmark times: every row of two whole heads compared."""
    w = WORKLOADS["n8192_causal"]
    inp = make_e4m3_inputs(w)
    o, lse = run_fp8(inp, True, w.scale, torch.float16)
    assert torch.isfinite(o).all()
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        sub = {n: inp[n][b:b + 1, h:h + 1] for n in "qkv"}
        sub.update({n + "_scale": inp[n + "_scale"] for n in "qkv"})
        check(sub, o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], True, w.scale, torch.float16, f"n8192 head ({b},{h})")


def test_fp8_scales_fold_exactly():
    """Doubling q_scale and halving k_scale leaves every score, hence O and lse, unchanged bit for bit."""
    w = Workload("fp8s", B=1, H=2, N=300, d=64, dtype="bf16", causal=True, seed=211)
    inp = make_e4m3_inputs(w)
    o1, l1 = run_fp8(inp, True, 0.125, torch.bfloat16)
    inp2 = dict(inp, q_scale=inp["q_scale"] * 2.0, k_scale=inp["k_scale"] * 0.5)
    o2, l2 = run_fp8(inp2, True, 0.125, torch.bfloat16)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
