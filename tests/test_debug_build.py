"""The debug build (libattn_debug.so, -DATTN_DEBUG=1): the same kernels with their device-side
index and range checks compiled in (work-unit decode, tile coordinates and their 16-byte
alignment, the tensor-memory allocation, output rows).  A failed check sets a bit of the status
word (ATTN_ERR_CHECK) instead of faulting.  These tests run representative problems of every
kernel variant through the debug build and require no check to fail and the results to match
the oracle as the release build's do."""
import math

import numpy as np
import pytest
import torch

from exact_attention_sdpa_b200 import _native as nat
from exact_attention_sdpa_b200 import build as build_mod
from exact_attention_sdpa_b200.workloads import Workload, make_e4m3_inputs, make_grad_output, make_inputs
from oracle import sdpa_backward, sdpa_forward, sdpa_varlen_forward
from helpers import assert_close_to_oracle, padded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def debug_lib():
    path = build_mod.build(debug=True)
    lib = nat.load_library(path)
    saved = nat._lib
    nat._lib = lib                 # the binding's calls go to the debug build for these tests
    yield lib
    nat._lib = saved


def test_debug_build_reports_itself(debug_lib):
    assert debug_lib.attn_build_flags() & nat.ATTN_BUILD_DEBUG_CHECKS
    assert nat.load_library(nat.LIB_PATH).attn_build_flags() == 0


def _status_ok():
    torch.cuda.synchronize()
    assert nat.last_device_status() == nat.ATTN_OK


FWD = [  # B, H, N, Nk, d, causal, dtype, bias, gate, mods (softcap, window)
    (2, 3, 300, 300, 64, True, "fp16", False, False, None),
    (1, 2, 1000, 1000, 128, True, "bf16", False, False, None),
    (2, 2, 256, 256, 32, False, "bf16", True, True, None),
    (1, 2, 129, 700, 64, True, "bf16", False, False, (2.0, 100)),
    (1, 3, 640, 2048, 64, True, "fp16", False, False, None),
]


@pytest.mark.parametrize("B,H,N,Nk,d,causal,dtype,bias,gate,mods", FWD)
def test_forward_without_check_failures(debug_lib, B, H, N, Nk, d, causal, dtype, bias, gate, mods):
    w = Workload("dbg", B=B, H=H, N=N, d=d, dtype=dtype, causal=causal, seed=300 + N % 11, Nk=Nk, bias=bias,
                 gate=gate)
    inp = make_inputs(w)
    dev = torch.device("cuda")
    softcap, window = mods if mods else (0.0, -1)
    o, lse = nat.attn_fwd(inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev),
                          bias=None if inp["bias"] is None else padded(inp["bias"], dev),
                          gate=None if inp["gate"] is None else inp["gate"].to(dev), causal=causal, scale=w.scale,
                          softcap=softcap, window_left=window)
    _status_ok()
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], bias=inp["bias"], gate=inp["gate"], causal=causal,
                                scale=w.scale, softcap=softcap, window_left=window)
    assert_close_to_oracle(o, lse, o_ref, l_ref, w.torch_dtype, "debug build")


def test_ragged_batch_without_check_failures(debug_lib):
    lens = [(100, 100), (0, 0), (257, 257), (1, 1), (700, 900)]
    g = torch.Generator().manual_seed(5)
    Tq, Tk = sum(a for a, _ in lens), sum(b for _, b in lens)
    q, k, v = (torch.randn(T, 2, 64, generator=g).half() for T in (Tq, Tk, Tk))
    cq = torch.tensor([0] + list(np.cumsum([a for a, _ in lens])), dtype=torch.int32)
    ck = torch.tensor([0] + list(np.cumsum([b for _, b in lens])), dtype=torch.int32)
    dev = torch.device("cuda")
    o, lse = nat.attn_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), cq, ck, causal=True)
    _status_ok()
    o_ref, l_ref = sdpa_varlen_forward(q, k, v, cq.tolist(), ck.tolist(), causal=True)
    assert_close_to_oracle(o, lse, o_ref, l_ref, torch.float16, "debug build ragged")


def test_fp8_and_backward_without_check_failures(debug_lib):
    dev = torch.device("cuda")
    w = Workload("dbg8", B=1, H=2, N=300, d=128, dtype="bf16", causal=True, seed=321)
    inp = make_e4m3_inputs(w)
    B, H, Nk, d = inp["v"].shape
    vt = torch.zeros(B, H, d, (Nk + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    vt[..., :Nk] = inp["v"].view(torch.uint8).transpose(-1, -2).to(dev)
    o, lse = nat.attn_fwd_fp8(inp["q"].to(dev), inp["k"].to(dev), vt[..., :Nk].view(torch.float8_e4m3fn),
                              inp["q_scale"], inp["k_scale"], inp["v_scale"], causal=True)
    _status_ok()
    assert torch.isfinite(o).all()
    w = Workload("dbgb", B=2, H=2, N=200, d=64, dtype="bf16", causal=True, seed=322)
    x = make_inputs(w)
    do = make_grad_output(w)
    q, k, v = (x[n].to(dev) for n in "qkv")
    out, lse = nat.attn_fwd(q, k, v, causal=True, scale=w.scale)
    grads = nat.attn_bwd(q, k, v, out, lse, do.to(dev), causal=True, scale=w.scale)
    _status_ok()
    for g, r in zip(grads, sdpa_backward(x["q"], x["k"], x["v"], do, causal=True, scale=w.scale)):
        err = float((g.double().cpu() - torch.as_tensor(r)).abs().max())
        assert err <= 2e-2 * max(1.0, float(np.abs(r).max()))
