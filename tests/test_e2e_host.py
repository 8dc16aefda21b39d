"""The end-to-end entry point with host buffers (attn_fwd_host, and attn_fwd_host_ex with
score modifications, reached through fwd()): host inputs are copied to device staging buffers, the same kernel runs,
O and lse come back to host memory.  Results must equal the device-path call bit
for bit and the oracle within tolerance; two streams with their own staging
buffers may run calls concurrently."""
import pytest
import torch

from exact_attention_sdpa_b200 import Staging, attn_fwd, fwd, last_device_status
from exact_attention_sdpa_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import sdpa_forward
from helpers import assert_close_to_oracle

pytestmark = pytest.mark.gpu


def _pinned(inp):
    return {k: (None if t is None else t.pin_memory()) for k, t in inp.items()}


@pytest.mark.parametrize("name", ["tiny", "gpt2_small", "evoformer_row"])
def test_host_path_matches_device_path_and_oracle(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    h = _pinned(inp)
    o_h, l_h = fwd(h["q"], h["k"], h["v"], bias=h["bias"], gate=h["gate"], causal=w.causal, scale=w.scale)
    assert not o_h.is_cuda and not l_h.is_cuda
    dev = torch.device("cuda")
    d = {k: (None if t is None else t.to(dev)) for k, t in inp.items()}
    o_d, l_d = attn_fwd(d["q"], d["k"], d["v"], bias=d["bias"], gate=d["gate"], causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], bias=inp["bias"], gate=inp["gate"],
                                causal=w.causal, scale=w.scale)
    assert_close_to_oracle(o_h, l_h, o_ref, l_ref, w.torch_dtype, name + "-host")


@pytest.mark.parametrize("softcap,alibi,window", [(30.0, True, -1), (0.0, False, 300), (2.0, False, 129)])
def test_host_path_with_score_modifications(softcap, alibi, window):
    """attn_fwd_host_ex: the same kernel as attn_fwd_ex on the staged inputs (ALiBi slopes on
    the device), so the host results equal the device path's bit for bit, and the oracle's."""
    w = Workload("hm", B=2, H=4, N=700, d=64, dtype="bf16", causal=True, seed=55)
    inp = make_inputs(w)
    h = _pinned(inp)
    dev = torch.device("cuda")
    slopes = torch.tensor([2.0 ** (-8.0 * (i + 1) / w.H) for i in range(w.H)], dtype=torch.float32) if alibi else None
    sd = None if slopes is None else slopes.to(dev)
    kw = dict(causal=True, scale=w.scale, softcap=softcap, alibi_slopes=sd, window_left=window)
    o_h, l_h = fwd(h["q"], h["k"], h["v"], **kw)
    assert not o_h.is_cuda
    o_d, l_d = attn_fwd(inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev), **kw)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], causal=True, scale=w.scale, softcap=softcap,
                                alibi_slopes=slopes, window_left=window)
    assert_close_to_oracle(o_h, l_h, o_ref, l_ref, w.torch_dtype, "host path with modifications")


def test_two_streams_pipeline():
    """Alternating calls on two streams with their own staging and host outputs:
    every call's outputs equal the single-call result."""
    ws = [Workload("p0", B=2, H=4, N=640, d=64, dtype="fp16", causal=True, seed=51),
          Workload("p1", B=2, H=4, N=640, d=64, dtype="fp16", causal=True, seed=52)]
    hs = [_pinned(make_inputs(w)) for w in ws]
    ref = [fwd(h["q"], h["k"], h["v"], causal=True, scale=ws[0].scale) for h in hs]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    stagings = [Staging(h["q"], h["k"], h["v"]) for h in hs]
    outs = []
    for it in range(6):
        s = it % 2
        h = hs[s]
        o = torch.empty(h["q"].shape, dtype=h["q"].dtype, pin_memory=True)
        l = torch.empty(h["q"].shape[:-1], dtype=torch.float32, pin_memory=True)
        fwd(h["q"], h["k"], h["v"], causal=True, scale=ws[0].scale, out=o, lse=l, staging=stagings[s],
            stream=streams[s], sync=False)
        outs.append((s, o, l))
    torch.cuda.synchronize()
    assert last_device_status() == 0
    for s, o, l in outs:
        assert torch.equal(o, ref[s][0]) and torch.equal(l, ref[s][1])


def test_host_path_with_padded_bias_rows():
    """A bias whose rows are padded for alignment (N=300) keeps its strides through staging."""
    w = Workload("hb", B=2, H=3, N=300, d=32, dtype="bf16", causal=False, seed=53, bias=True, gate=True)
    inp = make_inputs(w)
    n = w.N
    buf = torch.zeros(w.H, n, (n + 7) // 8 * 8, dtype=inp["bias"].dtype, pin_memory=True)
    buf[..., :n] = inp["bias"]
    bp = buf[..., :n]                      # pinned, rows 304 elements apart
    assert bp.stride(1) == 304
    h = _pinned({k: inp[k] for k in ("q", "k", "v", "gate")})
    o, l = fwd(h["q"], h["k"], h["v"], bias=bp, gate=h["gate"], scale=w.scale)
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], bias=inp["bias"], gate=inp["gate"], scale=w.scale)
    assert_close_to_oracle(o, l, o_ref, l_ref, w.torch_dtype, "host-padded-bias")
