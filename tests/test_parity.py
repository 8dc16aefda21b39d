"""GPU parity: the fused sm_100a kernel against the fp64 oracle on the same
seeded inputs (element by element), through the C ABI."""
import numpy as np
import pytest
import torch

from exact_attention_sdpa_b200 import attn_fwd, last_device_status
from exact_attention_sdpa_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import sdpa_forward, sdpa_rows
from helpers import assert_close_to_oracle, padded

pytestmark = pytest.mark.gpu


def _run(inp, w: Workload, scale=None):
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    bias = None if inp["bias"] is None else padded(inp["bias"], dev)
    gate = None if inp["gate"] is None else inp["gate"].to(dev)
    o, lse = attn_fwd(q, k, v, bias=bias, gate=gate, causal=w.causal, scale=w.scale if scale is None else scale)
    torch.cuda.synchronize()
    assert last_device_status() == 0, "a bounded device wait timed out"
    return o, lse


def _full_check(w: Workload, seed=None):
    inp = make_inputs(w, seed)
    o, lse = _run(inp, w)
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], bias=inp["bias"], gate=inp["gate"],
                                causal=w.causal, scale=w.scale)
    return assert_close_to_oracle(o, lse, o_ref, l_ref, w.torch_dtype, w.name)


@pytest.mark.parametrize("name", ["tiny", "gpt2_small", "evoformer_row"])
def test_workload_full(name):
    _full_check(WORKLOADS[name])


def _sampled_rows(w: Workload, n_bh=4, seed=0):
    """Rows every query tile boundary cares about, plus random ones, for a few (b, h)."""
    rng = np.random.default_rng(seed)
    picks = []
    bhs = [(0, 0), (w.B - 1, w.H - 1)] + [(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(n_bh - 2)]
    special = [0, 1, 127, 128, 129, w.N // 2, w.N - 129, w.N - 128, w.N - 2, w.N - 1]
    for b, h in bhs:
        rows = set(i for i in special if 0 <= i < w.N)
        rows.update(int(x) for x in rng.integers(0, w.N, size=24))
        picks += [(b, h, i) for i in sorted(rows)]
    return picks


@pytest.mark.parametrize("name", ["n8192_causal", "long_wide", "prefill_chunk"])
def test_workload_full_size_sampled(name):
    """Full-size problems in the launch configuration the benchmark times;
    the oracle computes a sample of output rows one by one."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    o, lse = _run(inp, w)
    picks = _sampled_rows(w)
    o_ref, l_ref = sdpa_rows(inp["q"], inp["k"], inp["v"], picks, bias=inp["bias"], gate=inp["gate"],
                             causal=w.causal, scale=w.scale)
    idx = tuple(np.array(x) for x in zip(*picks))
    o_s = o.cpu()[idx]
    l_s = lse.cpu()[idx]
    assert_close_to_oracle(o_s, l_s, o_ref, l_ref, w.torch_dtype, name)
    # every output row (not only the sampled ones) is finite
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    # whole heads, every row and column: the first and last (b, h) of the launch and random
    # others (every head has units in every wave of the persistent schedule)
    n_whole = WHOLE_HEADS.get(name, 0)
    if n_whole:
        rng = np.random.default_rng(1)
        heads = [(0, 0), (w.B - 1, w.H - 1)]
        while len(heads) < n_whole:
            bh = (int(rng.integers(w.B)), int(rng.integers(w.H)))
            if bh not in heads:
                heads.append(bh)
        o_c, l_c = o.cpu(), lse.cpu()
        for b, h in heads:
            sl = (slice(b, b + 1), slice(h, h + 1))
            o_ref, l_ref = sdpa_forward(inp["q"][sl], inp["k"][sl], inp["v"][sl], causal=w.causal, scale=w.scale)
            assert_close_to_oracle(o_c[sl], l_c[sl], o_ref, l_ref, w.torch_dtype, f"{name} head ({b},{h})")


# heads compared in full at the full-size workloads (the oracle takes ~1 s per N=8192 head
# and ~15 s per N=32768 head on a 16-core host)
WHOLE_HEADS = {"n8192_causal": 8, "long_wide": 2, "prefill_chunk": 2}


SWEEP = []
for d in (32, 64, 128):
    for N in (1, 17, 128, 129, 255, 1000):
        for causal in (False, True):
            SWEEP.append((d, N, causal))


@pytest.mark.parametrize("d,N,causal", SWEEP)
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_sweep_ragged(d, N, causal, dtype):
    w = Workload("sweep", B=1, H=3, N=N, d=d, dtype=dtype, causal=causal, seed=100 + d + N)
    _full_check(w)


@pytest.mark.parametrize("bias,gate", [(True, False), (False, True), (True, True)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,N", [(32, 200), (64, 256), (128, 129)])
def test_bias_gate_variants(bias, gate, causal, d, N):
    w = Workload("bg", B=3, H=2, N=N, d=d, dtype="bf16", causal=causal, seed=7 + N, bias=bias, gate=gate)
    _full_check(w)


def test_per_batch_bias_4d():
    w = Workload("b4", B=2, H=3, N=300, d=64, dtype="fp16", causal=False, seed=11)
    inp = make_inputs(w)
    bias = torch.randn(2, 3, 300, 304, generator=torch.Generator().manual_seed(5)).to(torch.float16)[..., :300]
    dev = torch.device("cuda")
    o, lse = attn_fwd(inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev), bias=padded(bias, dev), causal=False,
                      scale=w.scale)
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], bias=bias, scale=w.scale)
    assert_close_to_oracle(o, lse, o_ref, l_ref, torch.float16, "bias4d")


def test_strided_views():
    """Q/K/V as transposed views of [B, N, H, d] buffers; O written into a strided view."""
    B, H, N, d = 2, 4, 333, 64
    g = torch.Generator().manual_seed(3)
    mk = lambda: torch.randn(B, N, H, d, generator=g).to(torch.bfloat16)
    qb, kb, vb = mk(), mk(), mk()
    dev = torch.device("cuda")
    q, k, v = (x.to(dev).transpose(1, 2) for x in (qb, kb, vb))
    out_buf = torch.zeros(B, N, H, d, device=dev, dtype=torch.bfloat16)
    out = out_buf.transpose(1, 2)
    _, lse = attn_fwd(q, k, v, causal=True, out=out)
    torch.cuda.synchronize()
    o_ref, l_ref = sdpa_forward(qb.transpose(1, 2), kb.transpose(1, 2), vb.transpose(1, 2), causal=True)
    assert_close_to_oracle(out_buf.transpose(1, 2), lse, o_ref, l_ref, torch.bfloat16, "strided")


def test_same_storage_in_two_layouts():
    """One storage read back to back as [B, H, N, d] and as a transposed [B, N, H, d] view: the
    same base pointer and shape with other strides must not reuse the first call's tensor maps."""
    B, H, N, d = 2, 4, 256, 64
    g = torch.Generator().manual_seed(11)
    dev = torch.device("cuda")
    bufs = [torch.randn(B * H * N * d, generator=g).to(torch.float16).to(dev) for _ in range(3)]
    for layout in ("bhnd", "bnhd", "bhnd"):
        if layout == "bhnd":
            q, k, v = (x.view(B, H, N, d) for x in bufs)
        else:
            q, k, v = (x.view(B, N, H, d).transpose(1, 2) for x in bufs)
        o, lse = attn_fwd(q, k, v, causal=True)
        torch.cuda.synchronize()
        o_ref, l_ref = sdpa_forward(q.cpu(), k.cpu(), v.cpu(), causal=True)
        assert_close_to_oracle(o, lse, o_ref, l_ref, torch.float16, f"layout {layout}")


def test_evoformer_column_gated_attention():
    """Column-wise gated self-attention of an Evoformer MSA block (the gated Evoformer variant of
    the FLASHLIGHT summary, along the other axis): the MSA activations are [R, C, H, d] and each
    column attends over its R rows, with a sigmoid gate and no pair bias.  The kernel runs on
    permuted views of the row-major buffers (batch = columns, sequence = rows), no copies."""
    R, C, H, d = 200, 24, 8, 32
    g = torch.Generator().manual_seed(12)
    mk = lambda: torch.randn(R, C, H, d, generator=g).to(torch.bfloat16)
    qb, kb, vb, gb = mk(), mk(), mk(), mk()
    dev = torch.device("cuda")
    col = lambda x: x.permute(1, 2, 0, 3)              # [C, H, R, d]
    q, k, v, gate = (col(x.to(dev)) for x in (qb, kb, vb, gb))
    out_buf = torch.zeros(R, C, H, d, device=dev, dtype=torch.bfloat16)
    _, lse = attn_fwd(q, k, v, gate=gate, causal=False, out=col(out_buf))
    torch.cuda.synchronize()
    assert last_device_status() == 0, "a bounded device wait timed out"
    o_ref, l_ref = sdpa_forward(col(qb), col(kb), col(vb), gate=col(gb))
    assert_close_to_oracle(col(out_buf), lse, o_ref, l_ref, torch.bfloat16, "evoformer column")


@pytest.mark.parametrize("name", ["gpt2_small", "evoformer_row"])
def test_deterministic(name):
    """Repeated launches give bit-identical results (no atomics; any race in the
    barrier protocol between the warp roles shows up here)."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    o1, l1 = _run(inp, w)
    for _ in range(10):
        o2, l2 = _run(inp, w)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_batch_heads_many():
    w = Workload("bh", B=5, H=7, N=160, d=64, dtype="fp16", causal=True, seed=21)
    _full_check(w)


def test_head_grouped_order_with_partial_group():
    """Long sequences whose K/V exceed the L2 are scheduled a few heads at a time;
    9 heads at N=32768 (302 MB of K/V) form groups of 2 and a partial group of 1."""
    w = Workload("grouped", B=1, H=9, N=32768, d=128, dtype="bf16", causal=True, seed=31, amp=0.5)
    inp = make_inputs(w)
    o, lse = _run(inp, w)
    picks = _sampled_rows(w, n_bh=5)
    picks += [(0, h, i) for h in range(9) for i in (0, 255, 256, 16383, 32767)]
    o_ref, l_ref = sdpa_rows(inp["q"], inp["k"], inp["v"], picks, causal=True, scale=w.scale)
    idx = tuple(np.array(x) for x in zip(*picks))
    assert_close_to_oracle(o.cpu()[idx], lse.cpu()[idx], o_ref, l_ref, torch.bfloat16, "grouped")


@pytest.mark.parametrize("B", [8, 13])
def test_several_waves_of_units(B):
    """More 256-row units than CTAs: each CTA takes one unit per wave, alternate waves in
    reverse order.  B=8 (192 units on 148 SMs) ends in a partial reversed wave, B=13
    (312 units) in a partial forward one; every output row is compared."""
    w = Workload("waves", B=B, H=8, N=768, d=64, dtype="fp16", causal=True, seed=40 + B)
    _full_check(w)


@pytest.mark.parametrize("d,dtype,causal", [(64, "fp16", True), (64, "bf16", False), (128, "bf16", True)])
def test_more_than_32_units_per_cta(d, dtype, causal):
    """5120 single-pair units on 148 SMs: every CTA runs 34-35 units, every per-unit counter of
    the barrier protocol wraps its parity many times.  Units are heads here (one 256-row pair
    per head), and the CTAs' 33rd and later units are heads 4736 and up: those are compared in
    full, with a sample of the others."""
    w = Workload("units", B=128, H=40, N=256, d=d, dtype=dtype, causal=causal, seed=60 + d)
    inp = make_inputs(w)
    o, lse = _run(inp, w)
    BH = w.B * w.H
    rng = np.random.default_rng(7)
    sel = sorted(set(range(4736, BH)) | set(int(x) for x in rng.integers(0, 4736, size=64)))
    flat = lambda t: t.reshape(BH, *t.shape[2:])
    q, k, v = (flat(inp[n])[sel].unsqueeze(0) for n in "qkv")
    o_ref, l_ref = sdpa_forward(q, k, v, causal=causal, scale=w.scale)
    assert_close_to_oracle(flat(o.cpu())[sel].unsqueeze(0), flat(lse.cpu())[sel].unsqueeze(0), o_ref, l_ref,
                           w.torch_dtype, f"units d={d}")


RECT = [  # (N query rows, Nk key rows, causal, d, dtype, bias, gate)
    (128, 1024, True, 64, "fp16", False, False),      # prefill chunk against a KV cache
    (1, 777, True, 128, "bf16", False, False),        # decode step
    (3, 300, True, 64, "fp16", False, False),         # a few decode rows, ragged key tail
    (300, 100, True, 64, "bf16", False, False),       # more queries than keys: 200 dead rows
    (640, 2048, True, 64, "fp16", False, False),      # two and a half query pairs, offset 1408
    (200, 513, False, 32, "bf16", True, True),        # non-causal with pair bias and gate
    (257, 645, True, 32, "bf16", True, False),        # causal with bias, offset 388 (not a tile multiple)
    (1000, 300, False, 128, "bf16", False, False),    # non-causal, Nq > Nk
    (384, 500, True, 128, "fp16", True, True),        # d=128 bias path (global loads), offset 116
]


@pytest.mark.parametrize("N,Nk,causal,d,dtype,bias,gate", RECT)
def test_rectangular_q_and_kv(N, Nk, causal, d, dtype, bias, gate):
    """Nq != Nk: causal masking is aligned at the bottom right (query i sees keys
    j <= i + Nk - Nq); every output row is compared with the oracle."""
    w = Workload("rect", B=2, H=3, N=N, d=d, dtype=dtype, causal=causal, seed=60 + N % 17, Nk=Nk,
                 bias=bias, gate=gate)
    inp = make_inputs(w)
    o, lse = _run(inp, w)
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], bias=inp["bias"], gate=inp["gate"],
                                causal=causal, scale=w.scale)
    assert_close_to_oracle(o, lse, o_ref, l_ref, w.torch_dtype, f"rect{N}x{Nk}")
    if causal and N > Nk:
        dead = N - Nk
        assert torch.all(o[:, :, :dead] == 0)
        assert torch.all(torch.isneginf(lse[:, :, :dead]))
