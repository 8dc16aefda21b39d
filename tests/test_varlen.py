"""GPU parity of ragged batches (attn_fwd_varlen) against the oracle's
sdpa_varlen_forward, every output row, on seeded packed inputs."""
import pytest
import torch

from exact_attention_sdpa_b200 import attn_fwd_varlen, last_device_status
from exact_attention_sdpa_b200.workloads import WORKLOADS, make_varlen_inputs
from oracle import sdpa_varlen_forward
from helpers import assert_close_to_oracle

pytestmark = pytest.mark.gpu

CASES = [  # per-sequence (query, key) lengths, d, causal, dtype
    ([(100, 100), (0, 0), (257, 257), (1, 1), (700, 700)], 64, True, "fp16"),
    ([(128, 1024), (3, 300), (0, 50), (640, 2048)], 64, True, "bf16"),         # prefill chunks and decode rows
    ([(333, 333), (129, 400), (64, 64)], 128, False, "bf16"),
    ([(500, 200), (257, 600)], 32, True, "fp16"),                               # a sequence with dead rows
]


def _packed(lens, H, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    Tq, Tk = sum(a for a, _ in lens), sum(b for _, b in lens)
    mk = lambda T: torch.randn(T, H, d, generator=g).to(dtype)
    cq = torch.tensor([0] + list(torch.cumsum(torch.tensor([a for a, _ in lens]), 0)), dtype=torch.int32)
    ck = torch.tensor([0] + list(torch.cumsum(torch.tensor([b for _, b in lens]), 0)), dtype=torch.int32)
    return mk(Tq), mk(Tk), mk(Tk), cq, ck


@pytest.mark.parametrize("lens,d,causal,dtype", CASES)
def test_varlen_matches_oracle(lens, d, causal, dtype):
    dt = {"fp16": torch.float16, "bf16": torch.bfloat16}[dtype]
    q, k, v, cq, ck = _packed(lens, 3, d, dt, seed=90 + d)
    dev = torch.device("cuda")
    o, lse = attn_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), cq, ck, causal=causal)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    o_ref, l_ref = sdpa_varlen_forward(q, k, v, cq.tolist(), ck.tolist(), causal=causal)
    assert_close_to_oracle(o, lse, o_ref, l_ref, dt, f"varlen d={d}")


def test_varlen_workload_sampled():
    """The benchmarked ragged workload, every row of three of its sequences."""
    w = WORKLOADS["varlen_mix"]
    inp = make_varlen_inputs(w)
    dev = torch.device("cuda")
    cu = inp["cu_seqlens"]
    o, lse = attn_fwd_varlen(inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev), cu, cu, causal=True)
    torch.cuda.synchronize()
    for b in (1, 4, 12):
        r0, r1 = int(cu[b]), int(cu[b + 1])
        sub = [0, r1 - r0]
        o_ref, l_ref = sdpa_varlen_forward(inp["q"][r0:r1], inp["k"][r0:r1], inp["v"][r0:r1], sub, sub, causal=True)
        assert_close_to_oracle(o[r0:r1], lse[:, r0:r1], o_ref, l_ref, w.torch_dtype, f"varlen_mix seq {b}")


def test_varlen_more_sequences_than_one_launch_holds():
    """70 sequences: two launches of the fused kernel (64 sequences travel in one launch's
    parameters), lengths from 1 to 600 with a few empty ones; every row compared."""
    rng = torch.Generator().manual_seed(7)
    lens = []
    for i in range(70):
        n = int(torch.randint(1, 600, (1,), generator=rng))
        lens.append((0, 0) if i % 23 == 5 else (n, n))
    q, k, v, cq, ck = _packed(lens, 2, 64, torch.float16, seed=71)
    dev = torch.device("cuda")
    o, lse = attn_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), cq, ck, causal=True)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    o_ref, l_ref = sdpa_varlen_forward(q, k, v, cq.tolist(), ck.tolist(), causal=True)
    assert_close_to_oracle(o, lse, o_ref, l_ref, torch.float16, "varlen 70 sequences")


def test_varlen_single_sequence_equals_plain_forward():
    from exact_attention_sdpa_b200 import attn_fwd
    q, k, v, cq, ck = _packed([(777, 777)], 3, 128, torch.bfloat16, seed=72)
    dev = torch.device("cuda")
    o, lse = attn_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), cq, ck, causal=True)
    as4 = lambda x: x.to(dev).transpose(0, 1).unsqueeze(0)
    o4, lse4 = attn_fwd(as4(q), as4(k), as4(v), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o4[0].transpose(0, 1)) and torch.equal(lse, lse4[0])
