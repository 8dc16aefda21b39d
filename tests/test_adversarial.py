"""GPU edge cases the online softmax must survive: scores that force a rescale
on every tile, huge magnitudes, -inf biases, one dominant key, identical value
rows, scale 0 (a closed form), and fully masked rows."""
import math

import pytest
import torch

from exact_attention_sdpa_b200 import attn_fwd, last_device_status
from oracle import sdpa_forward
from helpers import assert_close_to_oracle, padded

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda") if torch.cuda.is_available() else None


def _gen(shape, seed, dtype, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(dtype)


def _check(q, k, v, bias=None, gate=None, causal=False, scale=None, what=""):
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), None if bias is None else padded(bias, DEV),
                      None if gate is None else gate.to(DEV), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert last_device_status() == 0, "a bounded device wait timed out"
    o_ref, l_ref = sdpa_forward(q, k, v, bias=bias, gate=gate, causal=causal, scale=scale)
    assert_close_to_oracle(o, lse, o_ref, l_ref, q.dtype, what)
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_large_magnitude_scores(dtype):
    # scale x20: score spreads of hundreds, many max changes
    s = (1, 2, 700, 64)
    _check(_gen(s, 1, dtype), _gen(s, 2, dtype), _gen(s, 3, dtype), scale=20.0 / 8.0, what="large")


def test_monotone_scores_rescale_every_tile():
    # q = 1-vector, k_j grows with j: the row max increases on every key tile
    B, H, N, d = 1, 2, 1024, 64
    q = torch.full((B, H, N, d), 0.25, dtype=torch.float16)
    ramp = torch.linspace(-2, 2, N).view(1, 1, N, 1).expand(B, H, N, d)
    k = ramp.to(torch.float16).contiguous()
    v = _gen((B, H, N, d), 4, torch.float16)
    _check(q, k, v, scale=1.0, what="monotone")
    _check(q, k, v, causal=True, scale=1.0, what="monotone-causal")


def test_neg_inf_bias_all_but_one_key():
    B, H, N, d = 2, 2, 300, 32
    q, k, v = (_gen((B, H, N, d), 10 + i, torch.bfloat16) for i in range(3))
    bias = torch.full((H, N, N), float("-inf"))
    keep = torch.randint(0, N, (H, N), generator=torch.Generator().manual_seed(0))
    bias.scatter_(2, keep.unsqueeze(-1), 0.0)
    bias = bias.to(torch.bfloat16)
    o, lse = _check(q, k, v, bias=bias, what="one-key")
    # one visible key: O equals that value row exactly up to the output rounding
    vv = v.float()
    for h in range(H):
        expect = vv[:, h, keep[h]]                  # [B, N, d]
        assert torch.allclose(o[:, h].float(), expect, atol=1e-2)


def test_fully_masked_rows():
    B, H, N, d = 1, 1, 200, 64
    q, k, v = (_gen((B, H, N, d), 20 + i, torch.float16) for i in range(3))
    bias = torch.zeros(H, N, N)
    bias[0, 5, :] = float("-inf")
    bias[0, 150, :] = float("-inf")
    bias = bias.to(torch.float16)
    o, lse = _check(q, k, v, bias=bias, what="masked rows")
    assert torch.all(o[0, 0, 5] == 0) and torch.all(o[0, 0, 150] == 0)
    assert lse[0, 0, 5] == float("-inf") and lse[0, 0, 150] == float("-inf")


def test_single_dominant_key():
    B, H, N, d = 1, 2, 513, 128
    q, k, v = (_gen((B, H, N, d), 30 + i, torch.bfloat16) for i in range(3))
    bias = torch.zeros(H, N, N)
    bias[:, :, 400] = 60.0
    o, _ = _check(q, k, v, bias=bias.to(torch.bfloat16), what="dominant")
    assert torch.allclose(o[0, :, :].float(), v[0, :, 400:401].float().expand(H, N, d), atol=2e-2)


def test_identical_value_rows():
    B, H, N, d = 2, 3, 257, 64
    q, k = (_gen((B, H, N, d), 40 + i, torch.float16, 3.0) for i in range(2))
    u = _gen((d,), 42, torch.float16)
    v = u.view(1, 1, 1, d).expand(B, H, N, d).contiguous()
    for causal in (False, True):
        o, _ = _check(q, k, v, causal=causal, what="identical-v")
        assert torch.allclose(o.float(), u.float().expand(B, H, N, d), atol=5e-3)


def test_scale_zero_closed_form():
    B, H, N, d = 1, 2, 384, 64
    q, k, v = (_gen((B, H, N, d), 50 + i, torch.float16) for i in range(3))
    o, lse = _check(q, k, v, causal=True, scale=0.0, what="scale0")
    cm = torch.cumsum(v.double(), 2) / torch.arange(1, N + 1).view(1, 1, N, 1)
    assert torch.allclose(o.double(), cm, atol=5e-3)
    assert torch.allclose(lse.double(), torch.log(torch.arange(1, N + 1).double()).expand(B, H, N), atol=1e-3)


def test_causal_row_zero_returns_v0():
    B, H, N, d = 2, 2, 640, 128
    q, k, v = (_gen((B, H, N, d), 60 + i, torch.bfloat16) for i in range(3))
    o, _ = _check(q, k, v, causal=True, what="row0")
    assert torch.equal(o[:, :, 0], v[:, :, 0])
