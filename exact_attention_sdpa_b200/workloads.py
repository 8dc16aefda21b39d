"""Seeded synthetic inputs for the attention forward.

This module only draws random numbers and fixes shapes; it holds none of the
attention arithmetic, so both the CUDA path and the fp64 oracle can consume
exactly the same input bits from it.

Recipe (identical for every workload): a CPU ``torch.Generator`` seeded with
the workload's seed draws fp32 standard-normal tensors in the fixed order
q, k, v, bias, gate; each is multiplied by the workload's amplitude (a power
of two, so the product is exact) and rounded to nearest-even into the
workload's dtype.  Shapes follow the problem statement of the pages: Q, K, V
and O are [B, H, N, d] with d contiguous (inskillml Module 9, the
``scaled_dot_product_attention`` example), the Evoformer-style pair bias is
[H, N, N] shared across the R rows that play the role of B, and the gate has
O's shape (gist.science FLASHLIGHT summary, the gated row/column Evoformer
variant).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_e4m3_inputs", "make_grad_output", "make_varlen_inputs",
           "alibi_slopes", "attention_flops", "algorithmic_bytes", "exponential_count"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str          # "fp16" | "bf16"
    causal: bool
    seed: int
    amp: float = 1.0    # inputs are amp * N(0,1); a power of two keeps it exact
    bias: bool = False  # additive pair bias [H, N, N], shared over B
    gate: bool = False  # O <- sigmoid(G) * O, G has O's shape
    description: str = ""
    Nk: Optional[int] = None   # key rows when they differ from the N query rows (KV-cache shapes)
    softcap: float = 0.0       # score modifications (0 / False / -1: off)
    alibi: bool = False        # per-head slopes 2^(-8 (h+1) / H), see alibi_slopes()
    window_left: int = -1
    lengths: Optional[tuple] = None   # ragged batch: per-sequence token counts (B = len, N = max)

    @property
    def n_keys(self) -> int:
        """Key rows: Nk when given, else N."""
        return self.N if self.Nk is None else self.Nk

    @property
    def scale(self) -> float:
        # 1/sqrt(d_k), aiinarabic.com "flash-attention", Equation (1)
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self) -> torch.dtype:
        """The torch dtype of the 16-bit inputs and outputs."""
        return {"fp16": torch.float16, "bf16": torch.bfloat16}[self.dtype]

    def with_(self, **kw) -> "Workload":
        """A copy with the given fields replaced."""
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", B=1, H=2, N=256, d=64, dtype="bf16", causal=False, seed=0,
                 description="tiny SDPA forward, B=1 H=2 N=256 d=64 bf16, non-causal"),
        Workload("gpt2_small", B=4, H=12, N=1024, d=64, dtype="fp16", causal=True, seed=1,
                 description="GPT-2-small-shaped attention, B=4 H=12 N=1024 d=64 fp16, causal"),
        Workload("n8192_causal", B=4, H=12, N=8192, d=64, dtype="fp16", causal=True, seed=2,
                 description="the inskillml Module 9 worked sizing, B=4 H=12 N=8192 d=64 fp16, causal"),
        Workload("long_wide", B=1, H=32, N=32768, d=128, dtype="bf16", causal=True, seed=3, amp=0.5,
                 description="long-context wide-head attention, B=1 H=32 N=32768 d=128 bf16 (x0.5), causal"),
        Workload("evoformer_row", B=256, H=8, N=256, d=32, dtype="bf16", causal=False, seed=4,
                 bias=True, gate=True,
                 description="Evoformer-style gated row attention, R=256 H=8 N=256 d=32 bf16, "
                             "pair bias [H,N,N], sigmoid gate"),
        Workload("n8192_alibi_softcap", B=4, H=12, N=8192, d=64, dtype="fp16", causal=True, seed=6,
                 softcap=30.0, alibi=True,
                 description="the B=4 H=12 N=8192 d=64 fp16 causal sizing with ALiBi slopes and a logit "
                             "softcap of 30"),
        Workload("varlen_mix", B=16, H=12, N=4096, d=64, dtype="fp16", causal=True, seed=7,
                 lengths=(3072, 512, 1911, 4096, 256, 2600, 1024, 3333, 768, 1500, 4000, 2048, 300, 2900, 1200, 3600),
                 description="a ragged batch of 16 sequences of 256-4096 tokens (36,920 in all), H=12 d=64 "
                             "fp16, causal, packed along the token axis"),
        Workload("n8192_window", B=4, H=12, N=8192, d=64, dtype="fp16", causal=True, seed=8, window_left=1023,
                 description="the B=4 H=12 N=8192 d=64 fp16 causal sizing with a left (sliding) window of "
                             "1024 keys per query"),
        Workload("prefill_chunk", B=8, H=12, N=2048, d=64, dtype="fp16", causal=True, seed=5, Nk=8192,
                 description="a 2048-row prefill chunk against an 8192-row KV cache, B=8 H=12 d=64 fp16, "
                             "causal (bottom-right aligned)"),
    ]
}


def make_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Draw the workload's inputs on the CPU (see the module docstring for the recipe).

    Returns a dict with keys q, k, v, bias, gate (bias/gate are None when the
    workload has none).  Tensors are contiguous CPU tensors in the workload's
    dtype; callers copy them to the device themselves.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.N, w.d)
    kv_shape = (w.B, w.H, w.n_keys, w.d)
    dt = w.torch_dtype

    def draw(*s):
        x = torch.randn(*s, generator=g, dtype=torch.float32)
        if w.amp != 1.0:
            x.mul_(w.amp)
        return x.to(dt)

    q = draw(*shape)
    k = draw(*kv_shape)
    v = draw(*kv_shape)
    bias = draw(w.H, w.N, w.n_keys) if w.bias else None
    gate = draw(*shape) if w.gate else None
    return {"q": q, "k": k, "v": v, "bias": bias, "gate": gate}


def make_e4m3_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, object]:
    """Inputs for the FP8 forward: q, k, v as e4m3 codes (torch.float8_e4m3fn, CPU) with one
    power-of-two scale per tensor.

    The fp32 draws are those of make_inputs (same generator, same order q, k, v, times amp).
    Each tensor's scale is the smallest power of two s with max|x| / s <= 448 (the largest e4m3
    value), so x / s is exact and torch's round-to-nearest conversion to e4m3 never saturates;
    element c of the codes stands for c * s.  Returns q, k, v and q_scale, k_scale, v_scale.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    out: Dict[str, object] = {}
    for name, n in (("q", w.N), ("k", w.n_keys), ("v", w.n_keys)):
        x = torch.randn(w.B, w.H, n, w.d, generator=g, dtype=torch.float32)
        if w.amp != 1.0:
            x.mul_(w.amp)
        amax = float(x.abs().max())
        s = 2.0 ** math.ceil(math.log2(amax / 448.0)) if amax > 0 else 1.0
        out[name] = (x / s).to(torch.float8_e4m3fn)
        out[name + "_scale"] = s
    return out


def make_varlen_inputs(w: Workload, seed: Optional[int] = None):
    """Packed inputs of a ragged workload: q, k, v [T, H, d] (T = sum of lengths) drawn as
    make_inputs does, and the host int32 offsets cu_seqlens (batch + 1 entries)."""
    assert w.lengths is not None
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    T = sum(w.lengths)

    def draw():
        x = torch.randn(T, w.H, w.d, generator=g, dtype=torch.float32)
        if w.amp != 1.0:
            x.mul_(w.amp)
        return x.to(w.torch_dtype)

    q, k, v = draw(), draw(), draw()
    cu = torch.zeros(len(w.lengths) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(w.lengths, dtype=torch.int64), 0).to(torch.int32)
    return {"q": q, "k": k, "v": v, "cu_seqlens": cu}


def attention_flops(w: Workload) -> float:
    """The metric's FLOP count: 4*B*H*N^2*d, halved for causal (square problems).  With
    Nk keys: 4*B*H*d times the number of visible (query, key) pairs, N*Nk without causal
    masking, and with it the pairs j <= i + (Nk - N) (N*Nk - N*(N-1)/2 when N <= Nk).
    With a left window w >= 0 (keys j >= i + (Nk - N) - w): the visible pairs, counted exactly."""
    if w.window_left is not None and w.window_left >= 0 and w.lengths is None:
        n, nk = w.N, w.n_keys
        off = nk - n
        pairs = 0
        for i in range(n):
            hi = min(nk - 1, i + off) if w.causal else nk - 1
            lo = max(0, i + off - w.window_left)
            pairs += max(0, hi - lo + 1)
        return 4.0 * w.B * w.H * w.d * pairs
    if w.lengths is not None:
        f = sum(4.0 * w.H * n * n * w.d for n in w.lengths)
        return f / 2.0 if w.causal else f
    if w.Nk is None:
        f = 4.0 * w.B * w.H * w.N * w.N * w.d
        return f / 2.0 if w.causal else f
    n, nk = w.N, w.Nk
    if not w.causal:
        pairs = n * nk
    else:
        off = nk - n
        pairs = sum(min(nk, max(0, i + off + 1)) for i in range(n))
    return 4.0 * w.B * w.H * w.d * pairs


def exponential_count(w: Workload) -> float:
    """Exponentials the method must evaluate at least once: one per visible (query, key) pair
    (the softmax weights) plus one per output element when a sigmoid gate is applied."""
    pairs = attention_flops(w) / (4.0 * w.d)
    if w.lengths is not None:
        rows = sum(w.lengths) * w.H
    else:
        rows = w.B * w.H * w.N
    return pairs + (rows * w.d if w.gate else 0.0)


def algorithmic_bytes(w: Workload) -> int:
    """Bytes one forward must move at least once: Q, K, V (and G, bias) read, O and lse written."""
    elem = 2
    if w.lengths is not None:                     # q, k, v, o of every token, lse
        T = sum(w.lengths)
        return 4 * T * w.H * w.d * elem + T * w.H * 4
    per_q = w.B * w.H * w.N * w.d * elem
    per_kv = w.B * w.H * w.n_keys * w.d * elem
    per_tensor = per_q
    n_tensors = 2 + (1 if w.gate else 0)          # q, o (+ gate); k, v below
    bias = w.H * w.N * w.n_keys * elem if w.bias else 0
    lse = w.B * w.H * w.N * 4
    return n_tensors * per_tensor + 2 * per_kv + bias + lse


def make_grad_output(w: Workload, seed: Optional[int] = None) -> torch.Tensor:
    """An upstream gradient dO for the backward: N(0,1) of O's shape in the workload's
    dtype, from its own generator (seed + 1000 by default) so that the forward inputs
    are the same bits with or without it."""
    g = torch.Generator(device="cpu")
    g.manual_seed((w.seed if seed is None else seed) + 1000)
    return torch.randn(w.B, w.H, w.N, w.d, generator=g, dtype=torch.float32).to(w.torch_dtype)


def alibi_slopes(w: Workload) -> Optional[torch.Tensor]:
    """The workload's ALiBi slopes (fp32 [H], the usual geometric 2^(-8 (h+1) / H)), or None."""
    if not w.alibi:
        return None
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / w.H) for h in range(w.H)], dtype=torch.float32)
