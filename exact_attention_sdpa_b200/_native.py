"""ctypes binding of libattn.so (argument marshalling only).

Every step of the attention forward runs in the library's CUDA kernel; this
module converts torch tensors into the C ABI's ``attn_tensor_t`` views, passes
the current CUDA stream and turns status codes into exceptions.  There is no
fallback: if the shared library is missing the call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn.so")

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT = range(5)
ATTN_F16, ATTN_BF16, ATTN_F32 = 0, 1, 2

# every function include/attn.h declares
EXPORTED = ("attn_fwd", "attn_status_string", "attn_last_device_status", "attn_set_wait_limit",
            "attn_debug_inject_stall", "attn_version")


class AttnTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class AttnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"attn status {code}: {msg}")
        self.code = code


_lib = None
_lock = threading.Lock()


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads libattn.so (once).  Raises RuntimeError if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with `python -m exact_attention_sdpa_b200.build` "
                               "(there is no fallback implementation)")
        lib = ctypes.CDLL(p)
        P = ctypes.POINTER(AttnTensor)
        lib.attn_fwd.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_float, P, ctypes.c_void_p, ctypes.c_void_p]
        lib.attn_fwd.restype = ctypes.c_int
        lib.attn_status_string.argtypes = [ctypes.c_int]
        lib.attn_status_string.restype = ctypes.c_char_p
        lib.attn_last_device_status.argtypes = [ctypes.c_void_p]
        lib.attn_last_device_status.restype = ctypes.c_int
        lib.attn_set_wait_limit.argtypes = [ctypes.c_uint64]
        lib.attn_set_wait_limit.restype = None
        lib.attn_debug_inject_stall.argtypes = [ctypes.c_int]
        lib.attn_debug_inject_stall.restype = None
        lib.attn_version.argtypes = []
        lib.attn_version.restype = ctypes.c_char_p
        if path is None:
            _lib = lib
        return lib


def status_string(code: int) -> str:
    return load_library().attn_status_string(code).decode()


def _check(code: int):
    if code != ATTN_OK:
        raise AttnError(code, status_string(code))


_DT = {torch.float16: ATTN_F16, torch.bfloat16: ATTN_BF16, torch.float32: ATTN_F32}


def make_view(t: Optional[torch.Tensor]) -> Optional[AttnTensor]:
    """An attn_tensor_t describing ``t`` (no copy).  Unknown dtypes map to an invalid code."""
    if t is None:
        return None
    if t.dim() > 4:
        raise ValueError("attn tensors have at most 4 dimensions")
    v = AttnTensor()
    v.data = t.data_ptr() if t.numel() > 0 else 0
    v.dtype = _DT.get(t.dtype, 99)
    v.ndim = t.dim()
    for i in range(t.dim()):
        v.shape[i] = t.shape[i]
        v.stride[i] = t.stride(i)
    return v


def _ref(view: Optional[AttnTensor]):
    return None if view is None else ctypes.byref(view)


def attn_fwd_raw(q, k, v, bias, gate, causal: bool, scale: float, out, lse, stream: int) -> int:
    """Direct call of the C entry point with torch tensors; returns the status code."""
    lib = load_library()
    vq, vk, vv, vb, vg, vo = (make_view(t) for t in (q, k, v, bias, gate, out))
    lse_ptr = None if lse is None else lse.data_ptr()
    return lib.attn_fwd(_ref(vq), _ref(vk), _ref(vv), _ref(vb), _ref(vg), int(bool(causal)), float(scale),
                        _ref(vo), lse_ptr, stream)


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, bias: Optional[torch.Tensor] = None,
             gate: Optional[torch.Tensor] = None, causal: bool = False, scale: Optional[float] = None,
             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """O = softmax(scale * Q K^T [+ bias]) V [* sigmoid(gate)] and the per-row logsumexp.

    q, k, v: CUDA tensors [B, H, N, d] (fp16 or bf16, d in {32, 64, 128}, last
    dim contiguous).  bias: [H, N, N] or [B, H, N, N]; gate: like q.  ``scale``
    defaults to 1/sqrt(d).  ``out``/``lse`` may be given preallocated.  The
    launch goes on ``stream`` (default: the current stream) and is asynchronous.
    """
    if not q.is_cuda:
        raise ValueError("attn_fwd takes CUDA tensors; use fwd() for host tensors")
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty(q.shape[:-1], device=q.device, dtype=torch.float32)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(attn_fwd_raw(q, k, v, bias, gate, causal, scale, out, lse, s))
    return out, lse


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, bias: Optional[torch.Tensor] = None,
        gate: Optional[torch.Tensor] = None, causal: bool = False, scale: Optional[float] = None,
        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
        device: Optional[torch.device] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The end-to-end call: host (ideally pinned) tensors in, host tensors out.

    Copies the inputs to ``device`` (default: the current CUDA device), runs
    the fused kernel, copies O and lse back into ``out``/``lse`` (pinned host
    tensors, allocated when not given) and waits for them.  Device tensors are
    accepted too; then nothing is staged and the device results are returned.
    """
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if q.is_cuda:
        return attn_fwd(q, k, v, bias, gate, causal, scale, out, lse)

    def stage(t):
        return None if t is None else t.to(dev, non_blocking=True)

    o, l = attn_fwd(stage(q), stage(k), stage(v), stage(bias), stage(gate), causal, scale)
    if out is None:
        out = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    if lse is None:
        lse = torch.empty(l.shape, dtype=l.dtype, pin_memory=True)
    out.copy_(o, non_blocking=True)
    lse.copy_(l, non_blocking=True)
    torch.cuda.current_stream(dev).synchronize()
    return out, lse


def last_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    s = (stream or torch.cuda.current_stream()).cuda_stream
    return load_library().attn_last_device_status(s)


def set_wait_limit(cycles: int):
    load_library().attn_set_wait_limit(int(cycles))


def debug_inject_stall(enable: bool):
    """Test hook: later launches time out on purpose (see include/attn.h)."""
    load_library().attn_debug_inject_stall(int(bool(enable)))


def version() -> str:
    return load_library().attn_version().decode()
