"""ctypes binding of libattn.so (argument marshalling only).

Every step of the attention forward and backward runs in the library's CUDA
kernels; this module converts torch tensors into the C ABI's ``attn_tensor_t``
views, passes the current CUDA stream and turns status codes into exceptions.
There is no fallback: if the shared library is missing the call raises.
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

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT, ATTN_ERR_CHECK = range(6)
ATTN_BUILD_DEBUG_CHECKS = 1
DEBUG_LIB_PATH = os.path.join(_PKG, "libattn_debug.so")
ATTN_F16, ATTN_BF16, ATTN_F32, ATTN_E4M3 = 0, 1, 2, 3

# every function include/attn.h declares
EXPORTED = ("attn_fwd", "attn_fwd_ex", "attn_fwd_varlen", "attn_fwd_host", "attn_fwd_host_ex", "attn_fwd_fp8", "attn_bwd", "attn_bwd_ex", "attn_status_string", "attn_last_device_status", "attn_set_wait_limit",
            "attn_debug_inject_stall", "attn_debug_exp2", "attn_build_flags", "attn_version")


class AttnTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class AttnMods(ctypes.Structure):
    _fields_ = [("alibi_slopes", ctypes.c_void_p), ("softcap", ctypes.c_float), ("window_left", ctypes.c_int32)]


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
        lib.attn_fwd_ex.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_float, ctypes.POINTER(AttnMods), P,
                                    ctypes.c_void_p, ctypes.c_void_p]
        lib.attn_fwd_ex.restype = ctypes.c_int
        lib.attn_fwd_varlen.argtypes = [P, P, P, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int,
                                        ctypes.c_float, P, ctypes.c_void_p, ctypes.c_void_p]
        lib.attn_fwd_varlen.restype = ctypes.c_int
        lib.attn_fwd_host.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_float, P, ctypes.c_void_p,
                                      P, P, P, P, P, P, ctypes.c_void_p, ctypes.c_void_p]
        lib.attn_fwd_host.restype = ctypes.c_int
        lib.attn_fwd_host_ex.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_float, ctypes.POINTER(AttnMods), P,
                                         ctypes.c_void_p, P, P, P, P, P, P, ctypes.c_void_p, ctypes.c_void_p]
        lib.attn_fwd_host_ex.restype = ctypes.c_int
        lib.attn_fwd_fp8.argtypes = [P, P, P, ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                     ctypes.c_float, P, ctypes.c_void_p, ctypes.c_void_p]
        lib.attn_fwd_fp8.restype = ctypes.c_int
        lib.attn_bwd.argtypes = [P, P, P, P, ctypes.c_void_p, P, ctypes.c_int, ctypes.c_float, P, P, P,
                                 ctypes.c_void_p]
        lib.attn_bwd.restype = ctypes.c_int
        lib.attn_bwd_ex.argtypes = [P, P, P, P, ctypes.c_void_p, P, ctypes.c_int, ctypes.c_float,
                                    ctypes.POINTER(AttnMods), P, P, P, ctypes.c_void_p]
        lib.attn_bwd_ex.restype = ctypes.c_int
        lib.attn_status_string.argtypes = [ctypes.c_int]
        lib.attn_status_string.restype = ctypes.c_char_p
        lib.attn_last_device_status.argtypes = [ctypes.c_void_p]
        lib.attn_last_device_status.restype = ctypes.c_int
        lib.attn_set_wait_limit.argtypes = [ctypes.c_uint64]
        lib.attn_set_wait_limit.restype = None
        lib.attn_debug_inject_stall.argtypes = [ctypes.c_int]
        lib.attn_debug_inject_stall.restype = None
        lib.attn_debug_exp2.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                        ctypes.c_void_p]
        lib.attn_debug_exp2.restype = ctypes.c_int
        lib.attn_build_flags.argtypes = []
        lib.attn_build_flags.restype = ctypes.c_int
        lib.attn_version.argtypes = []
        lib.attn_version.restype = ctypes.c_char_p
        if path is None:
            _lib = lib
        return lib


def status_string(code: int) -> str:
    """The library's text for a status code (attn_status_string)."""
    return load_library().attn_status_string(code).decode()


def _check(code: int):
    if code != ATTN_OK:
        raise AttnError(code, status_string(code))


_DT = {torch.float16: ATTN_F16, torch.bfloat16: ATTN_BF16, torch.float32: ATTN_F32,
       torch.float8_e4m3fn: ATTN_E4M3}


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


def attn_fwd_raw(q, k, v, bias, gate, causal: bool, scale: float, out, lse, stream: int,
                 softcap: float = 0.0, alibi_slopes: Optional[torch.Tensor] = None, window_left: int = -1) -> int:
    """Direct call of the C entry point with torch tensors; returns the status code."""
    lib = load_library()
    vq, vk, vv, vb, vg, vo = (make_view(t) for t in (q, k, v, bias, gate, out))
    lse_ptr = None if lse is None else lse.data_ptr()
    if not softcap and alibi_slopes is None and window_left < 0:
        return lib.attn_fwd(_ref(vq), _ref(vk), _ref(vv), _ref(vb), _ref(vg), int(bool(causal)), float(scale),
                            _ref(vo), lse_ptr, stream)
    mods = AttnMods(None if alibi_slopes is None else alibi_slopes.data_ptr(), float(softcap), int(window_left))
    return lib.attn_fwd_ex(_ref(vq), _ref(vk), _ref(vv), _ref(vb), _ref(vg), int(bool(causal)), float(scale),
                           ctypes.byref(mods), _ref(vo), lse_ptr, stream)


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, bias: Optional[torch.Tensor] = None,
             gate: Optional[torch.Tensor] = None, causal: bool = False, scale: Optional[float] = None,
             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None, softcap: float = 0.0,
             alibi_slopes: Optional[torch.Tensor] = None, window_left: int = -1
             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """O = softmax(scale * Q K^T [+ bias]) V [* sigmoid(gate)] and the per-row logsumexp.

    q, k, v: CUDA tensors [B, H, N, d] (fp16 or bf16, d in {32, 64, 128}, last
    dim contiguous).  bias: [H, N, N] or [B, H, N, N]; gate: like q.  ``scale``
    defaults to 1/sqrt(d).  ``out``/``lse`` may be given preallocated.  The
    launch goes on ``stream`` (default: the current stream) and is asynchronous.
    Optional score modifications (include/attn.h, attn_mods_t): ``alibi_slopes``
    (CUDA fp32 [H]), ``softcap`` (> 0), ``window_left`` (>= 0).
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
    _check(attn_fwd_raw(q, k, v, bias, gate, causal, scale, out, lse, s, softcap, alibi_slopes, window_left))
    return out, lse


def attn_fwd_varlen_raw(q, k, v, cu_q, cu_k, causal: bool, scale: float, out, lse, stream: int) -> int:
    """Direct call of attn_fwd_varlen; cu_q, cu_k are host int32 tensors of batch + 1 offsets."""
    lib = load_library()
    vq, vk, vv, vo = (make_view(t) for t in (q, k, v, out))
    return lib.attn_fwd_varlen(_ref(vq), _ref(vk), _ref(vv), cu_q.data_ptr(), cu_k.data_ptr(), int(cu_q.numel() - 1),
                               int(bool(causal)), float(scale), _ref(vo), None if lse is None else lse.data_ptr(), stream)


def attn_fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q, cu_seqlens_k,
                    causal: bool = False, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                    lse: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Ragged batch packed along the token axis: q [Tq, H, d], k, v [Tk, H, d] (CUDA);
    sequence b owns rows cu_seqlens_q[b]..cu_seqlens_q[b+1] of q (cu_seqlens_k for k, v).
    The offsets are read on the host.  Returns O [Tq, H, d] and lse [H, Tq]."""
    if not q.is_cuda:
        raise ValueError("attn_fwd_varlen takes CUDA tensors")
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    cu_q = torch.as_tensor(cu_seqlens_q, dtype=torch.int32).cpu().contiguous()
    cu_k = torch.as_tensor(cu_seqlens_k, dtype=torch.int32).cpu().contiguous()
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty(q.shape[1], q.shape[0], device=q.device, dtype=torch.float32)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(attn_fwd_varlen_raw(q, k, v, cu_q, cu_k, causal, scale, out, lse, s))
    return out, lse


def attn_fwd_fp8_raw(q, k, v_t, q_scale: float, k_scale: float, v_scale: float, causal: bool, scale: float, out,
                     lse, stream: int) -> int:
    """Direct call of attn_fwd_fp8 with torch tensors; returns the status code."""
    lib = load_library()
    vq, vk, vv, vo = (make_view(t) for t in (q, k, v_t, out))
    return lib.attn_fwd_fp8(_ref(vq), _ref(vk), _ref(vv), float(q_scale), float(k_scale), float(v_scale),
                            int(bool(causal)), float(scale), _ref(vo), None if lse is None else lse.data_ptr(), stream)


def attn_fwd_fp8(q: torch.Tensor, k: torch.Tensor, v_t: torch.Tensor, q_scale: float = 1.0, k_scale: float = 1.0,
                 v_scale: float = 1.0, causal: bool = False, scale: Optional[float] = None,
                 out_dtype: torch.dtype = torch.bfloat16, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The forward on e4m3 inputs (include/attn.h, attn_fwd_fp8): q [B, H, N, d], k [B, H, Nk, d]
    and v_t = V transposed [B, H, d, Nk] as CUDA torch.float8_e4m3fn tensors (d in {64, 128}),
    element x meaning x * its tensor's scale.  Returns (out [B, H, N, d] in out_dtype, lse)."""
    if not q.is_cuda:
        raise ValueError("attn_fwd_fp8 takes CUDA tensors")
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if out is None:
        out = torch.empty(q.shape, device=q.device, dtype=out_dtype)
    if lse is None:
        lse = torch.empty(q.shape[:-1], device=q.device, dtype=torch.float32)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(attn_fwd_fp8_raw(q, k, v_t, q_scale, k_scale, v_scale, causal, scale, out, lse, s))
    return out, lse


def attn_bwd_raw(q, k, v, out, lse, dout, causal: bool, scale: float, dq, dk, dv, stream: int,
                 softcap: float = 0.0, alibi_slopes: Optional[torch.Tensor] = None, window_left: int = -1) -> int:
    """Direct call of attn_bwd (attn_bwd_ex when a score modification is on); returns the status code."""
    lib = load_library()
    vq, vk, vv, vo, vdo, vdq, vdk, vdv = (make_view(t) for t in (q, k, v, out, dout, dq, dk, dv))
    lse_p = None if lse is None else lse.data_ptr()
    if softcap != 0.0 or alibi_slopes is not None or window_left >= 0:
        mods = AttnMods(None if alibi_slopes is None else alibi_slopes.data_ptr(), float(softcap), int(window_left))
        return lib.attn_bwd_ex(_ref(vq), _ref(vk), _ref(vv), _ref(vo), lse_p, _ref(vdo), int(bool(causal)),
                               float(scale), ctypes.byref(mods), _ref(vdq), _ref(vdk), _ref(vdv), stream)
    return lib.attn_bwd(_ref(vq), _ref(vk), _ref(vv), _ref(vo), lse_p, _ref(vdo),
                        int(bool(causal)), float(scale), _ref(vdq), _ref(vdk), _ref(vdv), stream)


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
             dout: torch.Tensor, causal: bool = False, scale: Optional[float] = None,
             stream: Optional[torch.cuda.Stream] = None, softcap: float = 0.0,
             alibi_slopes: Optional[torch.Tensor] = None,
             window_left: int = -1) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(dQ, dK, dV) of attn_fwd (no bias or gate) for the upstream gradient ``dout``.

    ``out`` and ``lse`` are attn_fwd's outputs for the same q, k, v, causal, scale and
    score modifications (softcap, alibi_slopes, window_left as in attn_fwd).  CUDA
    tensors; asynchronous on ``stream`` (default: the current one).
    """
    if not q.is_cuda:
        raise ValueError("attn_bwd takes CUDA tensors")
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    dq = torch.empty_like(q, memory_format=torch.contiguous_format)
    dk = torch.empty_like(k, memory_format=torch.contiguous_format)
    dv = torch.empty_like(v, memory_format=torch.contiguous_format)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    _check(attn_bwd_raw(q, k, v, out, lse, dout, causal, scale, dq, dk, dv, s, softcap=softcap,
                        alibi_slopes=alibi_slopes, window_left=window_left))
    return dq, dk, dv


class Staging:
    """Device buffers for one end-to-end problem: the layout of each host tensor
    (dtype, shape, strides) on the device.  Reusing one across calls of the same
    shape avoids an allocation per call; two of them on two streams let one
    call's copies run under the other's kernel."""

    def __init__(self, q, k, v, bias=None, gate=None, device=None):
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)

        def like(t):
            return None if t is None else torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device=dev)

        self.q, self.k, self.v, self.bias, self.gate = (like(t) for t in (q, k, v, bias, gate))
        self.out = like(q if q.is_contiguous() else q.contiguous())
        self.lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)


def attn_fwd_host_raw(q, k, v, bias, gate, causal: bool, scale: float, out, lse, staging: Staging,
                      stream: int, softcap: float = 0.0, alibi_slopes: Optional[torch.Tensor] = None,
                      window_left: int = -1) -> int:
    """Direct call of attn_fwd_host (attn_fwd_host_ex with score modifications): host tensors in
    and out, device staging from ``staging``; ``alibi_slopes`` is a CUDA tensor."""
    lib = load_library()
    hq, hk, hv, hb, hg, ho = (make_view(t) for t in (q, k, v, bias, gate, out))
    dq, dk, dv, db, dg, do = (make_view(t) for t in (staging.q, staging.k, staging.v, staging.bias, staging.gate,
                                                    staging.out))
    lse_h = None if lse is None else lse.data_ptr()
    lse_d = None if lse is None else staging.lse.data_ptr()
    if not softcap and alibi_slopes is None and window_left < 0:
        return lib.attn_fwd_host(_ref(hq), _ref(hk), _ref(hv), _ref(hb), _ref(hg), int(bool(causal)), float(scale),
                                 _ref(ho), lse_h, _ref(dq), _ref(dk), _ref(dv), _ref(db), _ref(dg), _ref(do),
                                 lse_d, stream)
    mods = AttnMods(None if alibi_slopes is None else alibi_slopes.data_ptr(), float(softcap), int(window_left))
    return lib.attn_fwd_host_ex(_ref(hq), _ref(hk), _ref(hv), _ref(hb), _ref(hg), int(bool(causal)), float(scale),
                                ctypes.byref(mods), _ref(ho), lse_h, _ref(dq), _ref(dk), _ref(dv), _ref(db),
                                _ref(dg), _ref(do), lse_d, stream)


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, bias: Optional[torch.Tensor] = None,
        gate: Optional[torch.Tensor] = None, causal: bool = False, scale: Optional[float] = None,
        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
        device: Optional[torch.device] = None, staging: Optional[Staging] = None,
        stream: Optional[torch.cuda.Stream] = None, sync: bool = True, softcap: float = 0.0,
        alibi_slopes: Optional[torch.Tensor] = None, window_left: int = -1) -> Tuple[torch.Tensor, torch.Tensor]:
    """The end-to-end call: host tensors in, host tensors out (through attn_fwd_host).

    The inputs should be pinned (``tensor.pin_memory()``) for asynchronous
    copies.  ``out``/``lse`` are the host destinations (pinned, allocated when
    not given); ``staging`` holds the device buffers (allocated when not given).
    Everything is enqueued on ``stream`` (default: the current stream); with
    ``sync`` the call waits for it, else the results are valid once the stream
    has reached the call.  Device tensors are accepted too; then nothing is
    staged and the device results are returned.  Score modifications as in attn_fwd
    (``alibi_slopes`` on the device).
    """
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if q.is_cuda:
        return attn_fwd(q, k, v, bias, gate, causal, scale, out, lse, stream, softcap=softcap,
                        alibi_slopes=alibi_slopes, window_left=window_left)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if staging is None:
        staging = Staging(q, k, v, bias, gate, dev)
    if out is None:
        out = torch.empty(staging.out.shape, dtype=q.dtype, pin_memory=True)
    if lse is None:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, pin_memory=True)
    st = stream or torch.cuda.current_stream(dev)
    _check(attn_fwd_host_raw(q, k, v, bias, gate, causal, scale, out, lse, staging, st.cuda_stream, softcap,
                             alibi_slopes, window_left))
    if sync:
        st.synchronize()
    return out, lse


def last_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronises `stream` (default: the current one) and returns ATTN_ERR_TIMEOUT if any kernel
    of the library gave up a bounded wait since the last call, else ATTN_OK, and clears the word
    (ATTN_ERR_CUDA if the synchronisation or the read fails)."""
    s = (stream or torch.cuda.current_stream()).cuda_stream
    return load_library().attn_last_device_status(s)


def set_wait_limit(cycles: int):
    """Clock cycles a device-side wait polls before it gives up (applies to later launches)."""
    load_library().attn_set_wait_limit(int(cycles))


def debug_inject_stall(enable: bool):
    """Test hook: later launches time out on purpose (see include/attn.h)."""
    load_library().attn_debug_inject_stall(int(bool(enable)))


EXP2_FMA_PIPE, EXP2_MUFU, EXP2_CUDA_EXP2F = 0, 1, 2


def debug_exp2(x: torch.Tensor, mode: int) -> torch.Tensor:
    """Test hook: 2^x on the device with one of the kernel's exponentials (attn_debug_exp2);
    ``x`` is a contiguous float32 CUDA tensor.  Returns a new tensor (the stream is not synchronised)."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("debug_exp2 takes a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    s = torch.cuda.current_stream(x.device).cuda_stream
    _check(load_library().attn_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), int(mode), s))
    return y


def version() -> str:
    """The library's version string."""
    return load_library().attn_version().decode()
