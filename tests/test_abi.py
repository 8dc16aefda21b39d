"""Host-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments with the documented status codes
before touching the GPU (so these run without one)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from exact_attention_sdpa_b200 import _native as nat
from exact_attention_sdpa_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return nat.load_library()


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_binding_surface():
    assert set(_declared_functions()) == set(nat.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", nat.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (attn_\w+)", out))
    for name in _declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code in range(5):
        s = nat.status_string(code)
        assert isinstance(s, str) and len(s) > 0
    assert nat.status_string(123) == "unknown status"
    assert nat.version().count(".") == 2


def _qkv(B=1, H=2, N=64, d=64, dtype=torch.float16):
    # CPU tensors: only their addresses/shapes are read by the host-side checks
    mk = lambda: torch.zeros(B, H, N, d, dtype=dtype)
    return mk(), mk(), mk(), mk()


def call(q, k, v, out, bias=None, gate=None, causal=False, scale=0.125, lse=None):
    return nat.attn_fwd_raw(q, k, v, bias, gate, causal, scale, out, lse, 0)


def test_null_arguments(lib):
    q, k, v, o = _qkv()
    P = ctypes.POINTER(nat.AttnTensor)
    vq, vk, vv, vo = (nat.make_view(t) for t in (q, k, v, o))
    r = lib.attn_fwd(None, ctypes.byref(vk), ctypes.byref(vv), None, None, 0, 0.1, ctypes.byref(vo), None, None)
    assert r == nat.ATTN_ERR_INVALID_ARG
    r = lib.attn_fwd(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), None, None, 0, 0.1, None, None, None)
    assert r == nat.ATTN_ERR_INVALID_ARG
    vq.data = None
    r = lib.attn_fwd(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), None, None, 0, 0.1, ctypes.byref(vo),
                     None, None)
    assert r == nat.ATTN_ERR_INVALID_ARG


def test_fp32_is_unsupported(lib):
    q, k, v, o = _qkv(dtype=torch.float32)
    assert call(q, k, v, o) == nat.ATTN_ERR_UNSUPPORTED


def test_mixed_dtypes_unsupported(lib):
    q, k, v, o = _qkv()
    assert call(q, k.to(torch.bfloat16), v, o) == nat.ATTN_ERR_UNSUPPORTED
    assert call(q, k, v, o.to(torch.bfloat16)) == nat.ATTN_ERR_UNSUPPORTED


def test_unknown_dtype_invalid(lib):
    q, k, v, o = _qkv()
    assert call(q.to(torch.int16), k, v, o) == nat.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("d", [16, 48, 96, 256])
def test_head_dim_unsupported(lib, d):
    q, k, v, o = _qkv(d=d)
    assert call(q, k, v, o) == nat.ATTN_ERR_UNSUPPORTED


def test_shape_mismatch(lib):
    q, k, v, o = _qkv()
    k2 = torch.zeros(1, 2, 65, 64, dtype=torch.float16)
    assert call(q, k2, v, o) == nat.ATTN_ERR_INVALID_ARG
    o2 = torch.zeros(1, 3, 64, 64, dtype=torch.float16)
    assert call(q, k, v, o2) == nat.ATTN_ERR_INVALID_ARG
    assert call(q[0], k[0], v[0], o[0]) == nat.ATTN_ERR_INVALID_ARG          # rank 3


def test_non_unit_inner_stride(lib):
    q, k, v, o = _qkv()
    qt = torch.zeros(1, 2, 64, 64, dtype=torch.float16).transpose(2, 3)
    assert call(qt, k, v, o) == nat.ATTN_ERR_INVALID_ARG


def test_misaligned_row_stride(lib):
    # rows 68 elements apart (136 bytes): not a multiple of 16 bytes
    base = torch.zeros(1, 2, 64, 68, dtype=torch.float16)
    q = base[..., :64]
    _, k, v, o = _qkv()
    assert call(q, k, v, o) == nat.ATTN_ERR_INVALID_ARG


def test_misaligned_base(lib):
    flat = torch.zeros(1 * 2 * 64 * 64 + 8, dtype=torch.float16)
    q = flat[1:1 + 2 * 64 * 64].view(1, 2, 64, 64)                            # 2-byte offset
    _, k, v, o = _qkv()
    assert call(q, k, v, o) == nat.ATTN_ERR_INVALID_ARG


def test_non_finite_scale(lib):
    q, k, v, o = _qkv()
    assert call(q, k, v, o, scale=float("nan")) == nat.ATTN_ERR_INVALID_ARG
    assert call(q, k, v, o, scale=float("inf")) == nat.ATTN_ERR_INVALID_ARG


def test_out_aliasing_input(lib):
    q, k, v, _ = _qkv()
    assert call(q, k, v, q) == nat.ATTN_ERR_INVALID_ARG
    assert call(q, k, v, v) == nat.ATTN_ERR_INVALID_ARG


def test_bias_and_gate_shapes(lib):
    q, k, v, o = _qkv()
    bad_bias = torch.zeros(2, 64, 32, dtype=torch.float16)
    assert call(q, k, v, o, bias=bad_bias) == nat.ATTN_ERR_INVALID_ARG
    bad_bias4 = torch.zeros(2, 2, 64, 64, dtype=torch.float16)               # B mismatch
    assert call(q, k, v, o, bias=bad_bias4) == nat.ATTN_ERR_INVALID_ARG
    assert call(q, k, v, o, bias=torch.zeros(64, 64, dtype=torch.float16)) == nat.ATTN_ERR_INVALID_ARG
    assert call(q, k, v, o, bias=torch.zeros(2, 64, 64, dtype=torch.bfloat16)) == nat.ATTN_ERR_UNSUPPORTED
    bad_gate = torch.zeros(1, 2, 64, 32, dtype=torch.float16)
    assert call(q, k, v, o, gate=bad_gate) == nat.ATTN_ERR_INVALID_ARG


def test_misaligned_lse(lib):
    q, k, v, o = _qkv()
    lse = torch.zeros(1 + 2 * 64, dtype=torch.uint8)[1:]
    r = nat.attn_fwd_raw(q, k, v, None, None, False, 0.1, o, None, 0)
    vq, vk, vv, vo = (nat.make_view(t) for t in (q, k, v, o))
    r = nat.load_library().attn_fwd(ctypes.byref(vq), ctypes.byref(vk), ctypes.byref(vv), None, None, 0, 0.1,
                                    ctypes.byref(vo), lse.data_ptr(), None)
    assert r == nat.ATTN_ERR_INVALID_ARG


def test_empty_problem_is_ok_without_launch(lib):
    q = torch.zeros(1, 2, 0, 64, dtype=torch.float16)
    assert call(q, q.clone(), q.clone(), q.clone()) == nat.ATTN_OK
    q = torch.zeros(0, 2, 16, 64, dtype=torch.float16)
    assert call(q, q.clone(), q.clone(), q.clone()) == nat.ATTN_OK
    k = torch.zeros(1, 2, 3, 64, dtype=torch.float16)
    assert call(torch.zeros(1, 2, 0, 64, dtype=torch.float16), k, k, k) == nat.ATTN_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no fallback"):
        nat.load_library(str(tmp_path / "libattn.so"))


def test_product_path_does_not_reach_the_oracle():
    # no import of, or path into, the oracle package anywhere in the product
    pat = re.compile(r"^\s*(from\s+oracle\b|import\s+oracle\b)|oracle/|importlib.*oracle", re.M)
    pkg = os.path.join(ROOT, "exact_attention_sdpa_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not pat.search(text), fn


# ---- attn_fwd_host: every check happens before the first copy is enqueued, so
# CPU tensors stand in for both the host buffers and the device staging here.

class _FakeStaging:
    def __init__(self, q, k, v, bias=None, gate=None, out=None):
        self.q, self.k, self.v, self.bias, self.gate = q, k, v, bias, gate
        self.out = torch.zeros_like(q) if out is None else out
        self.lse = torch.zeros(q.shape[:-1], dtype=torch.float32)


def call_host(hq, hk, hv, ho, st, bias=None, gate=None, lse=None, scale=0.125):
    return nat.attn_fwd_host_raw(hq, hk, hv, bias, gate, False, scale, ho, lse, st, 0)


def test_host_entry_rejects_layout_mismatch(lib):
    q, k, v, o = _qkv()
    st = _FakeStaging(*_qkv()[:3])
    assert call_host(q, k, v, o, _FakeStaging(*_qkv(N=32)[:3])) == nat.ATTN_ERR_INVALID_ARG      # shapes
    padded = torch.zeros(1, 2, 64, 72, dtype=torch.float16)[..., :64]
    assert call_host(q, k, v, o, _FakeStaging(padded, *_qkv()[1:3])) == nat.ATTN_ERR_INVALID_ARG  # strides
    assert call_host(q, k, v, o, _FakeStaging(q.to(torch.bfloat16), *_qkv()[1:3])) != nat.ATTN_OK  # dtype
    bias = torch.zeros(2, 64, 64, dtype=torch.float16)
    assert call_host(q, k, v, o, st, bias=bias) == nat.ATTN_ERR_INVALID_ARG                        # bias vs none
    st_b = _FakeStaging(*_qkv()[:3], bias=torch.zeros(2, 64, 64, dtype=torch.float16))
    assert call_host(q, k, v, o, st_b) == nat.ATTN_ERR_INVALID_ARG                                 # none vs bias
    assert call_host(q, k, v, torch.zeros(1, 2, 64, 32, dtype=torch.float16), st) == nat.ATTN_ERR_INVALID_ARG


def test_host_entry_applies_device_checks_and_null_rules(lib):
    q, k, v, o = _qkv()
    f32 = _FakeStaging(*_qkv(dtype=torch.float32)[:3])
    assert call_host(*_qkv(dtype=torch.float32), f32) == nat.ATTN_ERR_UNSUPPORTED
    st = _FakeStaging(*_qkv()[:3])
    assert call_host(q, k, v, o, st, scale=float("nan")) == nat.ATTN_ERR_INVALID_ARG
    # lse on the host side without an lse staging buffer (and the reverse)
    P = ctypes.POINTER(nat.AttnTensor)
    views = [nat.make_view(t) for t in (q, k, v, o, st.q, st.k, st.v, st.out)]
    refs = [ctypes.byref(x) for x in views]
    lse = torch.zeros(1, 2, 64, dtype=torch.float32)
    r = lib.attn_fwd_host(refs[0], refs[1], refs[2], None, None, 0, 0.1, refs[3], lse.data_ptr(),
                          refs[4], refs[5], refs[6], None, None, refs[7], None, None)
    assert r == nat.ATTN_ERR_INVALID_ARG
    r = lib.attn_fwd_host(refs[0], refs[1], refs[2], None, None, 0, 0.1, refs[3], None,
                          refs[4], refs[5], refs[6], None, None, refs[7], st.lse.data_ptr(), None)
    assert r == nat.ATTN_ERR_INVALID_ARG
    r = lib.attn_fwd_host(refs[0], refs[1], refs[2], None, None, 0, 0.1, refs[3], None,
                          None, refs[5], refs[6], None, None, refs[7], None, None)
    assert r == nat.ATTN_ERR_INVALID_ARG


def test_host_entry_checks_score_modifications_before_any_copy(lib):
    q, k, v, o = _qkv()
    st = _FakeStaging(*_qkv()[:3])
    assert nat.attn_fwd_host_raw(q, k, v, None, None, True, 0.125, o, None, st, 0,
                                 softcap=-1.0) == nat.ATTN_ERR_INVALID_ARG
    assert nat.attn_fwd_host_raw(q, k, v, None, None, True, 0.125, o, None, st, 0,
                                 softcap=float("nan")) == nat.ATTN_ERR_INVALID_ARG
    bias = torch.zeros(2, 64, 64, dtype=torch.float16)
    st_b = _FakeStaging(*_qkv()[:3], bias=torch.zeros(2, 64, 64, dtype=torch.float16))
    assert nat.attn_fwd_host_raw(q, k, v, bias, None, True, 0.125, o, None, st_b, 0,
                                 window_left=10) == nat.ATTN_ERR_UNSUPPORTED
    # a misaligned slopes pointer (never dereferenced: rejected first)
    slopes = torch.zeros(4, dtype=torch.float32)
    views = [nat.make_view(t) for t in (q, k, v, o, st.q, st.k, st.v, st.out)]
    refs = [ctypes.byref(x) for x in views]
    mods = nat.AttnMods(slopes.data_ptr() + 2, 0.0, -1)
    r = lib.attn_fwd_host_ex(refs[0], refs[1], refs[2], None, None, 1, 0.125, ctypes.byref(mods), refs[3], None,
                             refs[4], refs[5], refs[6], None, None, refs[7], None, None)
    assert r == nat.ATTN_ERR_INVALID_ARG


def test_host_entry_empty_problem_is_ok(lib):
    q = torch.zeros(1, 2, 0, 64, dtype=torch.float16)
    st = _FakeStaging(q.clone(), q.clone(), q.clone())
    assert call_host(q, q.clone(), q.clone(), q.clone(), st) == nat.ATTN_OK


def test_rectangular_shape_rules(lib):
    q = torch.zeros(1, 2, 48, 64, dtype=torch.float16)
    o = torch.zeros_like(q)
    k = torch.zeros(1, 2, 80, 64, dtype=torch.float16)
    v80, v64 = torch.zeros_like(k), torch.zeros(1, 2, 64, 64, dtype=torch.float16)
    assert call(q, k, v64, o) == nat.ATTN_ERR_INVALID_ARG                       # K and V key counts differ
    assert call(q, k, v80, torch.zeros(1, 2, 80, 64, dtype=torch.float16)) == nat.ATTN_ERR_INVALID_ARG  # O not Q's shape
    assert call(q, k, v80, o, bias=torch.zeros(2, 48, 48, dtype=torch.float16)) == nat.ATTN_ERR_INVALID_ARG
    assert call(q, k, v80, o, bias=torch.zeros(2, 80, 80, dtype=torch.float16)) == nat.ATTN_ERR_INVALID_ARG
    k32 = torch.zeros(1, 2, 80, 32, dtype=torch.float16)
    assert call(q, k32, torch.zeros_like(k32), o) == nat.ATTN_ERR_INVALID_ARG    # head dims differ
    k0 = torch.zeros(1, 2, 0, 64, dtype=torch.float16)
    assert call(q, k0, k0.clone(), o) == nat.ATTN_ERR_INVALID_ARG               # no keys for 48 queries


def test_backward_argument_checks(lib):
    q, k, v, o = _qkv()
    lse = torch.zeros(1, 2, 64, dtype=torch.float32)
    do, dq, dk, dv = (torch.zeros_like(q) for _ in range(4))

    def bwd(**kw):
        a = dict(q=q, k=k, v=v, out=o, lse=lse, dout=do, dq=dq, dk=dk, dv=dv)
        a.update(kw)
        return nat.attn_bwd_raw(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], False, 0.125,
                                a["dq"], a["dk"], a["dv"], 0)

    assert bwd(lse=None) == nat.ATTN_ERR_INVALID_ARG
    assert bwd(dq=torch.zeros(1, 2, 32, 64, dtype=torch.float16)) == nat.ATTN_ERR_INVALID_ARG
    assert bwd(dk=q) == nat.ATTN_ERR_INVALID_ARG                                  # overlaps an input
    assert bwd(dv=dk) == nat.ATTN_ERR_INVALID_ARG                                 # overlaps another output
    assert bwd(dout=do.to(torch.bfloat16)) == nat.ATTN_ERR_UNSUPPORTED
    q32 = torch.zeros(1, 2, 64, 64, dtype=torch.float32)
    assert bwd(q=q32) == nat.ATTN_ERR_UNSUPPORTED
    e = torch.zeros(1, 2, 0, 64, dtype=torch.float16)
    assert nat.attn_bwd_raw(e, k, v, e.clone(), None, e.clone(), False, 0.1, e.clone(), torch.zeros_like(k),
                            torch.zeros_like(v), 0) == nat.ATTN_OK                 # no query rows: nothing to do


def test_modification_argument_checks(lib):
    q, k, v, o = _qkv()
    r = nat.attn_fwd_raw(q, k, v, None, None, False, 0.1, o, None, 0, softcap=-1.0)
    assert r == nat.ATTN_ERR_INVALID_ARG
    r = nat.attn_fwd_raw(q, k, v, None, None, False, 0.1, o, None, 0, softcap=float("inf"))
    assert r == nat.ATTN_ERR_INVALID_ARG
    bias = torch.zeros(2, 64, 64, dtype=torch.float16)
    r = nat.attn_fwd_raw(q, k, v, bias, None, False, 0.1, o, None, 0, window_left=4)
    assert r == nat.ATTN_ERR_UNSUPPORTED                                       # modifications with a bias
    bad = torch.zeros(3, dtype=torch.uint8)[1:]
    r = nat.attn_fwd_raw(q, k, v, None, None, False, 0.1, o, None, 0, alibi_slopes=bad)
    assert r == nat.ATTN_ERR_INVALID_ARG                                       # misaligned slopes


def test_varlen_argument_checks(lib):
    q = torch.zeros(10, 2, 64, dtype=torch.float16)
    k = torch.zeros(12, 2, 64, dtype=torch.float16)
    o = torch.zeros_like(q)
    ok_q = torch.tensor([0, 4, 10], dtype=torch.int32)
    ok_k = torch.tensor([0, 5, 12], dtype=torch.int32)

    def call_v(cq, ck, q_=q, k_=k, o_=o):
        return nat.attn_fwd_varlen_raw(q_, k_, k_.clone(), cq, ck, True, 0.1, o_, None, 0)

    assert call_v(torch.tensor([0, 4, 9], dtype=torch.int32), ok_k) == nat.ATTN_ERR_INVALID_ARG   # does not end at Tq
    assert call_v(torch.tensor([1, 4, 10], dtype=torch.int32), ok_k) == nat.ATTN_ERR_INVALID_ARG  # does not start at 0
    assert call_v(torch.tensor([0, 11, 10], dtype=torch.int32), ok_k) == nat.ATTN_ERR_INVALID_ARG  # decreasing
    assert call_v(ok_q, torch.tensor([0, 0, 12], dtype=torch.int32)) == nat.ATTN_ERR_INVALID_ARG   # queries, no keys
    assert call_v(ok_q, ok_k, q_=q.unsqueeze(0)) == nat.ATTN_ERR_INVALID_ARG                       # rank 4
    assert call_v(ok_q, ok_k, k_=torch.zeros(12, 2, 32, dtype=torch.float16)) == nat.ATTN_ERR_INVALID_ARG
    e = torch.zeros(0, 2, 64, dtype=torch.float16)
    z = torch.zeros(1, dtype=torch.int32)
    assert nat.attn_fwd_varlen_raw(e, e, e.clone(), z, z, True, 0.1, e.clone(), None, 0) == nat.ATTN_OK


def test_varlen_aliasing_across_sequences(lib):
    """O of one sequence must not overlap Q, K or V rows of another; lse overlaps nothing."""
    buf = torch.zeros(24, 2, 64, dtype=torch.float16)
    q, o_other = buf[:10], buf[10:20]                    # disjoint: fine
    k = torch.zeros(12, 2, 64, dtype=torch.float16)
    cq = torch.tensor([0, 4, 10], dtype=torch.int32)
    ck = torch.tensor([0, 5, 12], dtype=torch.int32)
    v = torch.zeros_like(k)
    call = lambda q_, o_, lse=None: nat.attn_fwd_varlen_raw(q_, k, v, cq, ck, True, 0.1, o_, lse, 0)
    # out's rows 4..9 (sequence 1) land on q's rows of the same buffer shifted by 6: sequence 0's out
    # rows and sequence 1's q rows overlap only across sequences
    o_shift = buf[6:16]
    assert call(buf[:10], o_shift) == nat.ATTN_ERR_INVALID_ARG
    lse_bad = buf.view(-1).view(torch.float32)[:2 * 10]   # lse aliasing q's storage
    assert call(q, o_other, lse_bad) == nat.ATTN_ERR_INVALID_ARG


def test_backward_lse_must_not_overlap_gradients(lib):
    q, k, v, o = _qkv()
    do, dk, dv = (torch.zeros_like(q) for _ in range(3))
    dq = torch.zeros_like(q)
    lse_in_dq = dq.view(-1).view(torch.float32)[:2 * 64]
    r = nat.attn_bwd_raw(q, k, v, o, lse_in_dq, do, False, 0.125, dq, dk, dv, 0)
    assert r == nat.ATTN_ERR_INVALID_ARG


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "attn.h"
int main(void) {
    /* host-side calls only: no device work */
    if (strchr(attn_version(), '.') == NULL) return 1;
    if (attn_status_string(ATTN_ERR_TIMEOUT) == NULL) return 2;
    attn_tensor_t q;
    memset(&q, 0, sizeof(q));
    if (attn_fwd(NULL, &q, &q, NULL, NULL, 0, 0.125f, &q, NULL, 0) != ATTN_ERR_INVALID_ARG) return 3;
    q.dtype = ATTN_F32;
    if (attn_fwd(&q, &q, &q, NULL, NULL, 0, 0.125f, &q, NULL, 0) != ATTN_ERR_UNSUPPORTED) return 4;
    printf("ok\n");
    return 0;
}
"""


def test_plain_c_client_compiles_links_and_calls(lib, tmp_path):
    """The boundary is a C ABI: a C99 program includes the header, links libattn.so and
    gets the documented status codes (host-side checks only)."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(nat.LIB_PATH)
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                        str(src), "-L", libdir, "-lattn", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)


def test_fp8_argument_checks(lib):
    """attn_fwd_fp8 rejects what it does not serve before any launch."""
    f8 = lambda *shape: torch.zeros(*shape, dtype=torch.uint8).view(torch.float8_e4m3fn)
    q, k = f8(1, 2, 64, 64), f8(1, 2, 80, 64)
    vt = f8(1, 2, 64, 80)
    o = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    call = lambda q_=q, k_=k, v_=vt, o_=o, sq=1.0, sk=1.0, sv=1.0: nat.attn_fwd_fp8_raw(
        q_, k_, v_, sq, sk, sv, True, 0.125, o_, None, 0)
    assert call(q_=torch.zeros(1, 2, 64, 64, dtype=torch.float16)) == nat.ATTN_ERR_UNSUPPORTED   # not e4m3
    assert call(o_=torch.zeros(1, 2, 64, 64, dtype=torch.float32)) == nat.ATTN_ERR_UNSUPPORTED   # out fp32
    assert call(q_=f8(1, 2, 64, 32), k_=f8(1, 2, 80, 32), v_=f8(1, 2, 32, 80),
                o_=torch.zeros(1, 2, 64, 32, dtype=torch.bfloat16)) == nat.ATTN_ERR_UNSUPPORTED  # d = 32
    assert call(sq=0.0) == nat.ATTN_ERR_INVALID_ARG
    assert call(sv=float("nan")) == nat.ATTN_ERR_INVALID_ARG
    assert call(v_=f8(1, 2, 80, 64)) == nat.ATTN_ERR_INVALID_ARG          # V not transposed
    assert call(o_=torch.zeros(1, 2, 48, 64, dtype=torch.bfloat16)) == nat.ATTN_ERR_INVALID_ARG
    bad = f8(1, 2, 64, 72)[..., :64]                                     # row stride 72 bytes: not 16-aligned
    assert call(q_=bad) == nat.ATTN_ERR_INVALID_ARG
    # e4m3 given to the 16-bit entry point
    assert nat.attn_fwd_raw(q, q, q, None, None, False, 0.1, o, None, 0) == nat.ATTN_ERR_UNSUPPORTED
