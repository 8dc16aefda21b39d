"""Shared test helpers: tolerances and GPU-vs-oracle comparison."""
import numpy as np
import torch

# Tolerances stated for the forward: max |O - O_ref| <= 2e-2 (bf16), 5e-3 (fp16)
# against the fp64 oracle, and 1e-3 relative on the logsumexp, read as
# |lse - lse_ref| <= 1e-3 * max(1, |lse_ref|) so that lse near 0 is well posed.
O_ATOL = {torch.bfloat16: 2e-2, torch.float16: 5e-3}
LSE_RTOL = 1e-3


def gpu_available():
    return torch.cuda.is_available()


def to_f64(t):
    return t.detach().cpu().double().numpy()


def assert_close_to_oracle(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    o = to_f64(o_gpu) if isinstance(o_gpu, torch.Tensor) else np.asarray(o_gpu, np.float64)
    l = to_f64(lse_gpu) if isinstance(lse_gpu, torch.Tensor) else np.asarray(lse_gpu, np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite O"
    err = np.abs(o - o_ref)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= O_ATOL[dtype], f"{what}: max |dO| = {worst:.3e} > {O_ATOL[dtype]:.1e}"
    if lse_ref is not None:
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(l), fin), f"{what}: lse finiteness differs"
        assert np.all(l[~fin] == lse_ref[~fin]), f"{what}: -inf rows differ"
        tol = LSE_RTOL * np.maximum(1.0, np.abs(lse_ref[fin]))
        lerr = np.abs(l[fin] - lse_ref[fin])
        assert np.all(lerr <= tol), f"{what}: lse err {float(lerr.max()):.3e} exceeds 1e-3 relative"
    return worst


def padded(t: torch.Tensor, device=None) -> torch.Tensor:
    """The same values, on ``device``, stored with the last dimension padded to a
    multiple of 8 elements (16 bytes), as the C ABI requires of bias rows.
    (The padding buffer is created on the target device because copying a
    non-dense view across devices would make it contiguous again.)"""
    n = t.shape[-1]
    device = t.device if device is None else torch.device(device)
    buf = torch.zeros(*t.shape[:-1], (n + 7) // 8 * 8, dtype=t.dtype, device=device)
    buf[..., :n] = t.to(device)
    return buf[..., :n]
