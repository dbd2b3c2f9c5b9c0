"""Shared test helpers: bf16 tolerance and device plumbing."""
import numpy as np
import torch


def bf16_ulp(r: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |r| (8 significant bits)."""
    a = np.abs(np.asarray(r, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_bf16_close(y_bits, r32, extra=None, what=""):
    """bf16 output within one bf16 ulp of the oracle's fp32 value (plus an
    optional absolute slack, e.g. for a reassociated fp32 sum).  Returns the
    fraction of outputs equal to the oracle's own bf16 rounding."""
    y = bits_to_f64(y_bits)
    r = np.asarray(r32, dtype=np.float64)
    tol = bf16_ulp(r)
    if extra is not None:
        tol = tol + extra
    bad = np.abs(y - r) > tol
    if bad.any():
        i = np.flatnonzero(bad.reshape(-1))[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside 1 bf16 ulp; "
                             f"y={y.reshape(-1)[i]} ref={r.reshape(-1)[i]}")
    nz = np.abs(r) > 0
    if nz.any():
        rel = np.abs(y[nz] - r[nz]) / np.abs(r[nz])
        assert rel.max() <= 4e-3 + (0 if extra is None else np.inf), f"{what}: max rel err {rel.max()}"
    ref_bits = torch.from_numpy(np.ascontiguousarray(r, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)
    return float((np.asarray(y_bits) == ref_bits).mean())


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)
