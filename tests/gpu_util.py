"""Helpers for the GPU parity tests (tests only)."""
import numpy as np
import torch

# Tolerance for attention outputs with fp32 accumulation: |err| <= 2e-3 + 2e-3 |ref|
# for fp16 and bf16.  A bf16 output is rounded once to 8 significant bits, which
# alone can move it by 2^-8 |ref| (more than 2e-3 |ref|), so bf16 adds that unit
# roundoff to the relative term.  fp32 outputs: 1e-5 + 1e-5 |ref|.
TOL = {"float16": (2e-3, 2e-3), "bfloat16": (2e-3, 2e-3 + 2.0 ** -8), "float32": (1e-5, 1e-5)}


def gpu_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def assert_close(got: torch.Tensor, ref: np.ndarray, dtype: str, what: str = "", rows=None):
    """|got - ref| <= atol + rtol |ref| element by element; ``rows`` restricts
    the comparison to the listed (sequence, head) rows."""
    g = gpu_f64(got)
    if rows is not None:
        idx = tuple(np.asarray(rows).T)
        g, ref = g[idx], ref[idx]
    atol, rtol = TOL[dtype]
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    lim = atol + rtol * np.abs(ref)
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                           f"max err {err.max():.3e}, worst ratio {(err / lim).max():.2f}")
    return float(err.max())


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a tensor as a numpy array (bit-exact comparisons)."""
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def np_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a).view(np.uint8)
