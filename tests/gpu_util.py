"""Helpers for the GPU parity tests (tests only)."""
import numpy as np
import torch

# Tolerance for attention outputs with fp32 accumulation: |err| <= 2e-3 + 2e-3 |ref|
# for fp16 and bf16; fp32 outputs: 1e-5 + 1e-5 |ref|.
#
# bf16 keeps 8 significant bits, so rounding a result to bf16 moves it by up to
# 2^-8 |ref| (half a unit in the last place): for |ref| >= 2 even the correctly
# rounded value of the exact result can fall outside 2e-3 + 2e-3 |ref|.  The bound
# is therefore checked on the fp32 result before that one rounding (the library's
# PA_DECODE_OUT_F32 output, see check_bf16), and a bf16 output is accepted where it
# meets the bound or is one of the two bf16 values next to ref (a faithful rounding
# of the exact result); check_bf16 also proves it is the fp32 result rounded to
# nearest even, bit for bit.
TOL = {"float16": (2e-3, 2e-3), "bfloat16": (2e-3, 2e-3), "float32": (1e-5, 1e-5)}


def gpu_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def bf16_neighbours(ref: np.ndarray):
    """The bf16 values just below and just above each element of ref (equal when
    ref is a bf16 value; via fp32, which keeps 16 more bits than bf16)."""
    f = np.ascontiguousarray(ref, dtype=np.float32)
    u = f.view(np.uint32)
    lo = (u & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)  # toward zero
    exact = (u & np.uint32(0xFFFF)) == 0
    hi = ((u & np.uint32(0xFFFF0000)) + np.uint32(0x10000)).view(np.float32).astype(np.float64)
    hi = np.where(exact, lo, hi)  # away from zero
    return np.minimum(lo, hi), np.maximum(lo, hi)


def assert_close(got: torch.Tensor, ref: np.ndarray, dtype: str, what: str = "", rows=None):
    """|got - ref| <= atol + rtol |ref| element by element (bf16: or got a bf16
    neighbour of ref); ``rows`` restricts the comparison to the listed
    (sequence, head) rows."""
    g = gpu_f64(got)
    if rows is not None:
        idx = tuple(np.asarray(rows).T)
        g, ref = g[idx], ref[idx]
    atol, rtol = TOL[dtype]
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    lim = atol + rtol * np.abs(ref)
    bad = err > lim
    if dtype == "bfloat16" and got.dtype == torch.bfloat16:
        lo, hi = bf16_neighbours(ref)
        bad &= (g != lo) & (g != hi)
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                           f"max err {err.max():.3e}, worst ratio {(err / lim).max():.2f}")
    return float(err.max())


def check_bf16(got_bf16: torch.Tensor, got_f32: torch.Tensor, ref: np.ndarray, what: str = "", rows=None):
    """A bf16 decode against the oracle: its fp32 result (the same call with a
    float32 out) meets |err| <= 2e-3 + 2e-3 |ref| element by element, and the
    bf16 output is exactly that fp32 result rounded to nearest even."""
    assert got_f32.dtype == torch.float32 and got_bf16.dtype == torch.bfloat16
    assert_close(got_f32, ref, "bfloat16", f"{what} (fp32 result)", rows=rows)
    rne = got_f32.to(torch.bfloat16)
    assert np.array_equal(bits(got_bf16), bits(rne)), f"{what}: bf16 output is not the fp32 result rounded"
    assert_close(got_bf16, ref, "bfloat16", what, rows=rows)


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a tensor as a numpy array (bit-exact comparisons)."""
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def np_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a).view(np.uint8)
