"""Helpers shared by the tests: raw-bit extraction for the oracle and
tolerance checks."""
import numpy as np
import torch

import oracle

_FMT = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float8_e4m3fn: "e4m3",
        torch.float8_e5m2: "e5m2"}


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Decode a bf16/fp16/FP8 tensor exactly to float64 through the oracle's
    format decoders (from the raw storage bits)."""
    t = t.detach().cpu().contiguous()
    fmt = _FMT[t.dtype]
    if fmt in ("bf16", "fp16"):
        bits = t.view(torch.int16).numpy().view(np.uint16)
    else:
        bits = t.view(torch.uint8).numpy()
    return oracle.decode(bits, fmt)


def round_bf16(x):
    """float64 values rounded to the nearest bf16 value (8 significant bits),
    ties to even; the normal range only (|x| >= 2^-126), which is all the
    outputs compared here need."""
    m, e = np.frexp(np.asarray(x, np.float64))   # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)   # np.rint rounds half to even


def assert_close_out(got, want, atol, what="out", rounded=True):
    """Every element within atol of the fp64 oracle, or (rounded) equal to the
    oracle's value correctly rounded to bf16. The output is bf16 by definition
    (MATE "Attention", FMHA dtype notes), and its own rounding moves an element
    by up to half a bf16 unit: 2^-7 = 0.0078 for |O| in [2, 4), 0.0156 in
    [4, 8). Where that alone reaches the tolerance, the correctly rounded
    value is the best any kernel can return, and it is accepted."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    bad = err > atol
    if rounded:
        bad &= got != round_bf16(want)
    if bad.any():
        e = np.where(bad, err, 0.0)
        i = np.unravel_index(np.argmax(e), e.shape)
        raise AssertionError(f"{what}: max abs err {err[i]:.3e} at {i} (got {got[i]}, "
                             f"want {want[i]}), {int(bad.sum())} elements beyond {atol}")
    return float(err.max())


def assert_close_lse(got, want, atol=1e-3, what="lse"):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    ninf_w = np.isneginf(want)
    assert np.array_equal(np.isneginf(got), ninf_w), f"{what}: -inf pattern differs"
    ok = ~ninf_w
    if ok.any():
        err = np.abs(got[ok] - want[ok])
        assert np.all(np.isfinite(got[ok])) and err.max() <= atol, f"{what}: max abs err {err.max():.3e}"
        return float(err.max())
    return 0.0
