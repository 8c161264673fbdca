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


def assert_close_out(got, want, atol, what="out"):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    i = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= atol, f"{what}: max abs err {err.max():.3e} at {i} (got {got[i]}, want {want[i]})"
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
