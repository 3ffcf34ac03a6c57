"""Shared test helpers: device transfer of generator output and the float tolerance.

Tolerance for the fp32 attention output against the float64 oracle: max-abs 1e-2
and relative RMS 1e-3 (inputs are bf16, accumulation fp32)."""
import numpy as np
import torch

MAX_ABS = 1e-2
REL_RMS = 1e-3


def dev_bf16(a_u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).to("cuda").view(torch.bfloat16)


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def assert_close_out(got: np.ndarray, want: np.ndarray, what: str = "out"):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - want)
    assert err.max(initial=0.0) <= MAX_ABS, f"{what}: max abs err {err.max()}"
    denom = np.sqrt(np.mean(want ** 2)) if want.size else 0.0
    if denom > 0:
        rel = np.sqrt(np.mean((got - want) ** 2)) / denom
        assert rel <= REL_RMS, f"{what}: rel RMS err {rel}"
