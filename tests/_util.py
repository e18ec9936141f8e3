"""Helpers shared by the tests (conversion and comparison only)."""
import numpy as np
import torch


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def npraw(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def rms(a) -> float:
    a = np.asarray(a, np.float64)
    return float(np.sqrt(np.mean(a * a)))


def assert_within_rms(got, ref, frac=2e-3, what=""):
    """max |got - ref| <= frac * RMS(ref), the float tolerance of the contract."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    bound = frac * rms(ref)
    assert err <= bound, f"{what}: max|err| {err:.3e} > {frac}*RMS(ref) = {bound:.3e}"
    return err / max(rms(ref), 1e-300)


def e4m3_step_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance between E4M3 codes in representable steps (sign-magnitude)."""
    def ordinal(c):
        c = c.astype(np.int64)
        mag = c & 0x7F
        return np.where(c & 0x80, -mag, mag)
    return np.abs(ordinal(a) - ordinal(b))
