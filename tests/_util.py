"""Small helpers shared by the tests (tolerances, dtype conversion)."""
import numpy as np
import torch

# Tolerances for floating-point outputs (compressor and attention) against
# the float64 oracle: max-abs <= 1e-2 and relative L2 <= 5e-3.
MAX_ABS = 1e-2
REL_L2 = 5e-3


def scaled_max_abs(ref) -> float:
    """The max-abs bound for outputs of inputs scaled beyond unit N(0,1)
    rows: MAX_ABS x max(1, max|ref|).  The stated bound is absolute for the
    workloads' unit-scale rows, whose outputs stay below 1; for rows scaled
    up (stress tests of the rescale and row-scale paths) the same relative
    precision is asked of larger outputs.  The relative L2 bound is unchanged."""
    return MAX_ABS * max(1.0, float(np.max(np.abs(np.asarray(ref, dtype=np.float64)))))


def bf16_half_ulp(x) -> np.ndarray:
    """Half the spacing of bf16 values (8 significand bits) in the binade of |x|."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return np.exp2(e - 8)


def assert_bf16_rounding_of(got, ref, what="", acc_rel=1e-5):
    """Outputs stored in bf16 from an fp32 computation: each is a bf16
    rounding of a value within acc_rel x max(1, |ref|) of the exact ref, so it
    lies within half a bf16 ulp of ref plus that.  (Comparing with the bf16
    rounding of ref itself fails by one ulp wherever ref and the fp32 value
    straddle a rounding midpoint.)"""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = np.abs(got - ref)
    bad = err > bf16_half_ulp(ref) + acc_rel * np.maximum(1.0, np.abs(ref))
    assert not bad.any(), f"{what}: {int(bad.sum())} outputs beyond half a bf16 ulp, worst error {err[bad].max():.3e}"


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def assert_close(got, ref, max_abs=MAX_ABS, rel_l2=REL_L2, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= max_abs and rel <= rel_l2, f"{what}: max-abs {err.max():.3e} rel-L2 {rel:.3e}"
    return float(err.max()), float(rel)
