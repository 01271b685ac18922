"""The fp32 bound the near-tie refine relies on, checked on the host.

For a token v (bf16) and a centroid c (fp64), the refine computes in fp32,
from the centroid's bf16 pair (hi = RN(c), lo = RN(c - hi)):
  c32 = RN32(hi + lo),   D32 = sum over channels of (v - c32)^2
(d/8 channels a lane summed in order, then a three-level butterfly over the
eight lanes of the tie), and trusts
  |D32 - D| <= E = 2^-16 sqrt(D32) |c| + 2^-35 |c|^2 + 2^-18 D32,
D the exact squared distance.  The model below rounds each square separately
before adding it (the kernel's fused multiply-add rounds once), so it errs at
least as much as the kernel; the bound must hold on every draw, for
near-centroid tokens, large and tiny magnitudes, and mixed signs."""
import numpy as np
import pytest
import torch

D = 128
TL = 8  # lanes per tie


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round to nearest even bf16, returned as float64 (via torch's cast)."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def d32_model(v: np.ndarray, c: np.ndarray) -> float:
    """fp32 distance in the refine's order: d/8 channels a lane, then a
    three-level butterfly; squares rounded before they are added."""
    hi = bf16_round(c)
    lo = bf16_round(c - hi)
    c32 = (hi.astype(np.float32) + lo.astype(np.float32)).astype(np.float32)
    diff = (v.astype(np.float32) - c32).astype(np.float32)
    sq = (diff * diff).astype(np.float32)
    part = np.zeros(TL, np.float32)
    cpt = D // TL
    for lane in range(TL):
        acc = np.float32(0.0)
        for i in range(cpt):
            acc = np.float32(acc + sq[lane * cpt + i])
        part[lane] = acc
    step = TL // 2
    while step:
        part = np.array([np.float32(part[l] + part[l ^ step]) for l in range(TL)], np.float32)
        step //= 2
    return float(part[0])


def bound(d32: float, cn2: float) -> float:
    return 2.0 ** -16 * np.sqrt(d32 * cn2) + 2.0 ** -35 * cn2 + 2.0 ** -18 * d32


@pytest.mark.parametrize("scale", [1e-3, 0.3, 2.0, 40.0, 3e3])
def test_fp32_distance_within_bound(scale):
    rng = np.random.default_rng(int(scale * 1000) % 2**31)
    worst = 0.0
    for trial in range(400):
        c = rng.standard_normal(D) * scale * np.exp(rng.normal(0.0, 1.0, D))
        # tokens near the centroid (the near ties), at several distances
        noise = rng.standard_normal(D) * scale * 10.0 ** rng.uniform(-4, 0)
        v = bf16_round(c + noise)
        if trial % 7 == 0:
            v[rng.integers(0, D, 8)] = 0.0
        if trial % 11 == 0:
            v = -v
        d_exact = float(np.sum((v - c) ** 2))
        d32 = d32_model(v, c)
        cn2 = float(np.sum(c * c))
        e = bound(d32, cn2)
        assert abs(d32 - d_exact) <= e, (trial, d32, d_exact, e)
        worst = max(worst, abs(d32 - d_exact) / e)
    assert worst < 1.0
