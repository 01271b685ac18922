import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU case")


def bf16_values(bits):
    """uint16 bf16 bit patterns -> float64 values (test helper, not method arithmetic)."""
    import numpy as np

    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def expcast_rounding_witnesses(seed: int, n: int = 400_000):
    """Seeded ExpCast inputs (A, s, cb) whose product A*s lies within half an
    fp32 ulp of a tie m + 1/2 but not on it.  Rounding A*s + cb once and
    rounding A*s to fp32 first then disagree: cb's parity is chosen so that
    the tie would round to the even byte on the far side from the exact
    value.  Input construction only (test helper, not method arithmetic);
    returns float32 A, s, cb and the exact float64 product."""
    import numpy as np

    rng = np.random.default_rng(seed)
    D = rng.integers(-120, 60, n) + 0.5
    A = rng.uniform(0.25, 2.0, n).astype(np.float32)
    s = (D / A.astype(np.float64)).astype(np.float32)
    prod = A.astype(np.float64) * s.astype(np.float64)  # exact: 24 x 24 bits
    keep = (prod.astype(np.float32).astype(np.float64) == D) & (prod != D)
    A, s, D, prod = A[keep], s[keep], D[keep], prod[keep]
    fl = np.floor(D).astype(np.int64)
    # bytes spread over about 10..120; fl + cb even when the exact value lies
    # above the tie (the tie would go down), odd when below (it would go up)
    cb = 60 - fl + 2 * rng.integers(-25, 30, fl.size) + (prod < D)
    return A, s, cb.astype(np.float32), prod
