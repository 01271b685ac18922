import os
import sys

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


NVFP4_TIE_SCALES = (2.0, 3.75, 3.5, 1.875, 7.5, 0.75, 13.0, 15.0, 0.5, 1.625, 0.013671875, 0.0390625, 104.0, 240.0)
E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def nvfp4_tie_values(seed: int, N: int = 256, d: int = 128):
    """Seeded V values [N, d] (float32, all bf16-exact) whose 4-bit residual
    without V-Smooth lands on E2M1 ties.  Token 0 of every channel is 2688,
    so the channel scale amax/2688 is exactly 1 and y = v.  Each 16-token
    block leads with 6*s, so its scale E4M3(6s/6) is exactly s, one of
    NVFP4_TIE_SCALES (448 in the first block).  The other 15 tokens are
    +-s * m, m an E2M1 midpoint (mostly) or grid value.  Input construction
    only (test helper, not method arithmetic); returns (v, scale per block
    [N/16, d])."""
    import numpy as np

    rng = np.random.default_rng(seed)
    assert N % 16 == 0
    nb = N // 16
    scales = np.empty((nb, d))
    v = np.empty((N, d))
    for j in range(nb):
        for c in range(d):
            s = 448.0 if j == 0 else NVFP4_TIE_SCALES[(j + 3 * c) % len(NVFP4_TIE_SCALES)]
            scales[j, c] = s
            m = np.where(rng.random(15) < 0.8, rng.choice(E2M1_MIDPOINTS, 15), rng.choice(E2M1_GRID, 15))
            v[16 * j, c] = 6.0 * s
            v[16 * j + 1:16 * j + 16, c] = s * m * rng.choice([-1.0, 1.0], 15)
    return v.astype(np.float32), scales
