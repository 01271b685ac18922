"""Bit-exact parity of the CUDA E4M3 encoder and ExpCast byte map with the
oracle, on identical fp32 inputs."""
import numpy as np
import pytest
import torch

import oracle
from conftest import expcast_rounding_witnesses

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


def test_e4m3_encode_bit_exact(vc):
    rng = np.random.default_rng(0)
    vals = oracle.e4m3_value(np.arange(127, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([
        rng.standard_normal(1_000_000).astype(np.float32) * 40,
        rng.standard_normal(200_000).astype(np.float32) * 0.005,
        rng.uniform(-460, 460, 200_000).astype(np.float32),
        mids, -mids, vals.astype(np.float32), -vals.astype(np.float32),
        np.array([0.0, -0.0, 448.0, 449.0, 464.0, 1e6, -1e6, 3e38, 1e-30, -1e-30], np.float32),
    ])
    got = vc.e4m3_encode(torch.from_numpy(x).cuda()).cpu().numpy()
    ref = oracle.e4m3_encode(x)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (x[bad[:8]], got[bad[:8]], ref[bad[:8]])


def test_expcast_bit_exact(vc):
    rng = np.random.default_rng(1)
    n = 2_000_000
    A = rng.uniform(0.0, 2.0, n).astype(np.float32)
    s = (rng.standard_normal(n) * 200).astype(np.float32)
    cb = rng.integers(-300, 127, n).astype(np.float32)
    # exact ties: A*s = m + 1/2
    A[:1000] = 0.5
    s[:1000] = (2 * rng.integers(-100, 200, 1000) + 1).astype(np.float32)
    # hugely negative scores and zero scale
    s[1000:1100] = -3e8
    A[1100:1200] = 0.0
    # the map's domain: 8z + 56 + beta <= 126 (the row reference keeps z <= 0)
    over = A.astype(np.float64) * s + cb > 126
    s[over] = 0.0
    # products within half an fp32 ulp of a tie: one rounding and two disagree
    wa, ws, wc, _ = expcast_rounding_witnesses(12)
    A, s, cb = np.concatenate([A, wa]), np.concatenate([s, ws]), np.concatenate([cb, wc])
    dev = [torch.from_numpy(a).cuda() for a in (A, s, cb)]
    got = vc.expcast_bytes(*dev).cpu().numpy()
    ref = oracle.expcast_bytes(A, s, cb)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (A[bad[:8]], s[bad[:8]], cb[bad[:8]], got[bad[:8]], ref[bad[:8]])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("tokens", [1, 31, 1000, 70001])
def test_quantize_q_bit_exact(vc, d, tokens):
    """The attention call's per-token Q quantiser against the oracle's: codes
    and scales bit-exact, on rows of mixed scale (lognormal), all-zero rows,
    rows of one nonzero channel, tiny (1e-30) and huge (1e30) rows, and rows
    of subnormal values beside one normal value, at token counts that leave a
    ragged last CTA.  (Rows whose amax is so small that 448/amax overflows are
    left out: both sides then encode 0 * inf, a NaN.)"""
    rng = np.random.default_rng(7 + d + tokens)
    q = (rng.standard_normal((tokens, d)) * np.exp(rng.normal(0.0, 2.0, (tokens, 1)))).astype(np.float32)
    q[::17] = 0.0
    q[5::23] = 0.0
    q[5::23, 3 % d] = -2.5
    q[7::29] *= 1e-30
    q[11::31] *= 1e30
    q[13::37] = 1e-39 * np.sign(q[13::37])
    q[13::37, 0] = 1.0
    bits = (torch.from_numpy(q).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16))
    codes, scales = vc.quantize_q(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda())
    ref_codes, ref_scales = oracle.quant_q(bits)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))


def test_quantize_q_rejects_bad_arguments(vc):
    q = torch.zeros(4, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError, match="vc_quantize_q"):
        vc.quantize_q(q)
