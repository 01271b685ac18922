"""Pins of the oracle's 4-bit (NVFP4) path.

Independent references:
- ml_dtypes' float4_e2m1fn, for the E2M1 codec;
- brute force over the eight E2M1 magnitudes, for the block coder;
- numpy recomputation of the residual and its scales, for the V residual;
- a small online replay in Python on top of the pinned primitives, for the
  P re-coding inside the attention replay.

The 4-bit residual is the NVFP4 option the pages give beside E4M3 for the
per-channel V residual (zerohour.day summary, key facts).
"""
import ml_dtypes
import numpy as np
import pytest

import oracle
from bit_fp8_attention_smooth_b200 import synth
from conftest import bf16_values

F4 = ml_dtypes.float4_e2m1fn
MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_e2m1_decode_exhaustive_vs_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(F4).astype(np.float64)
    np.testing.assert_array_equal(oracle.e2m1_value(codes), ref)


def test_e2m1_encode_vs_ml_dtypes():
    rng = np.random.default_rng(0)
    mids = (MAGS[1:] + MAGS[:-1]) / 2  # every tie
    x = np.concatenate([rng.standard_normal(20000) * 3, rng.uniform(-8, 8, 20000), mids, -mids, MAGS, -MAGS,
                        [7.0, 100.0, -100.0, 1e-30, -1e-30, 0.0, -0.0]]).astype(np.float32)
    ref = x.astype(F4).view(np.uint8)
    np.testing.assert_array_equal(oracle.e2m1_encode(x), ref)


def test_e2m1_ties_to_even_and_saturation():
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 1e9], np.float32)
    # ties go to the code whose mantissa bit is 0
    np.testing.assert_array_equal(oracle.e2m1_value(oracle.e2m1_encode(x)), [0, 1, 1, 2, 2, 4, 4, 6, 6])


def _brute_block(x):
    """NVFP4 block by brute force: scale E4M3(amax/6), then for each value the
    E2M1 code nearest to x*(1/s), ties to the even code."""
    x = np.asarray(x, np.float32)
    amax = np.float32(np.abs(x).max())
    s = oracle.e4m3_encode(np.float32(amax / np.float32(6.0)))[()]
    sv = np.float32(oracle.e4m3_value(np.uint8(s)))
    if sv == 0:
        return np.zeros(x.shape, np.uint8), s
    r = np.float32(np.float32(1.0) / sv)
    y = (x * r).astype(np.float32).astype(np.float64)
    codes = []
    for v in y:
        a = min(abs(v), 6.0)
        dist = np.abs(MAGS - a)
        best = np.flatnonzero(dist == dist.min())
        c = best[0] if len(best) == 1 else best[best % 2 == 0][0]
        codes.append(int(c) | (8 if np.signbit(v) else 0))
    return np.array(codes, np.uint8), s


def test_nvfp4_block_vs_brute_force():
    rng = np.random.default_rng(1)
    blocks = [rng.standard_normal(16) * 10 ** rng.uniform(-4, 2) for _ in range(300)]
    blocks += [rng.uniform(0, 448, 16), np.full(16, 6.0), np.zeros(16), np.r_[np.zeros(15), 1e-6],
               np.r_[448.0, np.zeros(15)], rng.standard_normal(7) * 3]
    for b in blocks:
        x = np.asarray(b, np.float32)
        codes, scale = oracle.nvfp4_blocks(x[None])
        ref_codes, ref_scale = _brute_block(x)
        assert scale[0] == ref_scale
        np.testing.assert_array_equal(codes[0], ref_codes)


def test_nvfp4_block_worked_example():
    # amax 6 -> scale E4M3(1.0) = 0x38, codes are plain E2M1 of x
    x = np.array([6, -3, 1.5, 0.25, 0.75, -0.5, 4, 2.5, 0, 1, -6, 5, 3.5, -1.25, 0.1, 2], np.float32)
    codes, scale = oracle.nvfp4_blocks(x[None])
    assert scale[0] == 0x38
    np.testing.assert_array_equal(codes[0], x.astype(F4).view(np.uint8))
    # all-zero block: zero scale, zero codes
    codes, scale = oracle.nvfp4_blocks(np.zeros((1, 16), np.float32))
    assert scale[0] == 0 and not codes.any()


@pytest.mark.parametrize("smooth", [True, False])
def test_smooth_v_nvfp4_matches_its_definition(smooth):
    w = synth.WORKLOADS["tiny_1k_d64"]
    k, v = synth.head_bits(w, "k", 0, 0), synth.head_bits(w, "v", 0, 0)
    n, d = v.shape
    bk = 64
    if smooth:
        labels, _ = oracle.kmeans(v, w.C, w.iters)
        perm = oracle.stable_perm(labels, w.C)
    else:
        perm = np.arange(n, dtype=np.int32)
    vq, vgs, vmu, vsc = oracle.smooth_v_nvfp4(v, perm, bk, smooth)
    vhat, vmu8, vsc8 = oracle.smooth_v(v, perm, bk, smooth)
    np.testing.assert_array_equal(vmu, vmu8)  # same block means as the E4M3 residual
    vals = bf16_values(v)[perm].astype(np.float32)
    T = n // bk
    res = (vals - np.repeat(vmu, bk, axis=0)).astype(np.float32)
    amax = np.abs(res).max(axis=0)
    np.testing.assert_array_equal(vsc, np.where(amax > 0, amax / np.float32(2688), 1).astype(np.float32))
    inv = np.where(amax > 0, np.float32(2688) / amax, 0).astype(np.float32)
    y = (res * inv).astype(np.float32)
    # blocks of 16 tokens along the token axis, per channel
    yb = y.reshape(T, bk // 16, 16, d).transpose(0, 1, 3, 2)
    codes, scales = oracle.nvfp4_blocks(yb)
    np.testing.assert_array_equal(vgs, scales)
    np.testing.assert_array_equal(vq, codes.transpose(0, 1, 3, 2).reshape(n, d))
    # coded values stay within half an E2M1 step (at most 1) times the block scale
    deq = oracle.nvfp4_v_values(vq, vgs)
    bound = np.repeat(oracle.e4m3_value(vgs), 16, axis=1).reshape(n, d) * 1.0 + 1e-30
    assert np.all(np.abs(deq - y) <= bound * 1.0000001 + np.abs(y) * 0.07)


def _replay_nvfp4_rows(qv, sq, kv, ksc, rv, vmu, vsc, n, bk, beta):
    """Online replay in Python for a few rows, P re-coded per 16 keys."""
    d = qv.shape[1]
    T = -(-n // bk)
    kap = np.float32(oracle.kappa(d))
    outs = []
    for i in range(qv.shape[0]):
        M, l, first = 0.0, 0.0, True
        ores = np.zeros(d)
        omean = np.zeros(d)
        for b in range(T):
            valid = min(bk, n - b * bk)
            A = np.float32(kap * np.float32(sq[i])) * np.float32(ksc[b])
            s = (kv[b * bk:b * bk + valid] @ qv[i]).astype(np.float32)
            Mc = np.ceil(float(np.float32(A * s.max())) / 8.0)
            Mnew = Mc if first else max(M, Mc)
            if not first and Mnew > M:
                f = 2.0 ** -(Mnew - M)
                ores *= f
                omean *= f
                l *= f
            M, first = Mnew, False
            cb = np.float32(56 + beta - 8 * M)
            p8 = oracle.e4m3_value(oracle.expcast_bytes(np.full(valid, A, np.float32), s, np.full(valid, cb)))
            x = np.zeros(bk, np.float32)
            x[:valid] = p8
            codes, sc = oracle.nvfp4_blocks(x.reshape(bk // 16, 16))
            p = (oracle.e4m3_value(sc)[:, None] * oracle.e2m1_value(codes)).reshape(bk)[:valid]
            ores += p @ rv[b * bk:b * bk + valid]
            omean += p.sum() * vmu[b].astype(np.float64)
            l += p.sum()
        outs.append((vsc * ores + omean) / l)
    return np.array(outs)


def test_attn_replay_nvfp4_p_vs_python_replay():
    w = synth.custom("nvfp4_pin", 1, 1, 200, 64, 5, pool=6, C=6, iters=3, block=64)
    q, k, v = (synth.head_bits(w, t, 0, 0) for t in "qkv")
    n, d = k.shape
    prep = oracle.prep_head(k, v, C=w.C, iters=w.iters, bk=64, resid_fmt=1)
    rows = np.arange(0, n, 23)
    qhat, sq = oracle.quant_q(q[rows])
    qv = oracle.e4m3_value(qhat)
    kv = oracle.e4m3_value(prep["khat"])
    rv = oracle.nvfp4_v_values(prep["vq"], prep["vgs"])
    out, M, l = oracle.attn_emul(qv, sq, kv, prep["ksc"], rv, prep["vmu"], prep["vsc"], n=n, bk=64, beta=64,
                                 pfmt=1)
    ref = _replay_nvfp4_rows(qv, sq, kv, prep["ksc"], rv, prep["vmu"], prep["vsc"], n, 64, 64)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    # and the 4-bit path stays near the 8-bit one and near exact attention
    r8 = oracle.forward_head(q, k, v, rows, C=w.C, iters=w.iters, bk=64, beta=64)["out"]
    exact = oracle.attn_exact(q, k, v, rows)
    ref_norm = np.linalg.norm(exact)
    assert np.linalg.norm(out - exact) / ref_norm < 0.2
    assert np.linalg.norm(out - r8) / ref_norm < 0.2


def torch_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (uint16), rounded by torch."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).bfloat16().view(torch.int16).numpy().view(np.uint16)


def _pin_head():
    w = synth.custom("nvfp4_pin", 1, 1, 200, 64, 5, pool=6, C=6, iters=3, block=64)
    return w, [synth.head_bits(w, t, 0, 0) for t in "qkv"]


@pytest.mark.parametrize("resid_fmt", [0, 1])
def test_q_zero_closed_form(resid_fmt):
    """Q = 0 makes every score 0, so M = 0 and every ExpCast byte is 56 + beta
    = 120 (value 256).  In the 8-bit path P = 256.  In the 4-bit path each
    16-key block of 256s takes the scale E4M3(256/6) = 44 (nearest of 40, 44)
    and the code E2M1(256/44 = 5.82) = 6, so P = 264, worked out by hand.  P is
    the same for every key, so the output is the plain mean of the dequantised
    V, and l = P * n.  The 200 keys leave a ragged last block of 8."""
    w, (q, k, v) = _pin_head()
    n, d = k.shape
    rows = np.arange(0, n, 9)
    r = oracle.forward_head(np.zeros((n, d), np.uint16), k, v, rows, C=w.C, iters=w.iters, bk=64, beta=64,
                            resid_fmt=resid_fmt)
    np.testing.assert_array_equal(r["M"], 0)
    np.testing.assert_array_equal(r["l"], (264.0 if resid_fmt else 256.0) * n)
    prep = r["prep"]
    rv = oracle.nvfp4_v_values(prep["vq"], prep["vgs"]) if resid_fmt else oracle.e4m3_value(prep["vhat"])
    deq = np.repeat(prep["vmu"].astype(np.float64), 64, 0)[:n] + prep["vsc"] * rv[:n]
    np.testing.assert_allclose(r["out"], np.broadcast_to(deq.mean(0), r["out"].shape), rtol=1e-12, atol=1e-12)
    # and near the mean of V itself: each coded residual lies within half an
    # E2M1 step (at most one block-scale unit, 6.25% more for the scale's own
    # rounding) of the true one, and E4M3 within 1/16 of amax
    if resid_fmt:
        unit = prep["vsc"] * np.repeat(oracle.e4m3_value(prep["vgs"]), 16, axis=1).reshape(-1, d).max(0)
        tol = unit * 1.07
    else:
        tol = prep["vsc"] * 448.0 / 16
    assert np.all(np.abs(r["out"][0] - bf16_values(v).mean(0)) <= tol + 1e-9)


@pytest.mark.parametrize("resid_fmt", [0, 1])
def test_v_constant_per_channel_closed_form(resid_fmt):
    """V constant along the tokens: every block mean is that constant, the
    residual is 0 (all codes 0), and O = sum_b l_b mu / sum_b l_b is the
    constant again, whatever Q and K are."""
    w, (q, k, _) = _pin_head()
    n, d = k.shape
    c = (np.random.default_rng(8).standard_normal(d)).astype(np.float32)
    cb = torch_bf16_bits(c)
    v = np.broadcast_to(cb, (n, d)).copy()
    r = oracle.forward_head(q, k, v, np.arange(0, n, 7), C=w.C, iters=w.iters, bk=64, beta=64, resid_fmt=resid_fmt)
    prep = r["prep"]
    assert not np.any(prep["vq"] if resid_fmt else prep["vhat"])
    np.testing.assert_allclose(r["out"], np.broadcast_to(bf16_values(cb), r["out"].shape), rtol=1e-12, atol=0)


@pytest.mark.parametrize("resid_fmt", [0, 1])
def test_single_token_returns_its_value(resid_fmt):
    """One key: the block mean is the token itself, the residual is 0, and the
    output is v_0 exactly (bf16 values, products by P exact in fp64)."""
    rng = np.random.default_rng(9)
    q, k, v = (torch_bf16_bits(rng.standard_normal((1, 128)).astype(np.float32)) for _ in range(3))
    r = oracle.forward_head(q, k, v, np.arange(1), C=1, iters=2, bk=128, beta=64, resid_fmt=resid_fmt)
    np.testing.assert_array_equal(r["out"], bf16_values(v))


def test_nvfp4_code_uses_the_fp32_reciprocal_of_the_scale():
    """Worked by hand.  The block {22.5, 4.6875} has amax/6 = 3.75, an E4M3
    value (code 0x47), so the scale is exact.  Divided exactly, 4.6875/3.75 =
    1.25 is an E2M1 tie that goes to the even code 2 (value 1.0).  The reading
    taken codes x * RN(1/s): RN(1/3.75) lies above 1/3.75, the product
    rounds to 1.2500001 in fp32, past the tie, and the code is 3 (value 1.5)."""
    from fractions import Fraction

    x = np.zeros(16, np.float32)
    x[0], x[1] = 22.5, 4.6875
    codes, scale = oracle.nvfp4_blocks(x[None])
    assert scale[0] == 0x47 and oracle.e4m3_value(scale)[0] == 3.75
    assert Fraction(4.6875) / Fraction(3.75) == Fraction(5, 4)  # the exact quotient is the tie
    r = np.float32(1.0) / np.float32(3.75)
    assert np.float32(np.float32(4.6875) * r) > np.float32(1.25)
    np.testing.assert_array_equal(codes[0][:2], [7, 3])
    assert not codes[0][2:].any()


def test_crafted_tie_blocks():
    """On the crafted tie workload (V-Smooth off) the channel scales are 1,
    each block takes the scale it was built with, and every code follows
    the reading: an exact E2M1 tie of y * RN(1/s) goes to the even code, and
    a value that only the exact quotient would put on a tie rounds from the
    fp32 product.  Both kinds occur by the thousand."""
    from conftest import nvfp4_tie_values

    v, scales = nvfp4_tie_values(21)
    vb = torch_bf16_bits(v)
    assert np.array_equal(bf16_values(vb), v.astype(np.float64))  # bf16-exact
    n, d = v.shape
    vq, vgs, vmu, vsc = oracle.smooth_v_nvfp4(vb, np.arange(n, dtype=np.int32), 128, False)
    assert np.all(vsc == 1.0) and not vmu.any()
    np.testing.assert_array_equal(oracle.e4m3_value(vgs).reshape(-1, d), scales)
    sv = np.repeat(scales, 16, axis=0).astype(np.float32)
    prod = (v * (np.float32(1.0) / sv)).astype(np.float32).astype(np.float64)
    quotient = v.astype(np.float64) / sv
    mags = np.abs(prod)
    tie = np.isin(mags, (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0))
    witness = ~tie & np.isin(np.abs(quotient), (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0))
    assert tie.sum() > 1000 and witness.sum() > 1000, (tie.sum(), witness.sum())
    got = oracle.e2m1_value(vq)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    lo = grid[np.searchsorted(grid, mags, side="right") - 1]
    hi = grid[np.minimum(np.searchsorted(grid, mags, side="right"), 7)]
    lo_even = np.isin(lo, (0.0, 1.0, 2.0, 4.0))  # codes 0, 2, 4, 6
    want_tie = np.where(lo_even, lo, hi) * np.sign(prod)
    np.testing.assert_array_equal(got[tie], want_tie[tie])
    nearest = np.where(mags - lo < hi - mags, lo, hi) * np.sign(prod)
    np.testing.assert_array_equal(got[witness], nearest[witness])
