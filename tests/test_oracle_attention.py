"""Pins of the oracle's attention replay: torch's fp64 attention for the exact
reference, the identity-quantiser special case (mean restore from row sums is
exact algebra, chooseai.io news 7051 V-Smooth section), closed forms (V == 1,
Q == 0), permutation invariance and tiling invariance of the integer row
reference."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_fp8_attention_smooth_b200 import synth
from conftest import bf16_values

TINY = synth.WORKLOADS["tiny_1k_d64"]
BETA = 64


def heads(w=TINY, h=0):
    return [synth.head_bits(w, t, 0, h) for t in "qkv"]


def sdpa(q, k, v):
    qt, kt, vt = (torch.from_numpy(bf16_values(x))[None, None] for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, 0].numpy()


def test_exact_attention_vs_torch():
    q, k, v = heads()
    rows = np.arange(0, 1024, 7)
    ours = oracle.attn_exact(q, k, v, rows)
    ref = sdpa(q, k, v)[rows]
    np.testing.assert_allclose(ours, ref, rtol=1e-10, atol=1e-12)


def _raw_layout(k, v, perm, vmu, bk):
    n, d = k.shape
    T = -(-n // bk)
    kraw = np.zeros((T * bk, d))
    kraw[:n] = bf16_values(k)[perm]
    vraw = np.zeros((T * bk, d))
    vraw[:n] = bf16_values(v)[perm]
    res = vraw - np.repeat(vmu.astype(np.float64), bk, axis=0)
    res[n:] = 0
    return kraw, res


@pytest.mark.parametrize("h", [0, 1])
def test_identity_quantiser_equals_exact(h):
    """With no quantisation and the exact exponential, regrouping, block-mean
    subtraction and the l_b * mu_b restore reproduce plain attention."""
    q, k, v = heads(h=h)
    n, d = k.shape
    prep = oracle.prep_head(k, v, C=TINY.C, iters=TINY.iters, bk=64)
    kraw, res = _raw_layout(k, v, prep["perm"], prep["vmu"], 64)
    T = n // 64
    out, M, l = oracle.attn_emul(bf16_values(q), np.ones(n, np.float32), kraw, np.ones(T, np.float32), res,
                                 prep["vmu"], np.ones(d, np.float32), n=n, bk=64, beta=BETA, exact=True)
    ref = sdpa(q, k, v)
    np.testing.assert_allclose(out, ref, rtol=1e-9, atol=1e-11)
    # the integer row reference is the ceiling of the row's max in byte units / 8
    s = bf16_values(q) @ bf16_values(k).T * (8.0 / (math.log(2.0) * math.sqrt(d)))
    np.testing.assert_array_equal(M, np.ceil(s.max(axis=1) / 8.0))


def test_v_ones_gives_ones():
    q, k, _ = heads()
    n, d = k.shape
    ones = torch.ones(n, d, dtype=torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    r = oracle.forward_head(q, k, ones, np.arange(0, n, 5), C=16, iters=3, bk=64, beta=BETA)
    assert np.all(r["prep"]["vhat"] == 0)
    np.testing.assert_array_equal(r["out"], np.ones_like(r["out"]))


def test_q_zero_gives_mean_v():
    _, k, v = heads()
    n, d = k.shape
    zeros = np.zeros((n, d), np.uint16)
    r = oracle.forward_head(zeros, k, v, np.arange(0, n, 9), C=16, iters=4, bk=64, beta=BETA)
    prep = r["prep"]
    deq = np.repeat(prep["vmu"].astype(np.float64), 64, 0)[:n] + prep["vsc"] * oracle.e4m3_value(prep["vhat"])[:n]
    np.testing.assert_allclose(r["out"], np.broadcast_to(deq.mean(0), r["out"].shape), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["out"][0], bf16_values(v).mean(0), rtol=0, atol=2e-2)


def test_scores_round_to_fp32_before_expcast():
    """Worked by hand, on the replay with A = 1 (kappa = 1, unit scales).  Two
    keys in one tile: scores 8 and 4.5 + 2^-30.  The max gives M = ceil(8/8) =
    1, so cb = 56 + 64 - 8 = 112.  Byte 0 is 120 (value 256).  The second
    score rounds to 4.5 in fp32, t = 116.5 is a tie and goes to the even byte
    116 (0x74, value 1.5 * 2^7 = 192); unrounded it would be byte 117 (208).
    So l = 448 and O = (256 v_0 + 192 v_1)/448."""
    d, bk = 2, 16
    qv = np.array([[1.0, 1.0]])
    kv = np.zeros((bk, d))
    kv[0] = [8.0, 0.0]
    kv[1] = [4.5, 2.0 ** -30]
    rv = np.zeros((bk, d))
    rv[0] = [1.0, 0.0]
    rv[1] = [0.0, 1.0]
    out, M, l = oracle.attn_emul(qv, np.ones(1, np.float32), kv, np.ones(1, np.float32), rv, np.zeros((1, d)),
                                 np.ones(d, np.float32), n=2, bk=bk, beta=BETA, kappa_value=1.0)
    assert M[0] == 1 and l[0] == 448.0
    np.testing.assert_array_equal(out[0], [256.0 / 448.0, 192.0 / 448.0])


def test_row_reference_of_a_row_of_negative_scores():
    """Worked by hand, A = 1: scores -20 and -24 in the first (only) tile give
    M = ceil(-20/8) = -2, taken as it is (not raised from 0), so cb = 56 + 64
    + 16 = 136 and the bytes are 116 (192) and 112 (0x70, 128): l = 320 and
    O = (192 v_0 + 128 v_1)/320."""
    d, bk = 2, 16
    kv = np.zeros((bk, d))
    kv[0, 0], kv[1, 0] = -20.0, -24.0
    rv = np.zeros((bk, d))
    rv[0] = [1.0, 0.0]
    rv[1] = [0.0, 1.0]
    out, M, l = oracle.attn_emul(np.array([[1.0, 0.0]]), np.ones(1, np.float32), kv, np.ones(1, np.float32), rv,
                                 np.zeros((1, d)), np.ones(d, np.float32), n=2, bk=bk, beta=BETA, kappa_value=1.0)
    assert M[0] == -2 and l[0] == 320.0
    np.testing.assert_array_equal(out[0], [0.6, 0.4])


def test_joint_permutation_invariance():
    q, k, v = heads()
    n = k.shape[0]
    rows = np.arange(0, n, 11)
    perm = np.random.default_rng(3).permutation(n)
    exact = oracle.attn_exact(q, k, v, rows)
    exact_p = oracle.attn_exact(q, k[perm], v[perm], rows)
    np.testing.assert_allclose(exact, exact_p, rtol=1e-11, atol=1e-13)
    a = oracle.forward_head(q, k, v, rows, C=16, iters=8, bk=64, beta=BETA)["out"]
    b = oracle.forward_head(q, k[perm], v[perm], rows, C=16, iters=8, bk=64, beta=BETA)["out"]
    # quantised paths: regrouping changes the per-block K scales, so the two runs
    # differ by about the FP8 error level, and both stay within it of exact
    ref = np.linalg.norm(exact)
    assert np.linalg.norm(a - exact) / ref < 0.12 and np.linalg.norm(b - exact) / ref < 0.12
    assert np.linalg.norm(a - b) / ref < 0.15


def test_tiling_does_not_change_bytes_beyond_underflow():
    """The integer reference rises in whole steps, so a tile's bytes shift by
    multiples of 8 and decode to exact powers of two: one tile or sixteen give
    the same softmax as long as no weight underflows.  Keys ramp up over the
    tiles so the reference rises mid-row, and stay inside 12 octaves of the max."""
    q, k, v = heads()
    n, d = k.shape
    rng = np.random.default_rng(4)
    qhat, sq = oracle.quant_q(q[:64])
    qv = oracle.e4m3_value(qhat)
    u = qv[0] / np.linalg.norm(qv[0])
    ramp = np.repeat(np.arange(n // 64), 64)[:, None] / 16.0
    kv = ramp * u[None, :] * 6.0 + rng.standard_normal((n, d)) * 0.05
    kv = oracle.e4m3_value(oracle.e4m3_encode(kv.astype(np.float32)))
    rv = bf16_values(v)
    args = dict(rv=rv, vsc=np.ones(d, np.float32))
    one_t = oracle.attn_emul(qv, sq, kv, np.ones(1, np.float32), rv, np.zeros((1, d), np.float32),
                             np.ones(d, np.float32), n=n, bk=n, beta=BETA)
    tiled = oracle.attn_emul(qv, sq, kv, np.ones(n // 64, np.float32), rv, np.zeros((n // 64, d), np.float32),
                             np.ones(d, np.float32), n=n, bk=64, beta=BETA)
    first = oracle.attn_emul(qv, sq, kv[:64], np.ones(1, np.float32), rv[:64], np.zeros((1, d), np.float32),
                             np.ones(d, np.float32), n=64, bk=64, beta=BETA)
    # rows whose every key stays a normal byte under the final reference
    A = (np.float32(oracle.kappa(d)) * sq).astype(np.float64)
    s32 = (qv @ kv.T).astype(np.float32).astype(np.float64)
    tmin = (A[:, None] * s32).min(1) + 56 + BETA - 8 * one_t[1]
    ok = tmin >= 8.5
    rising = ok & (first[1] < one_t[1])
    assert ok.sum() >= 16 and rising.sum() >= 8
    np.testing.assert_array_equal(tiled[1], one_t[1])
    np.testing.assert_allclose(tiled[0][ok], one_t[0][ok], rtol=1e-12, atol=1e-12)


def test_quantised_error_budget():
    """Error vs exact attention splits into the FP8 Q/K, ExpCast and FP8 V
    parts; each is bounded, and ExpCast alone (exact Q/K/V) costs a few percent."""
    q, k, v = heads()
    n, d = k.shape
    rows = np.arange(n)
    ref = sdpa(q, k, v)
    full = oracle.forward_head(q, k, v, rows, C=16, iters=8, bk=64, beta=BETA)
    rel = np.linalg.norm(full["out"] - ref) / np.linalg.norm(ref)
    assert rel < 0.15
    prep = full["prep"]
    kraw, res = _raw_layout(k, v, prep["perm"], prep["vmu"], 64)
    only_expcast = oracle.attn_emul(bf16_values(q), np.ones(n, np.float32), kraw, np.ones(16, np.float32), res,
                                    prep["vmu"], np.ones(d, np.float32), n=n, bk=64, beta=BETA,
                                    kappa_value=8.0 / (math.log(2.0) * math.sqrt(d)))[0]
    rel_e = np.linalg.norm(only_expcast - ref) / np.linalg.norm(ref)
    assert 1e-3 < rel_e < 0.04
    assert np.all(full["l"] > 0)
