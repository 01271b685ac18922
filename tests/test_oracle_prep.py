"""Pins of the oracle's V-Smooth prep (k-means, stable regroup, Q/K/V
quantisation) against library routines (scipy, scikit-learn, numpy, torch),
Lloyd's invariants and closed forms."""
import numpy as np
import torch

import oracle
from bit_fp8_attention_smooth_b200 import synth
from conftest import bf16_values

TINY = synth.WORKLOADS["tiny_1k_d64"]


def tiny_head(h=0):
    return [synth.head_bits(TINY, t, 0, h) for t in "qkv"]


def small_pool(n, d, seed, pool=8):
    w = synth.custom("pin", 1, 1, n, d, seed, pool=pool, C=pool)
    return synth.head_bits(w, "v", 0, 0)


def test_kmeans_labels_are_argmin_vs_scipy():
    from scipy.cluster.vq import vq

    v = small_pool(777, 64, 3)
    labels, cent = oracle.kmeans(v, 8, 5)
    ref, _ = vq(bf16_values(v), cent)
    assert np.array_equal(labels, ref)


def test_kmeans_strided_init():
    from scipy.cluster.vq import vq

    v = small_pool(500, 64, 4)
    C = 7
    labels, cent = oracle.kmeans(v, C, 1)
    init = bf16_values(v)[[(k * 500) // C for k in range(C)]]
    assert np.array_equal(cent, init)
    assert np.array_equal(labels, vq(bf16_values(v), init)[0])


def test_kmeans_update_is_member_mean():
    v = small_pool(900, 64, 5)
    x = bf16_values(v)
    for it in (1, 2, 3):
        lab_i, cent_i = oracle.kmeans(v, 8, it)
        _, cent_next = oracle.kmeans(v, 8, it + 1)
        for k in range(8):
            members = x[lab_i == k]
            expect = members.mean(axis=0) if len(members) else cent_i[k]
            np.testing.assert_allclose(cent_next[k], expect, rtol=1e-12, atol=1e-12)


def test_kmeans_objective_non_increasing():
    v = small_pool(1200, 64, 6, pool=12)
    x = bf16_values(v)
    prev = np.inf
    for it in range(1, 7):
        labels, cent = oracle.kmeans(v, 12, it)
        obj = ((x - cent[labels]) ** 2).sum()
        assert obj <= prev * (1 + 1e-12)
        prev = obj


def test_kmeans_vs_sklearn_lloyd():
    from sklearn.cluster import KMeans

    v = small_pool(1024, 64, 7, pool=16)
    x = bf16_values(v)
    C, iters = 16, 8
    init = x[[(k * 1024) // C for k in range(C)]]
    labels, cent = oracle.kmeans(v, C, iters)
    assert np.bincount(labels, minlength=C).min() > 0  # sklearn relocates empty clusters
    km = KMeans(n_clusters=C, init=init, n_init=1, max_iter=iters - 1, tol=0.0, algorithm="lloyd").fit(x)
    agree = (km.labels_ == labels).mean()
    assert agree >= 0.999
    np.testing.assert_allclose(km.cluster_centers_, cent, rtol=0, atol=1e-9)


def test_kmeans_single_cluster_and_tiny_bruteforce():
    v = small_pool(40, 64, 8)
    labels, cent = oracle.kmeans(v, 1, 3)
    assert np.all(labels == 0)
    assert np.array_equal(oracle.stable_perm(labels, 1), np.arange(40))
    # brute force: every 1-D point set of size <= 8 with C = 2: labels are the argmin
    rng = np.random.default_rng(9)
    for _ in range(50):
        n = int(rng.integers(2, 9))
        x = torch.from_numpy(rng.normal(0, 3, (n, 1)).astype(np.float32)).to(torch.bfloat16)
        x = x.repeat(1, 64)  # same value in every channel
        bits = x.view(torch.int16).numpy().view(np.uint16)
        lab, c = oracle.kmeans(bits, 2, 3)
        xv = bf16_values(bits)[:, 0]
        d0, d1 = np.abs(xv - c[0, 0]), np.abs(xv - c[1, 0])
        assert np.array_equal(lab, np.where(d1 < d0, 1, 0))


def _bits(x):
    return torch.tensor(np.asarray(x, np.float32)).bfloat16().view(torch.int16).numpy().view(np.uint16)


def test_kmeans_equidistant_token_goes_to_the_lowest_cluster():
    """Worked by hand.  Tokens 0, 2, 1 with C = 2: the strided init gives
    c_0 = v[0] = 0 and c_1 = v[floor(3/2)] = 2, and token 2 (value 1) is at
    distance 1 from both, so it takes the lower index.  One update moves c_0
    to 0.5 and leaves c_1 at 2, and the second pass keeps those labels.
    Ties to the higher index would give [0, 1, 1] and c_1 = 1.5."""
    v = _bits([[0.0], [2.0], [1.0]])
    labels, cent = oracle.kmeans(v, 2, 1)
    np.testing.assert_array_equal(labels, [0, 1, 0])
    labels, cent = oracle.kmeans(v, 2, 2)
    np.testing.assert_array_equal(labels, [0, 1, 0])
    np.testing.assert_array_equal(cent[:, 0], [0.5, 2.0])
    # in 4 channels with C = 3: the init takes rows 0, 2 and 4, so c_0 and c_2
    # are both the origin and c_1 = (0, 4, 0, 0).  Tokens 1, 4 and 5 tie
    # between c_0 and c_2, and token 3 = (2, 2, 0, 0) is at squared distance 8
    # from all three: every tie goes to cluster 0.
    v = _bits([[0, 0, 0, 0], [4, 0, 0, 0], [0, 4, 0, 0], [2, 2, 0, 0], [0, 0, 0, 0], [0, 0, 0, 0]])
    labels, _ = oracle.kmeans(v, 3, 1)
    np.testing.assert_array_equal(labels, [0, 0, 1, 0, 0, 0])


def test_stable_perm_vs_numpy():
    rng = np.random.default_rng(10)
    for C in (1, 3, 64):
        labels = rng.integers(0, C, 5000).astype(np.int32)
        perm = oracle.stable_perm(labels, C)
        assert np.array_equal(perm, np.argsort(labels, kind="stable"))
        assert np.all(np.diff(labels[perm]) >= 0)


def test_quant_q_and_k_vs_torch_encode():
    q, k, v = tiny_head()
    qhat, sq = oracle.quant_q(q)
    x = bf16_values(q).astype(np.float32)
    amax = np.abs(x).max(axis=1)
    inv = (np.float32(448.0) / amax).astype(np.float32)
    ref = torch.from_numpy((x * inv[:, None]).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(qhat, ref)
    assert np.array_equal(sq, (amax / np.float32(448.0)).astype(np.float32))
    perm = np.random.default_rng(2).permutation(k.shape[0]).astype(np.int32)
    bk = 64
    khat, ksc = oracle.quant_k(k, perm, bk)
    kx = bf16_values(k)[perm].astype(np.float32)
    for b in range(k.shape[0] // bk):
        blk = kx[b * bk:(b + 1) * bk]
        am = np.abs(blk).max()
        assert ksc[b] == np.float32(am) / np.float32(448.0)
        r = torch.from_numpy(blk * (np.float32(448.0) / np.float32(am))).to(torch.float8_e4m3fn).view(torch.uint8)
        assert np.array_equal(khat[b * bk:(b + 1) * bk], r.numpy())
        assert np.abs(oracle.e4m3_value(khat[b * bk:(b + 1) * bk])).max() == 448.0


def test_quant_k_ragged_tail_and_padding():
    w = synth.custom("rag", 1, 1, 300, 64, 11)
    k = synth.head_bits(w, "k", 0, 0)
    perm = np.arange(300, dtype=np.int32)
    khat, ksc = oracle.quant_k(k, perm, 128)
    assert khat.shape == (384, 64) and ksc.shape == (3,)
    assert np.all(khat[300:] == 0)
    assert np.float32(np.abs(bf16_values(k)[256:300]).max()) / np.float32(448) == ksc[2]


def test_smooth_v_mean_and_residual():
    q, k, v = tiny_head(1)
    prep = oracle.prep_head(k, v, C=16, iters=8, bk=64)
    perm, vmu, vsc, vhat = prep["perm"], prep["vmu"], prep["vsc"], prep["vhat"]
    x = bf16_values(v)[perm]
    for b in range(16):
        mean = x[b * 64:(b + 1) * 64].mean(axis=0).astype(np.float32)
        np.testing.assert_array_max_ulp(vmu[b], mean, maxulp=1)
    res = (x.astype(np.float32) - np.repeat(vmu, 64, axis=0)).astype(np.float32)
    amax = np.abs(res).max(axis=0)
    np.testing.assert_array_equal(vsc, amax / np.float32(448.0))
    ref = torch.from_numpy((res * (np.float32(448.0) / amax)[None, :]).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(vhat, ref.view(torch.uint8).numpy())


def test_smooth_off_is_plain_per_channel():
    q, k, v = tiny_head(0)
    perm = np.arange(1024, dtype=np.int32)
    vhat, vmu, vsc = oracle.smooth_v(v, perm, 64, smooth=False)
    assert np.all(vmu == 0)
    x = bf16_values(v).astype(np.float32)
    np.testing.assert_array_equal(vsc, np.abs(x).max(axis=0) / np.float32(448.0))


def test_vsmooth_lowers_v_quantisation_error():
    """The pages' claim, at tensor level: subtracting block means of clustered
    tokens leaves a residual that quantises with less error than plain
    per-channel FP8 V (chooseai.io news 7051, V-Smooth section)."""
    for name, h in (("tiny_1k_d64", 0), ("tiny_1k_d64", 1)):
        w = synth.WORKLOADS[name]
        k, v = synth.head_bits(w, "k", 0, h), synth.head_bits(w, "v", 0, h)
        x = bf16_values(v)
        on = oracle.prep_head(k, v, C=w.C, iters=w.iters, bk=w.block, smooth=True)
        rec_on = np.repeat(on["vmu"], w.block, 0)[: w.N] + on["vsc"] * oracle.e4m3_value(on["vhat"])[: w.N]
        err_on = np.linalg.norm(rec_on - x[on["perm"]])
        off = oracle.prep_head(k, v, C=w.C, iters=w.iters, bk=w.block, smooth=False)
        rec_off = off["vsc"] * oracle.e4m3_value(off["vhat"])[: w.N]
        err_off = np.linalg.norm(rec_off - x)
        assert err_on < 0.8 * err_off, (err_on, err_off)
