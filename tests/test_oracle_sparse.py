"""Pins of the replay's block-sparse tile mask (the pages: VC-Attention stacks
with sparse attention, chooseai.io news 7051, 意义与局限).  Dropping a key
tile must be the same as removing its keys: the replay over a mask equals the
dense replay over the kept tiles only, bit for bit, and keeps the ragged tail
last; an all-ones mask changes nothing; a row with no tile left outputs 0."""
import numpy as np

import oracle
from bit_fp8_attention_smooth_b200 import synth

BK = 64


def _inputs(n=1000, seed=7):
    w = synth.custom("sparse_pin", 1, 1, n, 64, seed, pool=8, C=8, iters=3, block=BK)
    q, k, v = (synth.head_bits(w, t, 0, 0) for t in "qkv")
    prep = oracle.prep_head(k, v, C=w.C, iters=w.iters, bk=BK)
    qhat, sq = oracle.quant_q(q[:64])
    return (oracle.e4m3_value(qhat), sq, oracle.e4m3_value(prep["khat"]), prep["ksc"],
            oracle.e4m3_value(prep["vhat"]), prep["vmu"], prep["vsc"], n)


def test_all_ones_mask_is_dense():
    qv, sq, kv, ksc, rv, vmu, vsc, n = _inputs()
    T = -(-n // BK)
    dense = oracle.attn_emul(qv, sq, kv, ksc, rv, vmu, vsc, n=n, bk=BK, beta=64)
    ones = oracle.attn_emul(qv, sq, kv, ksc, rv, vmu, vsc, n=n, bk=BK, beta=64,
                            rowmask=np.ones((qv.shape[0], T), np.uint8))
    for a, b in zip(dense, ones):
        np.testing.assert_array_equal(a, b)


def test_dropping_tiles_equals_removing_their_keys():
    qv, sq, kv, ksc, rv, vmu, vsc, n = _inputs()
    T = -(-n // BK)  # 16 tiles, the last with 40 keys
    keep = [0, 3, 4, 9, 15]
    mask = np.zeros((qv.shape[0], T), np.uint8)
    mask[:, keep] = 1
    masked = oracle.attn_emul(qv, sq, kv, ksc, rv, vmu, vsc, n=n, bk=BK, beta=64, rowmask=mask)
    sel = np.concatenate([np.arange(b * BK, (b + 1) * BK) for b in keep])
    n2 = (len(keep) - 1) * BK + (n - (T - 1) * BK)
    reduced = oracle.attn_emul(qv, sq, kv[sel], ksc[keep], rv[sel], vmu[keep], vsc, n=n2, bk=BK, beta=64)
    for a, b in zip(masked, reduced):
        np.testing.assert_array_equal(a, b)


def test_row_without_tiles_outputs_zero():
    qv, sq, kv, ksc, rv, vmu, vsc, n = _inputs()
    T = -(-n // BK)
    mask = np.ones((qv.shape[0], T), np.uint8)
    mask[5] = 0
    out, M, l = oracle.attn_emul(qv, sq, kv, ksc, rv, vmu, vsc, n=n, bk=BK, beta=64, rowmask=mask)
    assert not out[5].any() and l[5] == 0
    assert np.all(l[np.arange(len(l)) != 5] > 0)
