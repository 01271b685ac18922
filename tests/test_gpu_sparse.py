"""GPU parity of the block-sparse attention (vc_attn_fwd_masked): key tiles
dropped per query tile by a mask (the pages: VC-Attention stacks with sparse
attention).  The kernel is fed the oracle's own prep and compared with the
oracle's masked replay (rel-L2 <= 3e-3, cosine >= 0.99999); rows whose key
tiles are all dropped are exactly 0; an all-ones mask is bit-identical to the
dense call."""
import numpy as np
import pytest
import torch

import oracle
from bit_fp8_attention_smooth_b200 import synth
from gpu_common import BETA, bits, make_inputs, metrics, oracle_head, oracle_prep_to_gpu

pytestmark = pytest.mark.gpu

CASES = [
    synth.custom("sparse_ragged_300_d128", 1, 2, 300, 128, 71, pool=8, C=8, iters=4, block=128),
    synth.custom("sparse_1000_d64_bk128", 2, 1, 1000, 64, 72, pool=12, C=12, iters=4, block=128),
    synth.custom("sparse_777_d128_bk64", 1, 2, 777, 128, 73, pool=10, C=10, iters=4, block=64),
    synth.custom("sparse_2100_d128", 1, 1, 2100, 128, 74, pool=16, C=16, iters=4, block=128),
]


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


def _mask(w, seed):
    Tq, T = -(-w.N // 128), -(-w.N // w.block)
    m = (np.random.default_rng(seed).random((w.B, w.H, Tq, T)) < 0.5).astype(np.uint8)
    m[0, 0, 0] = 0          # a query tile that keeps no key tile
    m[0, -1, -1, -1] = 1    # the ragged last key tile kept somewhere
    if Tq > 1:
        m[0, 0, 1] = 1      # and a dense query tile
    return m


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_masked_kernel_matches_masked_replay(vc, w):
    q, k, v, qd, kd, vd = make_inputs(w)
    rows = np.arange(w.N)
    preps = [[oracle_head(q, k, v, b, h, rows[:1], w)["prep"] for h in range(w.H)] for b in range(w.B)]
    params = vc.Params.for_workload(w, beta=BETA)
    gprep = oracle_prep_to_gpu(preps, tuple(q.shape), w.block)
    mask = _mask(w, 5)
    ws = vc.alloc_workspace(tuple(q.shape), params)
    out = vc.attn_fwd(qd, gprep, params, workspace=ws, tile_mask=torch.from_numpy(mask).cuda())
    vc.check(ws)
    out = out.float().cpu().numpy()
    for b in range(w.B):
        for h in range(w.H):
            ref = oracle.forward_head(bits(q[b, h]), bits(k[b, h]), bits(v[b, h]), rows, C=w.C, iters=w.iters,
                                      bk=w.block, beta=BETA, prep=preps[b][h], tile_mask=mask[b, h])["out"]
            empty = mask[b, h][rows // 128].sum(axis=1) == 0
            assert np.all(out[b, h][empty] == 0) and np.all(ref[empty] == 0)
            if (~empty).any():
                rel, cos, _ = metrics(out[b, h][~empty], ref[~empty])
                assert rel <= 3e-3 and cos >= 0.99999, (b, h, rel, cos)


def test_all_ones_mask_is_the_dense_call(vc):
    w = CASES[3]
    q, k, v, qd, kd, vd = make_inputs(w)
    params = vc.Params.for_workload(w, beta=BETA)
    ws = vc.alloc_workspace(tuple(q.shape), params)
    prep = vc.smooth_prepare(kd, vd, params, workspace=ws)
    dense = vc.attn_fwd(qd, prep, params, workspace=ws)
    ones = torch.ones((w.B, w.H, -(-w.N // 128), -(-w.N // w.block)), dtype=torch.uint8, device="cuda")
    masked = vc.attn_fwd(qd, prep, params, workspace=ws, tile_mask=ones)
    vc.check(ws)
    assert torch.equal(dense, masked)


def test_mask_argument_checks(vc):
    w = CASES[0]
    q, k, v, qd, kd, vd = make_inputs(w)
    params = vc.Params.for_workload(w, beta=BETA)
    prep = vc.smooth_prepare(kd, vd, params)
    with pytest.raises(ValueError):
        vc.attn_fwd(qd, prep, params, tile_mask=torch.ones((1, 2, 3), dtype=torch.uint8, device="cuda"))
    p4 = vc.Params.for_workload(w, beta=BETA, resid_fmt=1)
    prep4 = vc.smooth_prepare(kd, vd, p4)
    with pytest.raises(vc.VcError) as e:
        vc.attn_fwd(qd, prep4, p4, tile_mask=torch.ones((1, 2, 3, 3), dtype=torch.uint8, device="cuda"))
    assert e.value.status == vc.VC_ERR_UNSUPPORTED
