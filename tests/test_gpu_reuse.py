"""The reuse mode of the prep (Params.smooth = 2): a later step keeps the
regroup an earlier step's k-means produced and quantises its own K and V in
that order.  Parity against the oracle's quantisers given the same order:
bit-exact prep bytes; the attention within the end-to-end tolerance."""
import numpy as np
import pytest
import torch

import oracle
from bit_fp8_attention_smooth_b200 import synth
from gpu_common import BETA, COS_TOL, REL_L2_TOL, bits, gpu_prep_head, metrics, prep_to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


def _two_steps(seed_a, seed_b, N=700, d=128, H=2, bk=128):
    a = synth.custom(f"reuse_a_{N}", 1, H, N, d, seed_a, pool=8, C=8, iters=5, block=bk)
    b = synth.custom(f"reuse_b_{N}", 1, H, N, d, seed_b, pool=8, C=8, iters=5, block=bk)
    return a, b


@pytest.mark.parametrize("resid_fmt", [0, 1], ids=["e4m3", "nvfp4"])
def test_reuse_keeps_the_regroup_and_matches_oracle(vc, resid_fmt):
    wa, wb = _two_steps(61, 62)
    qa, ka, va = (synth.tensor_bf16(wa, t) for t in "qkv")
    qb, kb, vb = (synth.tensor_bf16(wb, t) for t in "qkv")
    shape = tuple(qa.shape)
    p1 = vc.Params.for_workload(wa, beta=BETA, resid_fmt=resid_fmt)
    ws = vc.alloc_workspace(shape, p1)
    prep = vc.smooth_prepare(ka.cuda(), va.cuda(), p1, workspace=ws)
    vc.check(ws)
    perm_a = prep["perm"].cpu().numpy().copy()
    p2 = vc.Params.for_workload(wb, beta=BETA, resid_fmt=resid_fmt, smooth=2)
    vc.smooth_prepare(kb.cuda(), vb.cuda(), p2, prep=prep, workspace=ws)
    out = vc.attn_fwd(qb.cuda(), prep, p2, workspace=ws).float().cpu().numpy()
    vc.check(ws)
    host = prep_to_host(prep)
    assert np.array_equal(host["perm"].numpy(), perm_a)  # the regroup was kept
    rows = np.arange(wb.N)
    for h in range(wb.H):
        perm = perm_a[0, h]
        khat, ksc = oracle.quant_k(bits(kb[0, h]), perm, wb.block)
        assert np.array_equal(host["k_fp8"][0, h].numpy(), khat)
        assert np.array_equal(host["k_scale"][0, h].numpy(), ksc)
        if resid_fmt == 1:
            vq, vgs, vmu, vsc = oracle.smooth_v_nvfp4(bits(vb[0, h]), perm, wb.block, True)
            ref_prep = dict(perm=perm, khat=khat, ksc=ksc, vq=vq, vgs=vgs, vmu=vmu, vsc=vsc)
            assert np.array_equal(host["v_bscale"][0, h].numpy().transpose(0, 2, 1), vgs)
        else:
            vhat, vmu, vsc = oracle.smooth_v(bits(vb[0, h]), perm, wb.block, True)
            ref_prep = dict(perm=perm, khat=khat, ksc=ksc, vhat=vhat, vmu=vmu, vsc=vsc)
            assert np.array_equal(gpu_prep_head(host, 0, h, wb.N, wb.block)["vhat"], vhat)
        assert np.array_equal(host["v_mean"][0, h].numpy(), vmu)
        assert np.array_equal(host["v_scale"][0, h].numpy(), vsc)
        ref = oracle.forward_head(bits(qb[0, h]), bits(kb[0, h]), bits(vb[0, h]), rows, C=wb.C, iters=wb.iters,
                                  bk=wb.block, beta=BETA, resid_fmt=resid_fmt, prep=ref_prep)["out"]
        rel, cos, _ = metrics(out[0, h], ref)
        assert rel <= REL_L2_TOL and cos >= COS_TOL, (h, rel, cos)


def test_reuse_with_out_of_range_perm_entries_stays_in_bounds(vc):
    """A caller's perm with entries outside [0, N) is read as token 0 there:
    the gather never leaves the head, and the result matches the oracle's
    quantisers on the clamped order."""
    wa, _ = _two_steps(63, 64, N=300, H=1)
    q, k, v = (synth.tensor_bf16(wa, t) for t in "qkv")
    shape = tuple(q.shape)
    params = vc.Params.for_workload(wa, beta=BETA, smooth=2)
    prep = vc.alloc_prep(shape, params)
    perm = np.random.default_rng(5).permutation(wa.N).astype(np.int32)
    perm[[3, 50, 299]] = [-7, wa.N, wa.N + 1000]
    prep["perm"][0, 0] = torch.from_numpy(perm)
    ws = vc.alloc_workspace(shape, params)
    vc.smooth_prepare(k.cuda(), v.cuda(), params, prep=prep, workspace=ws)
    vc.check(ws)
    clamped = np.where((perm >= 0) & (perm < wa.N), perm, 0).astype(np.int32)
    khat, ksc = oracle.quant_k(bits(k[0, 0]), clamped, wa.block)
    assert np.array_equal(prep["k_fp8"][0, 0].cpu().numpy(), khat)
    assert np.array_equal(prep["k_scale"][0, 0].cpu().numpy(), ksc)
