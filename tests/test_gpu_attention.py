"""GPU parity of the whole path (V-Smooth prep + ExpCast-FP8 attention)
against the oracle on small seeded workloads that span several tiles and a
ragged tail.  Element-wise comparisons; tolerances: bit-exact for integer and
byte outputs, rel-L2 <= 1e-2 and cosine >= 0.9995 for the attention output."""
import numpy as np
import pytest
import torch

import oracle
from bit_fp8_attention_smooth_b200 import synth
from gpu_common import (BETA, COS_TOL, REL_L2_TOL, bits, check_labels_valid, check_perm, gpu_prep_head, make_inputs,
                        metrics, oracle_head, oracle_prep_on_perm, oracle_prep_to_gpu, prep_to_host)

pytestmark = pytest.mark.gpu

CASES = [
    synth.WORKLOADS["tiny_1k_d64"],
    synth.custom("ragged_300_d128", 1, 2, 300, 128, 21, pool=8, C=8, iters=5, block=128),
    synth.custom("ragged_1000_d64_bk128", 2, 1, 1000, 64, 22, pool=12, C=12, iters=6, block=128),
    synth.custom("ragged_777_d128_bk64", 1, 3, 777, 128, 23, pool=10, C=10, iters=6, block=64),
    synth.custom("one_tile_90_d64", 1, 1, 90, 64, 24, pool=4, C=4, iters=3, block=64),
    synth.custom("single_token", 1, 2, 1, 128, 25, pool=1, C=1, iters=2, block=128),
]


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


def _run_gpu(vc, w, qd, kd, vd, smooth=True):
    params = vc.Params.for_workload(w, beta=BETA, smooth=smooth)
    ws = vc.alloc_workspace(tuple(qd.shape), params)
    prep = vc.smooth_prepare(kd, vd, params, workspace=ws)
    out = vc.attn_fwd(qd, prep, params, workspace=ws)
    vc.check(ws)
    return prep_to_host(prep), out.float().cpu().numpy()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("smooth", [True, False], ids=["vsmooth", "plain"])
def test_prep_parity(vc, w, smooth):
    q, k, v, qd, kd, vd = make_inputs(w)
    prep, _ = _run_gpu(vc, w, qd, kd, vd, smooth)
    for b in range(w.B):
        for h in range(w.H):
            ref = oracle.prep_head(bits(k[b, h]), bits(v[b, h]), C=w.C, iters=w.iters, bk=w.block, smooth=smooth)
            got = gpu_prep_head(prep, b, h, w.N, w.block)
            check_perm(got["perm"], got["labels"], w.N)
            assert (got["labels"] == ref["labels"]).mean() >= 0.999
            if smooth:
                check_labels_valid(bits(v[b, h]), got["labels"], ref["labels"], ref["centroids"])
                # the regroup is the stable sort of the GPU's own labels
                assert np.array_equal(got["perm"], oracle.stable_perm(got["labels"], w.C))
            else:
                assert np.array_equal(got["perm"], np.arange(w.N))
            # quantiser bytes, always: the oracle's quantisers on the GPU's order
            own = oracle_prep_on_perm(bits(k[b, h]), bits(v[b, h]), got["perm"], w.block, smooth)
            for key in ("khat", "ksc", "vmu", "vsc", "vhat"):
                assert np.array_equal(got[key], own[key]), (b, h, key)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_attention_kernel_on_oracle_prep(vc, w):
    """The attention kernel alone: fed the oracle's own prep, its output
    matches the oracle's replay closely (only fp32 accumulation order differs)."""
    q, k, v, qd, kd, vd = make_inputs(w)
    rows = np.arange(w.N)
    preps, refs = [], []
    for b in range(w.B):
        preps.append([])
        for h in range(w.H):
            r = oracle_head(q, k, v, b, h, rows, w)
            preps[-1].append(r["prep"])
            refs.append(r)
    params = vc.Params.for_workload(w, beta=BETA)
    gprep = oracle_prep_to_gpu(preps, tuple(q.shape), w.block)
    ws = vc.alloc_workspace(tuple(q.shape), params)
    out = vc.attn_fwd(qd, gprep, params, workspace=ws).float().cpu().numpy()
    vc.check(ws)
    i = 0
    for b in range(w.B):
        for h in range(w.H):
            rel, cos, _ = metrics(out[b, h], refs[i]["out"])
            assert rel <= 3e-3 and cos >= 0.99999, (b, h, rel, cos)
            i += 1


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("smooth", [True, False], ids=["vsmooth", "plain"])
def test_end_to_end_parity(vc, w, smooth):
    q, k, v, qd, kd, vd = make_inputs(w)
    _, out = _run_gpu(vc, w, qd, kd, vd, smooth)
    rows = np.arange(w.N)
    for b in range(w.B):
        for h in range(w.H):
            r = oracle_head(q, k, v, b, h, rows, w, smooth=smooth)
            rel, cos, psnr = metrics(out[b, h], r["out"])
            assert rel <= REL_L2_TOL and cos >= COS_TOL, (b, h, rel, cos)
            rel_x, cos_x, psnr_x = metrics(out[b, h], r["exact"])
            print(f"{w.name} smooth={smooth} b={b} h={h}: vs emulation rel={rel:.2e} cos={cos:.6f}; "
                  f"vs exact rel={rel_x:.3e} psnr={psnr_x:.1f} dB")


def test_attention_call_equals_two_step(vc):
    w = CASES[0]
    q, k, v, qd, kd, vd = make_inputs(w)
    params = vc.Params.for_workload(w, beta=BETA)
    a = vc.attention(qd, kd, vd, params)
    _, b = _run_gpu(vc, w, qd, kd, vd)
    assert torch.equal(a.float().cpu(), torch.from_numpy(b))


def test_rejects_bad_arguments(vc):
    w = CASES[0]
    q, k, v, qd, kd, vd = make_inputs(w)
    with pytest.raises(vc.VcError) as e:
        vc.attention(qd, kd, vd, vc.Params(C=16, iters=8, block=96))
    assert e.value.status == vc.VC_ERR_UNSUPPORTED
    with pytest.raises(vc.VcError) as e:
        vc.attention(qd, kd, vd, vc.Params(C=16, iters=8, block=64, beta=80))
    assert e.value.status == vc.VC_ERR_INVALID_ARG
    params = vc.Params.for_workload(w)
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(vc.VcError) as e:
        vc.attention(qd, kd, vd, params, workspace=small)
    assert e.value.status == vc.VC_ERR_WORKSPACE
