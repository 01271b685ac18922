"""GPU parity of the 4-bit path (resid_fmt 1): the NVFP4 V residual from the
prep, and the attention whose PV product takes NVFP4 P and V (tcgen05
kind::mxf4nvf4), against the oracle on small seeded workloads that span
several tiles and a ragged tail.

Tolerances:
- residual codes, block scales, block means and channel scales: bit-exact
  (given the same regroup order);
- the attention kernel fed the oracle's own prep: rel-L2 <= 3e-3 and cosine
  >= 0.99999 (only fp32 accumulation order differs);
- end to end: rel-L2 <= 1e-2 and cosine >= 0.9995.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_fp8_attention_smooth_b200 import synth
from gpu_common import BETA, COS_TOL, REL_L2_TOL, bits, check_perm, make_inputs, metrics, prep_to_host

pytestmark = pytest.mark.gpu

CASES = [
    synth.custom("nv4_ragged_300_d128", 1, 2, 300, 128, 31, pool=8, C=8, iters=5, block=128),
    synth.custom("nv4_ragged_1000_d64", 2, 1, 1000, 64, 32, pool=12, C=12, iters=6, block=128),
    synth.custom("nv4_1280_d128", 1, 2, 1280, 128, 33, pool=16, C=16, iters=4, block=128),
    synth.custom("nv4_single_token", 1, 1, 1, 128, 34, pool=1, C=1, iters=2, block=128),
]


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


def unpack_codes(vt: np.ndarray) -> np.ndarray:
    """[d, Tp/2] bytes, two E2M1 codes a byte (low nibble first) -> [Tp, d] codes."""
    codes = np.stack([vt & 0xF, vt >> 4], axis=-1).reshape(vt.shape[0], -1)
    return np.ascontiguousarray(codes.T)


def pack_codes(vq: np.ndarray) -> np.ndarray:
    """[Tp, d] codes -> [d, Tp/2] bytes."""
    c = vq.T
    return np.ascontiguousarray(c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def _params(vc, w, smooth=True):
    return vc.Params.for_workload(w, beta=BETA, smooth=smooth, resid_fmt=1)


def _run_gpu(vc, w, qd, kd, vd, smooth=True):
    params = _params(vc, w, smooth)
    ws = vc.alloc_workspace(tuple(qd.shape), params)
    prep = vc.smooth_prepare(kd, vd, params, workspace=ws)
    vc.check(ws)
    out = vc.attn_fwd(qd, prep, params, workspace=ws)
    vc.check(ws)
    return prep_to_host(prep), out.float().cpu().numpy()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("smooth", [True, False], ids=["vsmooth", "plain"])
def test_prep_parity_nvfp4(vc, w, smooth):
    q, k, v, qd, kd, vd = make_inputs(w)
    prep, _ = _run_gpu(vc, w, qd, kd, vd, smooth)
    T = -(-w.N // w.block)
    assert tuple(prep["vt_fp8"].shape) == (w.B, w.H, w.d, T * w.block // 2)
    assert tuple(prep["v_bscale"].shape) == (w.B, w.H, T, w.d, w.block // 16)
    for b in range(w.B):
        for h in range(w.H):
            perm = prep["perm"][b, h].numpy()
            check_perm(perm, prep["labels"][b, h].numpy(), w.N)
            # the residual from the GPU's own regroup order
            vq, vgs, vmu, vsc = oracle.smooth_v_nvfp4(bits(v[b, h]), perm, w.block, smooth)
            khat, ksc = oracle.quant_k(bits(k[b, h]), perm, w.block)
            assert np.array_equal(prep["k_fp8"][b, h].numpy(), khat)
            assert np.array_equal(prep["k_scale"][b, h].numpy(), ksc)
            assert np.array_equal(prep["v_mean"][b, h].numpy(), vmu)
            assert np.array_equal(prep["v_scale"][b, h].numpy(), vsc)
            assert np.array_equal(prep["v_bscale"][b, h].numpy().transpose(0, 2, 1), vgs)
            got = unpack_codes(prep["vt_fp8"][b, h].numpy())
            assert np.array_equal(got, vq), (np.argwhere(got != vq)[:5], got[got != vq][:5], vq[got != vq][:5])


def _oracle_prep4(w, k, v, b, h):
    return oracle.prep_head(bits(k[b, h]), bits(v[b, h]), C=w.C, iters=w.iters, bk=w.block, resid_fmt=1)


def _oracle_prep_to_gpu4(vc, preps, shape, bk):
    B, H, N, d = shape
    out = vc.alloc_prep(shape, vc.Params(block=bk, resid_fmt=1), "cuda")
    for b in range(B):
        for h in range(H):
            p = preps[b][h]
            out["perm"][b, h] = torch.from_numpy(p["perm"])
            out["labels"][b, h] = torch.from_numpy(p["labels"])
            out["k_fp8"][b, h] = torch.from_numpy(p["khat"])
            out["k_scale"][b, h] = torch.from_numpy(p["ksc"])
            out["vt_fp8"][b, h] = torch.from_numpy(pack_codes(p["vq"]))
            out["v_bscale"][b, h] = torch.from_numpy(np.ascontiguousarray(p["vgs"].transpose(0, 2, 1)))
            out["v_mean"][b, h] = torch.from_numpy(p["vmu"])
            out["v_scale"][b, h] = torch.from_numpy(p["vsc"])
    return out


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_attention_kernel_on_oracle_prep_nvfp4(vc, w):
    """The 4-bit attention kernel alone, fed the oracle's own prep."""
    q, k, v, qd, kd, vd = make_inputs(w)
    rows = np.arange(w.N)
    preps = [[_oracle_prep4(w, k, v, b, h) for h in range(w.H)] for b in range(w.B)]
    params = _params(vc, w)
    gprep = _oracle_prep_to_gpu4(vc, preps, tuple(q.shape), w.block)
    ws = vc.alloc_workspace(tuple(q.shape), params)
    out = vc.attn_fwd(qd, gprep, params, workspace=ws).float().cpu().numpy()
    vc.check(ws)
    for b in range(w.B):
        for h in range(w.H):
            ref = oracle.forward_head(bits(q[b, h]), bits(k[b, h]), bits(v[b, h]), rows, C=w.C, iters=w.iters,
                                      bk=w.block, beta=BETA, resid_fmt=1, prep=preps[b][h])["out"]
            rel, cos, _ = metrics(out[b, h], ref)
            assert rel <= 3e-3 and cos >= 0.99999, (b, h, rel, cos)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("smooth", [True, False], ids=["vsmooth", "plain"])
def test_end_to_end_parity_nvfp4(vc, w, smooth):
    q, k, v, qd, kd, vd = make_inputs(w)
    _, out = _run_gpu(vc, w, qd, kd, vd, smooth)
    rows = np.arange(w.N)
    for b in range(w.B):
        for h in range(w.H):
            qb, kb, vb = bits(q[b, h]), bits(k[b, h]), bits(v[b, h])
            r = oracle.forward_head(qb, kb, vb, rows, C=w.C, iters=w.iters, bk=w.block, beta=BETA, smooth=smooth,
                                    resid_fmt=1)
            rel, cos, _ = metrics(out[b, h], r["out"])
            assert rel <= REL_L2_TOL and cos >= COS_TOL, (b, h, rel, cos)
            rel_x, _, psnr_x = metrics(out[b, h], oracle.attn_exact(qb, kb, vb, rows))
            print(f"{w.name} smooth={smooth} b={b} h={h}: vs emulation rel={rel:.2e} cos={cos:.6f}; "
                  f"vs exact rel={rel_x:.3e} psnr={psnr_x:.1f} dB")


def test_four_bit_rejects_block_64(vc):
    w = synth.WORKLOADS["tiny_1k_d64"]
    q, k, v, qd, kd, vd = make_inputs(w)
    with pytest.raises(vc.VcError) as e:
        vc.attention(qd, kd, vd, vc.Params(C=16, iters=8, block=64, resid_fmt=1))
    assert e.value.status == vc.VC_ERR_UNSUPPORTED


def test_prep_nvfp4_ties_bit_exact(vc):
    """The crafted tie workload (V-Smooth off, channel scales 1, block scales
    set by construction): every code, including thousands of exact E2M1 ties
    of y * RN(1/s) and of values that only the exact quotient puts on a tie,
    matches the oracle."""
    from conftest import nvfp4_tie_values

    v, _ = nvfp4_tie_values(21)
    n, d = v.shape
    rng = torch.Generator().manual_seed(5)
    k = torch.randn((1, 1, n, d), generator=rng).bfloat16()
    vt = torch.from_numpy(v).bfloat16().reshape(1, 1, n, d)
    params = vc.Params(C=4, iters=2, block=128, smooth=0, resid_fmt=1)
    ws = vc.alloc_workspace((1, 1, n, d), params)
    prep = vc.smooth_prepare(k.cuda(), vt.cuda(), params, workspace=ws)
    vc.check(ws)
    prep = prep_to_host(prep)
    vq, vgs, vmu, vsc = oracle.smooth_v_nvfp4(bits(vt[0, 0]), np.arange(n, dtype=np.int32), 128, False)
    assert np.array_equal(prep["perm"][0, 0].numpy(), np.arange(n))
    assert np.array_equal(prep["v_scale"][0, 0].numpy(), vsc)
    assert np.array_equal(prep["v_mean"][0, 0].numpy(), vmu)
    assert np.array_equal(prep["v_bscale"][0, 0].numpy().transpose(0, 2, 1), vgs)
    got = unpack_codes(prep["vt_fp8"][0, 0].numpy())
    bad = np.argwhere(got != vq)
    assert bad.size == 0, (bad[:5], got[got != vq][:5], vq[got != vq][:5])
