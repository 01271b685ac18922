"""Edge cases of the attention forward where the score scale A = kappa*sq*sk is
zero, or V is constant, through every kernel (8-bit at block 128 and 64, the
4-bit path, the block-sparse instantiation), against the oracle.

- Zero Q rows: sq = 0, so every key of the row gets the same byte and the row
  is the plain mean of the dequantised V (chooseai.io news 7051, section
  "核心方法之二：ExpCast-FP8 换掉 softmax 里的指数": the byte map covers the
  row's keys, no others).  Padding tokens of a real sequence are such rows.
- All-zero K blocks (sk = 0), among them the ragged last block, where the
  keys past N must still carry no weight.
- V constant along the tokens: every path returns the constant (the block
  mean restores it exactly; the residual is zero).

Both sides run on the same regroup order (the GPU's), so the prep bytes must
match exactly and the output only differs by fp32 accumulation order:
rel-L2 <= 3e-3 and cosine >= 0.99999 per head, every zero-Q row within
rel-L2 1e-2, and no NaN anywhere."""
import numpy as np
import pytest
import torch

import oracle
from bit_fp8_attention_smooth_b200 import synth
from gpu_common import BETA, bits, metrics, oracle_prep_on_perm

pytestmark = pytest.mark.gpu

CASES = [
    # name, N, d, block, resid_fmt
    ("e4m3_300_d128_bk128", 300, 128, 128, 0),
    ("e4m3_777_d128_bk64", 777, 128, 64, 0),
    ("e4m3_1000_d64_bk128", 1000, 64, 128, 0),
    ("nvfp4_300_d128", 300, 128, 128, 1),
    ("nvfp4_777_d64", 777, 64, 128, 1),
]


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


def _workload(name, N, d, block, seed):
    return synth.custom(name, 1, 2, N, d, seed, pool=6, C=6, iters=4, block=block)


def _zero_q_rows(N):
    """Rows spanning the first, an inner and the ragged last query tile."""
    return sorted({0, 5, min(N - 1, 129), N - 2, N - 1})


def _zero_k_blocks(T):
    """The ragged last block, and one inner block when there is one."""
    return sorted({T - 1} | ({T // 2} if T >= 3 else set()))


def _gpu_prep(vc, k, v, params):
    ws = vc.alloc_workspace(tuple(k.shape), params)
    prep = vc.smooth_prepare(k, v, params, workspace=ws)
    vc.check(ws)
    return prep, ws


def _oracle_out(q, k, v, b, h, perm, w, smooth, resid_fmt, tile_mask=None):
    qb, kb, vb = bits(q[b, h]), bits(k[b, h]), bits(v[b, h])
    own = oracle_prep_on_perm(kb, vb, perm, w.block, smooth, resid_fmt)
    r = oracle.forward_head(qb, kb, vb, np.arange(w.N), C=w.C, iters=w.iters, bk=w.block, beta=BETA,
                            smooth=smooth, resid_fmt=resid_fmt, prep=own, tile_mask=tile_mask)
    return own, r["out"]


def _check_prep_bytes(prep, own, b, h, resid_fmt):
    assert np.array_equal(prep["k_fp8"][b, h].cpu().numpy(), own["khat"])
    assert np.array_equal(prep["k_scale"][b, h].cpu().numpy(), own["ksc"])
    assert np.array_equal(prep["v_mean"][b, h].cpu().numpy(), own["vmu"])
    assert np.array_equal(prep["v_scale"][b, h].cpu().numpy(), own["vsc"])
    if resid_fmt == 0:
        assert np.array_equal(prep["vt_fp8"][b, h].cpu().numpy().T, own["vhat"])


def _zero_inputs(vc, w, params, smooth):
    """Seeded inputs with zero Q rows and all-zero K blocks in the GPU's own
    regroup order (the regroup depends on V only, so zeroing K keeps it)."""
    q, k, v = (synth.tensor_bf16(w, t) for t in "qkv")
    zq = _zero_q_rows(w.N)
    q[:, :, zq] = 0
    prep0, _ = _gpu_prep(vc, k.cuda(), v.cuda(), params)
    T = -(-w.N // w.block)
    for b in range(w.B):
        for h in range(w.H):
            perm = prep0["perm"][b, h].cpu().numpy()
            for blk in _zero_k_blocks(T):
                k[b, h, perm[blk * w.block:min(w.N, (blk + 1) * w.block)]] = 0
    return q, k, v, zq, prep0["perm"].cpu()


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("smooth", [True, False], ids=["vsmooth", "plain"])
def test_zero_q_rows_and_zero_k_blocks(vc, case, smooth):
    name, N, d, block, resid_fmt = case
    w = _workload(name, N, d, block, 61)
    params = vc.Params.for_workload(w, beta=BETA, smooth=smooth, resid_fmt=resid_fmt)
    q, k, v, zq, perm0 = _zero_inputs(vc, w, params, smooth)
    prep, ws = _gpu_prep(vc, k.cuda(), v.cuda(), params)
    assert torch.equal(prep["perm"].cpu(), perm0)  # zeroing K left the regroup alone
    out = vc.attn_fwd(q.cuda(), prep, params, workspace=ws)
    vc.check(ws)
    out = out.float().cpu().numpy()
    assert np.isfinite(out).all()
    for b in range(w.B):
        for h in range(w.H):
            perm = prep["perm"][b, h].cpu().numpy()
            own, ref = _oracle_out(q, k, v, b, h, perm, w, smooth, resid_fmt)
            _check_prep_bytes(prep, own, b, h, resid_fmt)
            rel, cos, _ = metrics(out[b, h], ref)
            assert rel <= 3e-3 and cos >= 0.99999, (b, h, rel, cos)
            for r in zq:
                rr, _, _ = metrics(out[b, h, r], ref[r])
                assert rr <= 1e-2, (b, h, r, rr)


@pytest.mark.parametrize("case", [c for c in CASES if c[4] == 0], ids=lambda c: c[0])
def test_zero_rows_block_sparse(vc, case):
    """The block-sparse kernel on the same inputs, with a seeded tile mask
    that keeps the ragged last key tile for some query tiles."""
    name, N, d, block, resid_fmt = case
    w = _workload(name, N, d, block, 62)
    params = vc.Params.for_workload(w, beta=BETA)
    q, k, v, zq, _ = _zero_inputs(vc, w, params, True)
    prep, ws = _gpu_prep(vc, k.cuda(), v.cuda(), params)
    Tq, T = -(-N // 128), -(-N // block)
    g = torch.Generator().manual_seed(5)
    mask = (torch.rand((w.B, w.H, Tq, T), generator=g) < 0.6).to(torch.uint8)
    mask[:, :, ::2, T - 1] = 1
    out = vc.attn_fwd(q.cuda(), prep, params, workspace=ws, tile_mask=mask.cuda())
    vc.check(ws)
    out = out.float().cpu().numpy()
    assert np.isfinite(out).all()
    for b in range(w.B):
        for h in range(w.H):
            perm = prep["perm"][b, h].cpu().numpy()
            _, ref = _oracle_out(q, k, v, b, h, perm, w, True, 0, tile_mask=mask[b, h].numpy())
            rel, cos, _ = metrics(out[b, h], ref)
            assert rel <= 3e-3 and cos >= 0.99999, (b, h, rel, cos)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("smooth", [True, False], ids=["vsmooth", "plain"])
def test_constant_v_returns_the_constant(vc, case, smooth):
    """V equal to one row for every token: the output is that row (the mean
    restore gives it back exactly; the residual is zero), within one bf16
    rounding, on every query row, for any Q and K."""
    name, N, d, block, resid_fmt = case
    w = _workload(name, N, d, block, 63)
    params = vc.Params.for_workload(w, beta=BETA, smooth=smooth, resid_fmt=resid_fmt)
    q, k, v = (synth.tensor_bf16(w, t) for t in "qkv")
    q[:, :, :3] = 0
    v[:] = v[:, :, :1].clone()
    out = vc.attention(q.cuda(), k.cuda(), v.cuda(), params).float().cpu()
    want = v.float()
    assert torch.isfinite(out).all()
    assert torch.all((out - want).abs() <= 2.0 ** -8 * want.abs()), (out - want).abs().max()
