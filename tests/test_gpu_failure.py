"""Failure detection on the GPU without a fault.

Every device-side wait in the library is bounded by params.wait_limit_ns.  A
limit under 1 us leaves no time to wait: the first wait whose phase is not
already complete at its first (non-blocking) poll runs out, and the
kernel records VC_ERR_DEVICE_TIMEOUT in the workspace status word, lets its
own copies and MMAs land, frees its tensor memory and returns, so the context
stays usable.  These tests check the status vc_check reports, that kernels
launched while an error is recorded do nothing, and that the next call with
the default limit gives the same bytes as a run that never failed.

Inputs stay valid throughout (zero-filled prep buffers, seeded tensors), so
no access could leave its buffer even if a kernel ignored the recorded error.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


def _case(vc, N=1000, d=128, block=128):
    from bit_fp8_attention_smooth_b200 import synth

    w = synth.custom(f"fail_{N}_{d}", 1, 2, N, d, 41, pool=8, C=8, iters=4, block=block)
    q, k, v = (synth.tensor_bf16(w, t).cuda() for t in "qkv")
    return w, q, k, v


def _zero_prep(vc, shape, params):
    return {n: torch.zeros_like(t) for n, t in vc.alloc_prep(shape, params).items()}


def _reference(vc, q, k, v, params):
    ws = vc.alloc_workspace(tuple(q.shape), params)
    prep = vc.smooth_prepare(k, v, params, workspace=ws)
    out = vc.attn_fwd(q, prep, params, workspace=ws)
    vc.check(ws)
    return out


def _expect_timeout(vc, ws):
    with pytest.raises(vc.VcError) as e:
        vc.check(ws)
    assert e.value.status == vc.VC_ERR_DEVICE_TIMEOUT


def test_prep_timeout_is_reported_and_blocks_later_kernels(vc):
    w, q, k, v = _case(vc)
    params = vc.Params.for_workload(w, beta=64)
    ref = _reference(vc, q, k, v, params)
    shape = tuple(q.shape)
    ws = vc.alloc_workspace(shape, params)
    prep = _zero_prep(vc, shape, params)
    fast = vc.Params.for_workload(w, beta=64, wait_limit_ns=1)
    vc.smooth_prepare(k, v, fast, prep=prep, workspace=ws)
    # The attention launched on the same workspace sees the recorded error and
    # writes nothing.
    sentinel = torch.full_like(q, 7.0)
    out = vc.attn_fwd(q, prep, params, out=sentinel.clone(), workspace=ws)
    _expect_timeout(vc, ws)
    assert torch.equal(out, sentinel)
    # vc_check cleared the word: the next call on the same buffers is whole.
    vc.smooth_prepare(k, v, params, prep=prep, workspace=ws)
    out = vc.attn_fwd(q, prep, params, workspace=ws)
    vc.check(ws)
    assert torch.equal(out, ref)


@pytest.mark.parametrize("resid_fmt", [0, 1], ids=["e4m3", "nvfp4"])
@pytest.mark.parametrize("limit_ns", [1, 3000, 30000])
def test_attention_timeout_then_recovers(vc, limit_ns, resid_fmt):
    w, q, k, v = _case(vc)
    params = vc.Params.for_workload(w, beta=64, resid_fmt=resid_fmt)
    ref = _reference(vc, q, k, v, params)
    ws = vc.alloc_workspace(tuple(q.shape), params)
    prep = vc.smooth_prepare(k, v, params, workspace=ws)
    vc.check(ws)
    fast = vc.Params.for_workload(w, beta=64, wait_limit_ns=limit_ns, resid_fmt=resid_fmt)
    for _ in range(3):
        out = vc.attn_fwd(q, prep, fast, workspace=ws)
        try:
            vc.check(ws)
        except vc.VcError as e:  # the run stopped early: O is undefined
            assert e.status == vc.VC_ERR_DEVICE_TIMEOUT
        else:  # every wait finished inside the limit
            assert limit_ns > 1 and torch.equal(out, ref)
    out = vc.attn_fwd(q, prep, params, workspace=ws)
    vc.check(ws)
    assert torch.equal(out, ref)


def test_one_ns_limit_always_times_out(vc):
    w, q, k, v = _case(vc, N=3000, d=64, block=64)
    params = vc.Params.for_workload(w, beta=64)
    ws = vc.alloc_workspace(tuple(q.shape), params)
    prep = vc.smooth_prepare(k, v, params, workspace=ws)
    vc.check(ws)
    fast = vc.Params.for_workload(w, beta=64, wait_limit_ns=1)
    vc.attn_fwd(q, prep, fast, workspace=ws)
    _expect_timeout(vc, ws)
    # nothing is left behind: later work on the device still runs
    assert torch.ones(1 << 20, device="cuda").sum().item() == float(1 << 20)
