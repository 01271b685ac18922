"""vc_attention_host: the attention call from pinned host buffers, with the
copies of one run of (b, h) problems overlapped with the computation of its
neighbours.  Its output must equal, byte for byte, the device-resident call
vc_attention on the same inputs, for any number of runs, and two calls in a
row with different inputs must not see each other's data."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


def _inputs(B, H, N, d, seed):
    from bit_fp8_attention_smooth_b200 import synth

    w = synth.custom(f"host_{B}_{H}_{N}_{d}_{seed}", B, H, N, d, seed, pool=8, C=8, iters=4, block=128)
    return w, [synth.tensor_bf16(w, t) for t in "qkv"]


def _device_reference(vc, w, q, k, v, resid_fmt=0):
    params = vc.Params.for_workload(w, beta=64, resid_fmt=resid_fmt)
    ws = vc.alloc_workspace(tuple(q.shape), params)
    out = vc.attention(q.cuda(), k.cuda(), v.cuda(), params, workspace=ws)
    vc.check(ws)
    return out.cpu()


@pytest.mark.parametrize("B,H,N,d,groups,resid_fmt", [(1, 6, 1000, 128, 1, 0), (1, 6, 1000, 128, 4, 0),
                                                      (2, 3, 777, 64, 6, 0), (1, 5, 2100, 128, 64, 0),
                                                      (2, 3, 1300, 128, 4, 1)])
def test_host_call_equals_device_call(vc, B, H, N, d, groups, resid_fmt):
    w, (q, k, v) = _inputs(B, H, N, d, 51)
    ref = _device_reference(vc, w, q, k, v, resid_fmt)
    params = vc.Params.for_workload(w, beta=64, resid_fmt=resid_fmt)
    call = vc.HostAttention(tuple(q.shape), params, groups=groups)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(q).pin_memory()
    call(qh, kh, vh, oh)
    torch.cuda.synchronize()
    vc.check(call.ws)
    assert torch.equal(oh, ref)


def test_consecutive_host_calls_keep_their_inputs(vc):
    w1, (q1, k1, v1) = _inputs(1, 4, 1500, 128, 61)
    w2, (q2, k2, v2) = _inputs(1, 4, 1500, 128, 62)
    ref1 = _device_reference(vc, w1, q1, k1, v1)
    ref2 = _device_reference(vc, w2, q2, k2, v2)
    params = vc.Params.for_workload(w1, beta=64)
    call = vc.HostAttention(tuple(q1.shape), params, groups=4)
    o1 = torch.empty_like(q1).pin_memory()
    o2 = torch.empty_like(q2).pin_memory()
    call(q1.pin_memory(), k1.pin_memory(), v1.pin_memory(), o1)
    call(q2.pin_memory(), k2.pin_memory(), v2.pin_memory(), o2)
    torch.cuda.synchronize()
    vc.check(call.ws)
    assert torch.equal(o1, ref1)
    assert torch.equal(o2, ref2)
