"""Host-side argument checks of the Python binding, on the CPU.  The library
indexes raw pointers by the problem shape, so the binding refuses any buffer
whose dtype, shape, contiguity or device differs from what the call implies
before the library is reached."""
import pytest
import torch

import bit_fp8_attention_smooth_b200 as vc

CPU = torch.device("cpu")
SHAPE = (1, 2, 300, 64)


@pytest.mark.parametrize("resid_fmt,block", [(0, 64), (0, 128), (1, 128)])
def test_allocated_prep_passes_its_own_check(resid_fmt, block):
    params = vc.Params(C=8, iters=2, block=block, resid_fmt=resid_fmt)
    prep = vc.alloc_prep(SHAPE, params, CPU)
    vc._check_prep(prep, SHAPE, params, CPU)
    assert ("v_bscale" in prep) == (resid_fmt == 1)
    T = -(-300 // block)
    assert tuple(prep["k_fp8"].shape) == (1, 2, T * block, 64)
    assert tuple(prep["vt_fp8"].shape) == (1, 2, 64, T * block // (2 if resid_fmt else 1))


def test_prep_of_another_block_or_format_is_refused():
    p128 = vc.Params(C=8, iters=2, block=128)
    p64 = vc.Params(C=8, iters=2, block=64)
    with pytest.raises(ValueError, match="k_fp8"):
        vc._check_prep(vc.alloc_prep(SHAPE, p64, CPU), SHAPE, p128, CPU)
    p4 = vc.Params(C=8, iters=2, block=128, resid_fmt=1)
    with pytest.raises(ValueError, match="v_bscale|vt_fp8"):
        vc._check_prep(vc.alloc_prep(SHAPE, p128, CPU), SHAPE, p4, CPU)
    with pytest.raises(ValueError, match="perm"):
        vc._check_prep(vc.alloc_prep((1, 2, 301, 64), p128, CPU), SHAPE, p128, CPU)


@pytest.mark.parametrize("field", ["perm", "k_scale", "vt_fp8", "v_mean"])
def test_prep_buffer_dtype_layout_and_device(field):
    params = vc.Params(C=8, iters=2, block=64)
    prep = vc.alloc_prep(SHAPE, params, CPU)
    good = prep[field]
    prep[field] = good.to(torch.float64)
    with pytest.raises(ValueError, match=field):
        vc._check_prep(prep, SHAPE, params, CPU)
    prep[field] = good.transpose(-1, -2).contiguous().transpose(-1, -2) if good.dim() > 1 else good[::1]
    if not prep[field].is_contiguous():
        with pytest.raises(ValueError, match="not contiguous"):
            vc._check_prep(prep, SHAPE, params, CPU)
    prep[field] = good.to("meta")  # another device
    with pytest.raises(ValueError, match=field):
        vc._check_prep(prep, SHAPE, params, CPU)
    del prep[field]
    with pytest.raises(ValueError, match="missing"):
        vc._check_prep(prep, SHAPE, params, CPU)


def test_out_must_match_q():
    q = torch.empty(SHAPE, dtype=torch.bfloat16)
    vc._check_out(torch.empty_like(q), q)
    for bad in (torch.empty(SHAPE, dtype=torch.float32), torch.empty((1, 2, 299, 64), dtype=torch.bfloat16),
                torch.empty((1, 2, 64, 300), dtype=torch.bfloat16).transpose(-1, -2), "not a tensor"):
        with pytest.raises(ValueError, match="out"):
            vc._check_out(bad, q)


def test_workspace_size_is_counted_in_bytes():
    ptr, nbytes = vc._ws_args(torch.zeros(10, dtype=torch.float32), CPU)
    assert nbytes == 40
    with pytest.raises(ValueError, match="workspace"):
        vc._ws_args(torch.zeros(10, 2, dtype=torch.uint8).t(), CPU)


def test_public_calls_refuse_host_tensors():
    x = torch.zeros(SHAPE, dtype=torch.bfloat16)
    params = vc.Params(C=8, iters=2, block=64)
    with pytest.raises(ValueError, match="CUDA"):
        vc.smooth_prepare(x, x, params)
    with pytest.raises(ValueError, match="CUDA"):
        vc.attn_fwd(x, vc.alloc_prep(SHAPE, params, CPU), params)
    with pytest.raises(ValueError, match="CUDA"):
        vc.e4m3_encode(torch.zeros(4))
    with pytest.raises(ValueError, match="CUDA"):
        vc.expcast_bytes(torch.zeros(4), torch.zeros(4), torch.zeros(4))


class _FakeLib:
    """Stands in for libvcattn.so: records each call's arguments, answers 0
    (and a workspace size of 4096 bytes)."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            if name == "vc_workspace_bytes":
                args[2]._obj.value = 4096
            return 0

        return fn


@pytest.fixture
def fake(monkeypatch):
    f = _FakeLib()
    monkeypatch.setattr(vc, "_lib", f)
    monkeypatch.setattr(vc, "_stream", lambda stream: None)

    def host_input(t, name):  # the CUDA requirement aside, the same checks
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(name)

    monkeypatch.setattr(vc, "_check_input", host_input)
    return f


def test_marshalling_of_every_entry_point(fake):
    """Each public call hands the library the buffers' own pointers and the
    workspace size in bytes; nothing else runs on the host."""
    q, k, v = (torch.randn(SHAPE).bfloat16() for _ in range(3))
    for resid_fmt, block in ((0, 64), (1, 128)):
        params = vc.Params(C=8, iters=2, block=block, resid_fmt=resid_fmt)
        ws = torch.zeros(4096, dtype=torch.uint8)
        prep = vc.smooth_prepare(k, v, params, workspace=ws)
        name, args = fake.calls[-1]
        assert name == "vc_smooth_prepare"
        assert args[0] == k.data_ptr() and args[1] == v.data_ptr() and args[5:7] == (ws.data_ptr(), 4096)
        assert args[4]._obj.k_fp8 == prep["k_fp8"].data_ptr()
        assert (args[4]._obj.v_bscale is not None) == (resid_fmt == 1)

        out = vc.attn_fwd(q, prep, params, workspace=ws)
        name, args = fake.calls[-1]
        assert name == "vc_attn_fwd" and args[4] == out.data_ptr() and args[5:7] == (ws.data_ptr(), 4096)

        mask = torch.ones((1, 2, 3, -(-300 // block)), dtype=torch.uint8)
        out = vc.attn_fwd(q, prep, params, workspace=ws, tile_mask=mask)
        name, args = fake.calls[-1]
        assert name == "vc_attn_fwd_masked" and args[4] == mask.data_ptr() and args[5] == out.data_ptr()
        assert args[6:8] == (ws.data_ptr(), 4096)

        out = vc.attention(q, k, v, params)  # allocates its own prep and workspace
        name, args = fake.calls[-1]
        assert name == "vc_attention" and args[6] == out.data_ptr() and args[8] == 4096

        out = vc.attn_fwd_noalloc(q, prep, params)
        assert fake.calls[-1][0] == "vc_attn_fwd_noalloc" and fake.calls[-1][1][4] == out.data_ptr()

        vc.check(ws)
        assert fake.calls[-1] == ("vc_check", (ws.data_ptr(), None))


def test_mismatched_buffers_never_reach_the_library(fake):
    q, k, v = (torch.randn(SHAPE).bfloat16() for _ in range(3))
    params = vc.Params(C=8, iters=2, block=64)
    prep = vc.alloc_prep(SHAPE, params, CPU)
    bad_calls = [
        lambda: vc.smooth_prepare(k, v[:, :1].contiguous(), params),
        lambda: vc.attn_fwd(q, vc.alloc_prep(SHAPE, vc.Params(block=128), CPU), params),
        lambda: vc.attn_fwd(q, prep, params, out=torch.empty(SHAPE, dtype=torch.float32)),
        lambda: vc.attn_fwd(q, prep, params, tile_mask=torch.ones((1, 2, 3), dtype=torch.uint8)),
        lambda: vc.attention(q, k[:, :, :299].contiguous(), v, params),
        lambda: vc.attn_fwd_noalloc(q, prep, vc.Params(block=64, resid_fmt=1)),
    ]
    for call in bad_calls:
        n = len(fake.calls)
        with pytest.raises(ValueError):
            call()
        assert all(name in ("vc_workspace_bytes",) for name, _ in fake.calls[n:])
