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
