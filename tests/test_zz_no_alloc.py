"""The allocation-free attention entry point (vc_attn_fwd_noalloc), called
through the C ABI, against the workspace entry point vc_attn_fwd.

Some callers cannot allocate device memory when they call the op (a host
runtime that owns all memory and passes only inputs and outputs, or a loop
that cannot take cudaMalloc's synchronisation); this entry point serves them
from a static per-device scratch array.  This file is collected last so that a
run stopping at its first failure has run every other test already; it also
passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

@pytest.mark.parametrize("N,d,block,resid_fmt", [(3000, 128, 128, 0), (1000, 64, 64, 0), (2100, 128, 128, 1)])
def test_noalloc_matches_workspace_entry_point(N, d, block, resid_fmt):
    import bit_fp8_attention_smooth_b200 as vc
    from bit_fp8_attention_smooth_b200 import synth

    L = vc.lib()
    w = synth.custom(f"noalloc_{N}_{d}", 1, 2, N, d, 31, pool=8, C=8, iters=4, block=block)
    q, k, v = (synth.tensor_bf16(w, t).cuda() for t in "qkv")
    q[:, :, :3] = 0  # zero rows (padding tokens): score scale 0 over the ragged last key tile too
    q[:, :, -2:] = 0
    params = vc.Params.for_workload(w, beta=64, resid_fmt=resid_fmt)
    ws = vc.alloc_workspace(tuple(q.shape), params)
    prep = vc.smooth_prepare(k, v, params, workspace=ws)
    ref = vc.attn_fwd(q, prep, params, workspace=ws)
    vc.check(ws)
    prep_c = vc._prep_struct(prep)
    shape_c = vc._Shape(*q.shape)
    params_c = params.c()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        st = L.vc_attn_fwd_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.byref(prep_c), ctypes.byref(shape_c),
                                   ctypes.byref(params_c), ctypes.c_void_p(out.data_ptr()), stream)
        assert st == vc.VC_OK, vc.status_string(st)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: the same bits
        assert torch.equal(out, ref), (call, (out.float() - ref.float()).abs().max().item())


def test_noalloc_rejects_oversized_problems():
    import bit_fp8_attention_smooth_b200 as vc

    L = vc.lib()
    q = torch.zeros((1, 8, 32768, 128), dtype=torch.bfloat16, device="cuda")  # 8*32768*132 B > 16 MiB
    params = vc.Params(C=4, iters=1, block=128)
    prep = vc.alloc_prep(tuple(q.shape), params)
    out = torch.empty_like(q)
    st = L.vc_attn_fwd_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.byref(vc._prep_struct(prep)),
                               ctypes.byref(vc._Shape(*q.shape)), ctypes.byref(params.c()),
                               ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(0))
    assert st == vc.VC_ERR_WORKSPACE
