"""No kernel writes outside the buffers it is given.

Every buffer the library writes (the prep outputs, the workspace and the
attention output) is carved out of a larger allocation whose margins hold a
known byte pattern.  After the prep, the dense attention and the block-sparse
attention, the margins must still hold it.  This stands in for a memory
checker on ragged shapes, both residual formats, both block sizes and
V-Smooth on and off.  The
margins are 16 KiB, so every base address keeps the alignment of an ordinary
allocation (512 bytes from the caching allocator; TMA needs 16)."""
import math

import pytest
import torch

from bit_fp8_attention_smooth_b200 import synth
from gpu_common import BETA, make_inputs

pytestmark = pytest.mark.gpu

CANARY = 0xA5
PAD_BYTES = 1 << 14

# (workload, residual format, V-Smooth mode)
CASES = [
    (synth.custom("canary_777_d128_b64", 1, 3, 777, 128, 41, pool=8, C=8, iters=4, block=64), 0, 1),
    (synth.custom("canary_1000_d64_b128_plain", 2, 1, 1000, 64, 42, pool=12, C=12, iters=4, block=128), 0, 0),
    (synth.custom("canary_300_d128_nvfp4", 1, 2, 300, 128, 43, pool=8, C=8, iters=4, block=128), 1, 1),
]


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


class Margins:
    def __init__(self):
        self.pools = []

    def carve(self, shape, dtype, fill=None):
        es = torch.empty((), dtype=dtype).element_size()
        n = math.prod(shape)
        pad = PAD_BYTES // es
        big = torch.empty(n + 2 * pad, dtype=dtype, device="cuda")
        big.view(torch.uint8).fill_(CANARY)
        view = big[pad:pad + n].view(shape)
        if fill is not None:
            view.view(torch.uint8).fill_(fill)
        self.pools.append((big, pad * es, n * es))
        return view

    def check(self):
        torch.cuda.synchronize()
        for big, pad, nbytes in self.pools:
            b = big.view(torch.uint8)
            lo, hi = b[:pad], b[pad + nbytes:]
            assert bool((lo == CANARY).all()) and bool((hi == CANARY).all()), (
                "a kernel wrote outside a buffer", tuple(big.shape), big.dtype,
                int((lo != CANARY).sum()), int((hi != CANARY).sum()))


@pytest.mark.parametrize("w,resid_fmt,smooth", CASES, ids=[c[0].name for c in CASES])
def test_writes_stay_inside_the_buffers(vc, w, resid_fmt, smooth):
    q, k, v, qd, kd, vd = make_inputs(w)
    params = vc.Params.for_workload(w, beta=BETA, resid_fmt=resid_fmt, smooth=smooth)
    shape = tuple(q.shape)
    m = Margins()
    prep = {n: m.carve(sh, dt) for n, (sh, dt) in vc.prep_layout(shape, params).items()}
    ws = m.carve((vc.workspace_bytes(shape, params),), torch.uint8, fill=0)  # the status word starts at 0
    out = m.carve(shape, torch.bfloat16)
    vc.smooth_prepare(kd, vd, params, prep=prep, workspace=ws)
    vc.attn_fwd(qd, prep, params, out=out, workspace=ws)
    vc.check(ws)
    m.check()
    # the result is that of an ordinary call (k-means sums in fp64 atomics, so
    # compare within the parity tolerance rather than bit for bit)
    ref = vc.attention(qd, kd, vd, params).float()
    got = out.float()
    assert torch.isfinite(got).all()
    rel = ((got - ref).norm() / ref.norm()).item()
    assert rel <= 1e-2, rel
    if resid_fmt == 0:  # block-sparse attention (the 8-bit kernel)
        g = torch.Generator().manual_seed(9)
        B, H, N, _ = shape
        mask = (torch.rand((B, H, -(-N // 128), -(-N // w.block)), generator=g) < 0.5).to(torch.uint8).cuda()
        out2 = m.carve(shape, torch.bfloat16)
        vc.attn_fwd(qd, prep, params, out=out2, workspace=ws, tile_mask=mask)
        vc.check(ws)
        m.check()
        assert torch.isfinite(out2.float()).all()
