"""The head split of the multi-GPU path, run on one device: every (b, h)
problem is independent, k-means included (chooseai.io news 7051, section
"意义与局限": VC-Attention combines with multi-GPU parallelism), so the heads
of each rank's head_range, run through the library as separate calls, must
give exactly the bytes of one call over all heads.  Each slice stands for one
rank; no collective is involved."""
import pytest
import torch

from bit_fp8_attention_smooth_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("resid_fmt", [0, 1], ids=["e4m3", "nvfp4"])
@pytest.mark.parametrize("world", [2, 3])
def test_head_slices_equal_the_full_call(world, resid_fmt):
    import bit_fp8_attention_smooth_b200 as vc

    w = synth.custom("split_1000_d128", 1, 5, 1000, 128, 41, pool=8, C=8, iters=4, block=128)
    q, k, v = (synth.tensor_bf16(w, t).cuda() for t in "qkv")
    params = vc.Params.for_workload(w, beta=64, resid_fmt=resid_fmt)
    full = vc.attention(q, k, v, params)
    parts = []
    for r in range(world):
        h0, h1 = vc.head_range(r, world, w.H)
        sl = [t[:, h0:h1].contiguous() for t in (q, k, v)]
        parts.append(vc.attention(*sl, params))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), full)
