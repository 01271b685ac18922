"""The V-Smooth prep's k-means at the edges of its pass schedule and of its
two flows, against the oracle (chooseai.io news 7051, V-Smooth section: a
lightweight k-means groups similar value tokens before the blocks are cut).

The library runs one fused launch a pass for C <= 64, and a pass of separate
assignment and update launches for larger C.  The fused passes differ by
their place in the schedule: the first sums every token, the second moves
the tokens whose label changed through the update warps, later ones move
them with atomics, and the last keeps no sums.  Pass counts of 1, 2 and 3
reach each of those first and last cases; C = 64 and 65 sit on both sides
of the switch between the flows (C = 65 pads to 80 clusters on the tensor
cores).

Checks, per head: the regroup is a stable sort of the GPU's own labels;
every label that differs from the oracle's is still a valid fp64 argmin
(within the near-tie margin of the minimum, to the oracle's centroids); the
quantiser bytes equal the oracle's on the GPU's regroup."""
import numpy as np
import pytest

import oracle
from bit_fp8_attention_smooth_b200 import synth
from gpu_common import BETA, bits, check_labels_valid, check_perm, gpu_prep_head, make_inputs, oracle_prep_on_perm, \
    prep_to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vc():
    import bit_fp8_attention_smooth_b200 as m

    m.lib()
    return m


@pytest.mark.parametrize("C, iters", [(8, 1), (8, 2), (8, 3), (64, 3), (65, 3)],
                         ids=["C8_1pass", "C8_2pass", "C8_3pass", "C64_fused", "C65_split"])
def test_kmeans_pass_schedule(vc, C, iters):
    w = synth.custom(f"modes_{C}_{iters}", 1, 2, 1500, 128, 51 + C + iters, pool=C, C=C, iters=iters, block=128)
    q, k, v, qd, kd, vd = make_inputs(w)
    params = vc.Params.for_workload(w, beta=BETA)
    ws = vc.alloc_workspace(tuple(kd.shape), params)
    prep = prep_to_host(vc.smooth_prepare(kd, vd, params, workspace=ws))
    vc.check(ws)
    for h in range(w.H):
        ref = oracle.prep_head(bits(k[0, h]), bits(v[0, h]), C=w.C, iters=w.iters, bk=w.block, smooth=True)
        got = gpu_prep_head(prep, 0, h, w.N, w.block)
        check_perm(got["perm"], got["labels"], w.N)
        assert np.array_equal(got["perm"], oracle.stable_perm(got["labels"], w.C))
        assert (got["labels"] == ref["labels"]).mean() >= 0.999
        check_labels_valid(bits(v[0, h]), got["labels"], ref["labels"], ref["centroids"])
        own = oracle_prep_on_perm(bits(k[0, h]), bits(v[0, h]), got["perm"], w.block)
        for key in ("khat", "ksc", "vmu", "vsc", "vhat"):
            assert np.array_equal(got[key], own[key]), (h, key)
