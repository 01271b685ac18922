"""The V-Smooth schedule over a denoising loop (host logic, no GPU): V-Smooth
only in the first quarter of the steps, as the pages report for B200
(chooseai.io news 7051, 意义与局限), with optional reuse of the regroup between
k-means runs."""
import pytest

import bit_fp8_attention_smooth_b200 as vc


def test_first_quarter_only():
    s = vc.VSmoothSchedule(50)
    modes = [s.mode(i) for i in range(50)]
    # steps 0..12 start in the first quarter of 50 (12 < 12.5), the rest do not
    assert modes == [1] * 13 + [0] * 37
    assert [vc.VSmoothSchedule(8).mode(i) for i in range(8)] == [1, 1, 0, 0, 0, 0, 0, 0]
    assert [vc.VSmoothSchedule(1).mode(0)] == [1]


def test_recluster_every_reuses_between():
    s = vc.VSmoothSchedule(40, recluster_every=4)
    assert [s.mode(i) for i in range(12)] == [1, 2, 2, 2, 1, 2, 2, 2, 1, 2, 0, 0]


def test_fraction_edges_and_params():
    assert all(vc.VSmoothSchedule(10, on_fraction=1.0).mode(i) == 1 for i in range(10))
    assert all(vc.VSmoothSchedule(10, on_fraction=0.0).mode(i) == 0 for i in range(10))
    base = vc.Params(C=32, iters=5, block=128, resid_fmt=1)
    p = vc.VSmoothSchedule(20, recluster_every=2).params(base, 1)
    assert p.smooth == 2 and p.C == 32 and p.resid_fmt == 1 and p.c().smooth == 2


@pytest.mark.parametrize("kw", [dict(total_steps=0), dict(total_steps=5, on_fraction=1.5),
                                dict(total_steps=5, recluster_every=0)])
def test_rejects_bad_schedules(kw):
    with pytest.raises(ValueError):
        vc.VSmoothSchedule(**kw)


def test_rejects_steps_outside_the_loop():
    s = vc.VSmoothSchedule(4)
    with pytest.raises(ValueError):
        s.mode(4)
    with pytest.raises(ValueError):
        s.mode(-1)
