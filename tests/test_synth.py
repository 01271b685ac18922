"""The seeded workload generator: determinism, per-head independence, and the
value structure the workloads are meant to have."""
import numpy as np
import torch

from bit_fp8_attention_smooth_b200 import synth


def test_workload_table():
    w = synth.WORKLOADS
    assert (w["tiny_1k_d64"].N, w["tiny_1k_d64"].d, w["tiny_1k_d64"].T) == (1024, 64, 16)
    assert w["mid_32k_d128"].T == 256
    assert w["grid720p_75600_d128"].T == 591 and 75600 % 128 == 80
    assert w["longclip_245952_d128"].T == 1922 and 245952 % 128 == 64
    assert w["mid_32k_d128"].attn_flops == 4 * 40 * 32768 ** 2 * 128
    g = w["longclip_245952_d128"].grid
    assert g[0] * g[1] * g[2] == 245952


def test_deterministic_and_independent_heads():
    w = synth.WORKLOADS["tiny_1k_d64"]
    a = synth.head_bits(w, "q", 0, 0)
    assert np.array_equal(a, synth.head_bits(w, "q", 0, 0))
    assert not np.array_equal(a, synth.head_bits(w, "q", 0, 1))
    assert not np.array_equal(a, synth.head_bits(w, "k", 0, 0))
    full = synth.tensor_bf16(w, "v")
    assert full.shape == (1, 2, 1024, 64) and full.dtype == torch.bfloat16
    assert torch.equal(full[0, 1], synth.head_bf16(w, "v", 0, 1))


def test_value_structure():
    w = synth.custom("s", 1, 1, 20000, 64, 5, pool=16)
    v = synth.head_f32(w, "v", 0, 0)
    # every token is a pool centroid plus small noise (outliers aside)
    pool_like = synth._rng(w, "v", 0, 0).normal(0.0, 2.0, size=(16, 64)).astype(np.float32)
    d2 = ((v[:, None, :] - pool_like[None]) ** 2).sum(-1).min(1)
    assert np.median(d2) < 64 * 0.3 ** 2 * 1.5
    q = synth.head_f32(w, "q", 0, 0)
    assert abs(q.std() - 1.3) < 1.2


def test_grid_patches_share_a_centroid():
    w = synth.custom("g", 1, 1, 6 * 10 * 10, 64, 6, v_kind="grid", grid=(6, 10, 10), pool=50)
    ids, n_patch = synth._patch_ids(w.grid)
    assert n_patch == 2 * 2 * 2 and ids.shape == (600,)
    v = synth.head_f32(w, "v", 0, 0)
    for p in range(n_patch):
        rows = v[ids == p]
        med = np.median(rows, axis=0)
        assert np.median(np.abs(rows - med)) < 0.5


def test_generator_holds_no_method_arithmetic():
    """Both the oracle and the CUDA path are fed from synth.py, so it must not
    load either of them or compute any step of the method: it imports only
    numpy, torch and the standard library, and calls no quantiser, ExpCast,
    k-means or library routine."""
    import ast
    import os

    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "bit_fp8_attention_smooth_b200", "synth.py"), encoding="utf-8").read()
    tree = ast.parse(src)
    mods = {a.name.split(".")[0] for n in ast.walk(tree) if isinstance(n, ast.Import) for a in n.names}
    mods |= {(n.module or "").split(".")[0] for n in ast.walk(tree) if isinstance(n, ast.ImportFrom)}
    assert mods <= {"__future__", "dataclasses", "typing", "numpy", "torch"}, mods
    calls = {n.func.attr if isinstance(n.func, ast.Attribute) else getattr(n.func, "id", "")
             for n in ast.walk(tree) if isinstance(n, ast.Call)}
    banned = {c for c in calls if any(w in c.lower() for w in ("e4m3", "e2m1", "expcast", "kmeans", "quant", "lib"))}
    assert not banned, banned
