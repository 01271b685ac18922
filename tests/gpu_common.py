"""Shared helpers of the GPU parity tests: run the oracle and the CUDA path on
the same seeded inputs and compare.  Inputs come from the seeded generator
only; oracle results never come from the CUDA path."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import bit_fp8_attention_smooth_b200 as vc
from bit_fp8_attention_smooth_b200 import synth

BETA = 64
REL_L2_TOL = 1e-2
COS_TOL = 0.9995


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CPU tensor -> uint16 bit patterns (oracle input form)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def metrics(out: np.ndarray, ref: np.ndarray):
    out = out.astype(np.float64).ravel()
    ref = ref.astype(np.float64).ravel()
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    cos = float(out @ ref / (np.linalg.norm(out) * np.linalg.norm(ref)))
    psnr = 20 * np.log10(np.abs(ref).max() / np.sqrt(np.mean((out - ref) ** 2)))
    return float(rel), cos, float(psnr)


def make_inputs(w, device="cuda"):
    q, k, v = (synth.tensor_bf16(w, t) for t in "qkv")
    return q, k, v, q.to(device), k.to(device), v.to(device)


def prep_to_host(prep):
    return {k: v.cpu() for k, v in prep.items()}


def oracle_head(q, k, v, b, h, rows, w, smooth=True, threads=None):
    """Oracle prep + replay + exact attention for one head; q/k/v are CPU bf16 [B,H,N,d]."""
    qb, kb, vb = bits(q[b, h]), bits(k[b, h]), bits(v[b, h])
    r = oracle.forward_head(qb, kb, vb, rows, C=w.C, iters=w.iters, bk=w.block, beta=BETA, smooth=smooth,
                            threads=threads)
    r["exact"] = oracle.attn_exact(qb, kb, vb, rows, threads=threads)
    return r


def gpu_prep_head(prep_h, b, h, n, bk):
    """GPU prep buffers of one head in the oracle's logical layout."""
    d = prep_h["k_fp8"].shape[-1]
    return dict(
        perm=prep_h["perm"][b, h].numpy(),
        labels=prep_h["labels"][b, h].numpy(),
        khat=prep_h["k_fp8"][b, h].numpy(),
        ksc=prep_h["k_scale"][b, h].numpy(),
        vhat=np.ascontiguousarray(prep_h["vt_fp8"][b, h].numpy().T),
        vmu=prep_h["v_mean"][b, h].numpy(),
        vsc=prep_h["v_scale"][b, h].numpy(),
    )


def oracle_prep_to_gpu(preps, shape, bk, device="cuda"):
    """Oracle prep results (per head, [B][H] nested list) as GPU prep buffers."""
    B, H, N, d = shape
    T = -(-N // bk)
    out = vc.alloc_prep(shape, vc.Params(block=bk), device)
    for b in range(B):
        for h in range(H):
            p = preps[b][h]
            out["perm"][b, h] = torch.from_numpy(p["perm"])
            out["labels"][b, h] = torch.from_numpy(p["labels"])
            out["k_fp8"][b, h] = torch.from_numpy(p["khat"])
            out["k_scale"][b, h] = torch.from_numpy(p["ksc"])
            out["vt_fp8"][b, h] = torch.from_numpy(np.ascontiguousarray(p["vhat"].T))
            out["v_mean"][b, h] = torch.from_numpy(p["vmu"])
            out["v_scale"][b, h] = torch.from_numpy(p["vsc"])
    return out


def oracle_prep_on_perm(k_bits, v_bits, perm, bk, smooth=True, resid_fmt=0):
    """The oracle's quantisers (K, V-Smooth residual) applied in a given
    regroup order -- the GPU's own, so that byte parity of the quantisers does
    not hinge on the two k-means agreeing on every near tie."""
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    khat, ksc = oracle.quant_k(k_bits, perm, bk)
    if resid_fmt == 1:
        vq, vgs, vmu, vsc = oracle.smooth_v_nvfp4(v_bits, perm, bk, smooth)
        return dict(perm=perm, khat=khat, ksc=ksc, vq=vq, vgs=vgs, vmu=vmu, vsc=vsc)
    vhat, vmu, vsc = oracle.smooth_v(v_bits, perm, bk, smooth)
    return dict(perm=perm, khat=khat, ksc=ksc, vhat=vhat, vmu=vmu, vsc=vsc)


# k-means decisions the tensor-core distance leaves open are re-decided in
# fp64 when two clusters lie within this fraction of (|v| + max|c|)^2 (the
# library's near-tie margin).
KMEANS_MARGIN = 2.0 ** -13


def check_labels_valid(v_bits, gpu_labels, ref_labels, centroids):
    """Where the GPU's k-means label differs from the oracle's, the GPU's
    cluster must still be a valid argmin: its fp64 squared distance (to the
    oracle's final centroids) lies within the near-tie margin of the minimum."""
    diff = np.nonzero(np.asarray(gpu_labels) != np.asarray(ref_labels))[0]
    if diff.size == 0:
        return 0
    v = bits_to_f64(v_bits[diff])
    c = np.asarray(centroids, dtype=np.float64)
    d2 = ((v[:, None, :] - c[None, :, :]) ** 2).sum(-1)
    got = d2[np.arange(diff.size), np.asarray(gpu_labels)[diff]]
    rad = np.linalg.norm(v, axis=1) + np.linalg.norm(c, axis=1).max()
    excess = got - d2.min(1)
    assert np.all(excess <= KMEANS_MARGIN * rad ** 2), (diff[:5], excess[:5], (KMEANS_MARGIN * rad ** 2)[:5])
    return int(diff.size)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 values (test helper)."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def check_perm(perm: np.ndarray, labels: np.ndarray, n: int):
    """perm is a bijection, labels[perm] is non-decreasing, and stable."""
    assert np.array_equal(np.sort(perm), np.arange(n))
    lp = labels[perm]
    assert np.all(np.diff(lp) >= 0)
    same = np.diff(lp) == 0
    assert np.all(np.diff(perm)[same] > 0)
