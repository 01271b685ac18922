"""Seeded synthetic Q/K/V workloads for VC-Attention (V-Smooth + ExpCast-FP8).

This module only draws random numbers.  It holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Each (tensor, batch, head) slice has its own random stream, so one head can be
generated without the others (the oracle checks sampled heads of the large
workloads).  All draws are float32; the result is rounded to bf16 with
round-to-nearest-even (torch's CPU conversion).

Value distributions (the pages' long spatiotemporal video-DiT token sequences):

* Q and K: N(0, 1) per element, times a per-channel lognormal(0, 0.5) scale;
  each channel is an outlier channel (an extra x8) with probability 0.02.
* V, "pool" kind: a pool of P centroids, each N(0, 2^2) per channel; every
  token picks a pool entry uniformly at random; plus N(0, 0.3^2) noise.
* V, "grid" kind: the tokens are a (t, h, w) latent grid flattened t-major;
  every 3x5x5 (t, h, w) patch picks one pool entry (partial patches at the grid
  edge), plus the same noise.
* V outliers (both kinds): each token with probability 0.001 has one random
  channel multiplied by 20.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np
import torch

_TENSOR_ID = {"q": 1, "k": 2, "v": 3}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention problem plus the V-Smooth settings run on it."""

    name: str
    B: int
    H: int
    N: int
    d: int
    seed: int
    v_kind: str  # "pool" or "grid"
    pool: int  # number of V centroids in the generator's pool
    C: int  # k-means clusters
    iters: int  # k-means assignment passes
    block: int  # hardware block = KV tile (tokens)
    grid: Optional[Tuple[int, int, int]] = None  # (t, h, w) latent grid for "grid"
    resid_fmt: str = "e4m3"

    @property
    def T(self) -> int:
        return -(-self.N // self.block)

    @property
    def attn_flops(self) -> float:
        """Algorithmic attention flops, 4*B*H*N^2*d (QK^T and PV)."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_1k_d64", 1, 2, 1024, 64, 0, "pool", 16, 16, 8, 64),
        Workload("mid_32k_d128", 1, 40, 32768, 128, 1, "pool", 64, 64, 10, 128),
        Workload("grid720p_75600_d128", 1, 40, 75600, 128, 2, "grid", 64, 64, 10, 128,
                 grid=(21, 45, 80)),
        Workload("nvfp4_32k_d128", 1, 24, 32768, 128, 3, "pool", 64, 64, 10, 128,
                 resid_fmt="nvfp4"),
        Workload("longclip_245952_d128", 1, 48, 245952, 128, 4, "grid", 256, 256, 10, 128,
                 grid=(61, 48, 84)),
    ]
}


def _rng(w: Workload, tensor: str, b: int, h: int) -> np.random.Generator:
    ss = np.random.SeedSequence([w.seed, _TENSOR_ID[tensor], b, h])
    return np.random.Generator(np.random.PCG64(ss))


def _qk_head(rng: np.random.Generator, N: int, d: int) -> np.ndarray:
    scale = rng.lognormal(0.0, 0.5, size=d).astype(np.float32)
    outlier = rng.random(d) < 0.02
    scale = np.where(outlier, scale * np.float32(8.0), scale).astype(np.float32)
    x = rng.standard_normal((N, d), dtype=np.float32)
    x *= scale[None, :]
    return x


def _patch_ids(grid: Tuple[int, int, int]) -> Tuple[np.ndarray, int]:
    t, hh, ww = grid
    pt, ph, pw = -(-t // 3), -(-hh // 5), -(-ww // 5)
    ti = np.arange(t)[:, None, None] // 3
    hi = np.arange(hh)[None, :, None] // 5
    wi = np.arange(ww)[None, None, :] // 5
    ids = (ti * ph + hi) * pw + wi
    return ids.reshape(-1), pt * ph * pw


def _v_head(rng: np.random.Generator, w: Workload) -> np.ndarray:
    N, d = w.N, w.d
    pool = rng.normal(0.0, 2.0, size=(w.pool, d)).astype(np.float32)
    if w.v_kind == "pool":
        assign = rng.integers(0, w.pool, size=N)
    elif w.v_kind == "grid":
        ids, n_patch = _patch_ids(w.grid)
        if ids.shape[0] != N:
            raise ValueError(f"grid {w.grid} has {ids.shape[0]} tokens, workload has N={N}")
        patch_entry = rng.integers(0, w.pool, size=n_patch)
        assign = patch_entry[ids]
    else:
        raise ValueError(f"unknown V kind {w.v_kind!r}")
    x = pool[assign]
    x += rng.normal(0.0, 0.3, size=(N, d)).astype(np.float32)
    out_tok = np.nonzero(rng.random(N) < 0.001)[0]
    out_ch = rng.integers(0, d, size=N)[out_tok]
    x[out_tok, out_ch] *= np.float32(20.0)
    return x


def head_f32(w: Workload, tensor: str, b: int, h: int) -> np.ndarray:
    """float32 [N, d] draw for one (tensor, b, h) slice, before bf16 rounding."""
    rng = _rng(w, tensor, b, h)
    if tensor in ("q", "k"):
        return _qk_head(rng, w.N, w.d)
    if tensor == "v":
        return _v_head(rng, w)
    raise ValueError(tensor)


def head_bf16(w: Workload, tensor: str, b: int, h: int) -> torch.Tensor:
    """bf16 [N, d] CPU tensor for one (tensor, b, h) slice."""
    return torch.from_numpy(head_f32(w, tensor, b, h)).to(torch.bfloat16)


def head_bits(w: Workload, tensor: str, b: int, h: int) -> np.ndarray:
    """uint16 [N, d] bf16 bit patterns for one slice (the oracle's input form)."""
    return head_bf16(w, tensor, b, h).view(torch.int16).numpy().view(np.uint16)


def tensor_bf16(w: Workload, tensor: str, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Full bf16 [B, H, N, d] tensor; ``out`` may be a (pinned) host buffer."""
    if out is None:
        out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16)
    for b in range(w.B):
        for h in range(w.H):
            out[b, h].copy_(head_bf16(w, tensor, b, h))
    return out


def custom(name: str, B: int, H: int, N: int, d: int, seed: int, **kw) -> Workload:
    """A workload with the same generator at other sizes (tests and edge cases)."""
    base = dict(v_kind="pool", pool=16, C=16, iters=4, block=128 if d == 128 else 64)
    base.update(kw)
    return Workload(name, B, H, N, d, seed, **base)
