"""VC-Attention (V-Smooth + ExpCast-FP8) forward for NVIDIA B200, Python binding.

A thin ctypes layer over the C ABI in include/vc_attention.h (libvcattn.so,
built in-tree by ``python -m bit_fp8_attention_smooth_b200.build``).  It only
marshals arguments: torch supplies device memory and streams, every step of
the computation runs in the library's CUDA kernels.  There is no CPU fallback:
if the library is missing or the device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Dict, Optional

import torch

from . import synth  # noqa: F401  (seeded workloads, no method arithmetic)

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvcattn.so")

VC_OK, VC_ERR_INVALID_ARG, VC_ERR_UNSUPPORTED, VC_ERR_CUDA, VC_ERR_DEVICE_TIMEOUT, VC_ERR_WORKSPACE = range(6)


class VcError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32)]


class _Params(ctypes.Structure):
    _fields_ = [("C", ctypes.c_int32), ("iters", ctypes.c_int32), ("block", ctypes.c_int32),
                ("beta", ctypes.c_int32), ("smooth", ctypes.c_int32), ("resid_fmt", ctypes.c_int32),
                ("wait_limit_ns", ctypes.c_int64)]


class _Prep(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p)
                for n in ("perm", "labels", "k_fp8", "k_scale", "vt_fp8", "v_mean", "v_scale", "v_bscale")]


PREP_FIELDS = ("perm", "labels", "k_fp8", "k_scale", "vt_fp8", "v_mean", "v_scale", "v_bscale")

_lib = None


def lib():
    """Load libvcattn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m bit_fp8_attention_smooth_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, S, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64
        PS, PP, PR = ctypes.POINTER(_Shape), ctypes.POINTER(_Params), ctypes.POINTER(_Prep)
        sig = {
            "vc_abi_version": (ctypes.c_int, []),
            "vc_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "vc_prep_buffer_bytes": (ctypes.c_int, [PS, PP, ctypes.POINTER(S)]),
            "vc_workspace_bytes": (ctypes.c_int, [PS, PP, ctypes.POINTER(S)]),
            "vc_smooth_prepare": (ctypes.c_int, [P, P, PS, PP, PR, P, S, P]),
            "vc_attn_fwd": (ctypes.c_int, [P, PR, PS, PP, P, P, S, P]),
            "vc_attn_fwd_masked": (ctypes.c_int, [P, PR, PS, PP, P, P, P, S, P]),
            "vc_attention": (ctypes.c_int, [P, P, P, PS, PP, PR, P, P, S, P]),
            "vc_attention_host": (ctypes.c_int, [P, P, P, P, PS, PP, ctypes.c_int, P, P, P, P, PR, P, S, P, P, P]),
            "vc_check": (ctypes.c_int, [P, P]),
            "vc_attn_fwd_noalloc": (ctypes.c_int, [P, PR, PS, PP, P, P]),
            "vc_e4m3_encode": (ctypes.c_int, [P, P, i64, P]),
            "vc_quantize_q": (ctypes.c_int, [P, P, P, i64, ctypes.c_int, P]),
            "vc_expcast_bytes": (ctypes.c_int, [P, P, P, P, i64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().vc_status_string(status).decode()
    except Exception:  # library not loadable: still give a readable message
        return f"status {status}"


def _ok(status: int, what: str):
    if status != VC_OK:
        raise VcError(status, what)


@dataclasses.dataclass
class Params:
    """V-Smooth / ExpCast settings (see vc_params in include/vc_attention.h)."""

    C: int = 64
    iters: int = 10
    block: int = 128
    beta: int = 64
    smooth: int = 1  # 1 V-Smooth, 0 plain FP8 V, 2 V-Smooth reusing the prep's regroup
    resid_fmt: int = 0
    wait_limit_ns: int = 0

    def c(self) -> _Params:
        return _Params(self.C, self.iters, self.block, self.beta, int(self.smooth), self.resid_fmt, self.wait_limit_ns)

    @classmethod
    def for_workload(cls, w, **kw) -> "Params":
        """The workload's k-means, block and residual format (the 4-bit
        residual for a workload that names nvfp4), overridable by keyword."""
        kw.setdefault("resid_fmt", 1 if getattr(w, "resid_fmt", "e4m3") == "nvfp4" else 0)
        return cls(C=w.C, iters=w.iters, block=w.block, **kw)


@dataclasses.dataclass(frozen=True)
class VSmoothSchedule:
    """Which prep each step of a denoising loop runs.

    The pages run V-Smooth only in the first quarter of the denoising steps on
    B200 and call its cost a scheduling trade-off (chooseai.io news 7051,
    意义与局限).  Step i (0-based) of `total_steps` runs V-Smooth when
    i < on_fraction * total_steps, and plain per-channel FP8 V after that.
    Within the V-Smooth steps, k-means runs on every `recluster_every`-th step
    (always on step 0); the steps in between reuse the latest regroup
    (Params.smooth = 2), which leaves only the block quantisation to run.
    """

    total_steps: int
    on_fraction: float = 0.25
    recluster_every: int = 1

    def __post_init__(self):
        if self.total_steps < 1 or not 0.0 <= self.on_fraction <= 1.0 or self.recluster_every < 1:
            raise ValueError(f"bad schedule {self}")

    def mode(self, step: int) -> int:
        """Params.smooth for this step: 1 cluster, 2 reuse the regroup, 0 off."""
        if not 0 <= step < self.total_steps:
            raise ValueError(f"step {step} outside 0..{self.total_steps - 1}")
        if step >= self.on_fraction * self.total_steps:
            return 0
        return 1 if step % self.recluster_every == 0 else 2

    def params(self, base: Params, step: int) -> Params:
        return dataclasses.replace(base, smooth=self.mode(step))


def head_range(rank: int, world: int, H: int):
    """Heads [h0, h1) of rank `rank` when H heads are split over `world`
    ranks: contiguous, sizes differing by at most one.  Every (b, h) problem of
    the path is independent, k-means included, so a head split needs no
    exchange on the data path."""
    if world < 1 or not 0 <= rank < world or H < 0:
        raise ValueError(f"bad split: rank {rank} of {world}, {H} heads")
    return H * rank // world, H * (rank + 1) // world


def gather_heads(o_local: torch.Tensor, H: int, group=None) -> torch.Tensor:
    """All-gather per-rank output heads [B, h1 - h0, N, d] (this rank's
    head_range) into the full [B, H, N, d] on every rank, over
    torch.distributed (NCCL for CUDA tensors).  Only for callers that need
    every head on every rank: the attention itself needs no collective."""
    import torch.distributed as dist

    world, rank = dist.get_world_size(group), dist.get_rank(group)
    B, h_loc, N, d = o_local.shape
    h0, h1 = head_range(rank, world, H)
    if h1 - h0 != h_loc:
        raise ValueError(f"rank {rank} holds {h_loc} heads, its range is {h1 - h0}")
    width = -(-H // world)  # uneven splits travel padded to the widest rank
    send = torch.zeros((B, width, N, d), dtype=o_local.dtype, device=o_local.device)
    send[:, :h_loc] = o_local
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send, group=group)
    out = torch.empty((B, H, N, d), dtype=o_local.dtype, device=o_local.device)
    for r, part in enumerate(parts):
        a, b = head_range(r, world, H)
        out[:, a:b] = part[:, :b - a]
    return out


def _shape(t: torch.Tensor) -> _Shape:
    if t.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    B, H, N, d = t.shape
    return _Shape(B, H, N, d)


def _check_input(t: torch.Tensor, name: str):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def prep_sizes(shape, params: Params):
    sh = _Shape(*shape) if not isinstance(shape, _Shape) else shape
    out = (ctypes.c_size_t * 8)()
    _ok(lib().vc_prep_buffer_bytes(ctypes.byref(sh), ctypes.byref(params.c()), out), "vc_prep_buffer_bytes")
    return list(out)


def workspace_bytes(shape, params: Params) -> int:
    sh = _Shape(*shape) if not isinstance(shape, _Shape) else shape
    n = ctypes.c_size_t()
    _ok(lib().vc_workspace_bytes(ctypes.byref(sh), ctypes.byref(params.c()), ctypes.byref(n)), "vc_workspace_bytes")
    return n.value


def alloc_workspace(shape, params: Params, device="cuda") -> torch.Tensor:
    """Zero-filled workspace (the status word must start at 0)."""
    return torch.zeros(workspace_bytes(shape, params), dtype=torch.uint8, device=device)


def prep_layout(shape, params: Params) -> Dict[str, tuple]:
    """Logical shape and dtype of each prep buffer (the 4-bit residual,
    resid_fmt 1: vt_fp8 holds two E2M1 codes a byte and v_bscale the UE4M3
    block scales; v_bscale exists only then)."""
    B, H, N, d = shape
    T = -(-N // params.block)
    Tp = T * params.block
    fp4 = params.resid_fmt == 1
    layout = {
        "perm": ((B, H, N), torch.int32),
        "labels": ((B, H, N), torch.int32),
        "k_fp8": ((B, H, Tp, d), torch.uint8),
        "k_scale": ((B, H, T), torch.float32),
        "vt_fp8": ((B, H, d, Tp // 2 if fp4 else Tp), torch.uint8),
        "v_mean": ((B, H, T, d), torch.float32),
        "v_scale": ((B, H, d), torch.float32),
    }
    if fp4:
        layout["v_bscale"] = ((B, H, T, d, params.block // 16), torch.uint8)
    return layout


def alloc_prep(shape, params: Params, device="cuda") -> Dict[str, torch.Tensor]:
    """Caller-owned prep buffers with their logical shapes and dtypes."""
    return {n: torch.empty(sh, dtype=dt, device=device) for n, (sh, dt) in prep_layout(shape, params).items()}


def _check_like(t, name: str, shape, dtype, device):
    """The library indexes raw pointers by the problem shape, so every buffer
    it touches must have exactly that shape and dtype, contiguous, on the
    device of the call."""
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or tuple(t.shape) != tuple(shape) \
            or not t.is_contiguous() or t.device != device:
        got = (f"{t.dtype} {tuple(t.shape)} on {t.device}" + ("" if t.is_contiguous() else ", not contiguous")
               if isinstance(t, torch.Tensor) else type(t).__name__)
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {device} "
                         f"(got {got})")


def _check_prep(prep, shape, params: Params, device):
    for n, (sh, dt) in prep_layout(shape, params).items():
        if n not in prep:
            raise ValueError(f"prep buffer {n!r} is missing (resid_fmt {params.resid_fmt})")
        _check_like(prep[n], f"prep[{n!r}]", sh, dt, device)


def _check_out(out, Q: torch.Tensor):
    _check_like(out, "out", Q.shape, torch.bfloat16, Q.device)


def _ws_args(ws: torch.Tensor, device):
    """Workspace pointer and size in bytes (the library checks the size)."""
    if not isinstance(ws, torch.Tensor) or not ws.is_contiguous() or ws.device != device:
        raise ValueError(f"workspace must be a contiguous tensor on {device}")
    return ws.data_ptr(), ws.numel() * ws.element_size()


def _prep_struct(prep: Dict[str, torch.Tensor]) -> _Prep:
    vals = []
    for n in PREP_FIELDS:
        t = prep.get(n)
        vals.append(None if t is None else t.data_ptr())
    return _Prep(*vals)


def smooth_prepare(K: torch.Tensor, V: torch.Tensor, params: Params, prep=None, workspace=None, stream=None):
    """V-Smooth prep; returns the prep buffers (k-means labels included)."""
    _check_input(K, "K")
    _check_like(V, "V", K.shape, torch.bfloat16, K.device)
    shape = tuple(K.shape)
    prep = alloc_prep(shape, params, K.device) if prep is None else prep
    _check_prep(prep, shape, params, K.device)
    ws_ptr, ws_bytes = _ws_args(alloc_workspace(shape, params, K.device) if workspace is None else workspace, K.device)
    st = lib().vc_smooth_prepare(K.data_ptr(), V.data_ptr(), ctypes.byref(_shape(K)), ctypes.byref(params.c()),
                                 ctypes.byref(_prep_struct(prep)), ws_ptr, ws_bytes, _stream(stream))
    _ok(st, "vc_smooth_prepare")
    return prep


def attn_fwd(Q: torch.Tensor, prep, params: Params, out=None, workspace=None, stream=None,
             tile_mask: Optional[torch.Tensor] = None) -> torch.Tensor:
    """ExpCast-FP8 attention over prepped K/V; returns O (bf16, Q's layout).
    tile_mask (uint8 [B, H, ceil(N/128), ceil(N/block)] on the device) makes it
    block-sparse: nonzero keeps a key tile for a query tile."""
    _check_input(Q, "Q")
    shape = tuple(Q.shape)
    _check_prep(prep, shape, params, Q.device)
    out = torch.empty_like(Q) if out is None else out
    _check_out(out, Q)
    ws_ptr, ws_bytes = _ws_args(alloc_workspace(shape, params, Q.device) if workspace is None else workspace, Q.device)
    if tile_mask is None:
        st = lib().vc_attn_fwd(Q.data_ptr(), ctypes.byref(_prep_struct(prep)), ctypes.byref(_shape(Q)),
                               ctypes.byref(params.c()), out.data_ptr(), ws_ptr, ws_bytes, _stream(stream))
        _ok(st, "vc_attn_fwd")
        return out
    B, H, N, _ = shape
    want = (B, H, -(-N // 128), -(-N // params.block))
    if tile_mask.dtype != torch.uint8 or tuple(tile_mask.shape) != want or not tile_mask.is_contiguous() \
            or tile_mask.device != Q.device:
        raise ValueError(f"tile_mask must be a contiguous uint8 {want} tensor on {Q.device}")
    st = lib().vc_attn_fwd_masked(Q.data_ptr(), ctypes.byref(_prep_struct(prep)), ctypes.byref(_shape(Q)),
                                  ctypes.byref(params.c()), tile_mask.data_ptr(), out.data_ptr(), ws_ptr,
                                  ws_bytes, _stream(stream))
    _ok(st, "vc_attn_fwd_masked")
    return out


def attention(Q, K, V, params: Params, out=None, prep=None, workspace=None, stream=None) -> torch.Tensor:
    """The drop-in call: V-Smooth prep then ExpCast-FP8 attention."""
    _check_input(Q, "Q")
    for t, n in ((K, "K"), (V, "V")):
        _check_like(t, n, Q.shape, torch.bfloat16, Q.device)
    shape = tuple(Q.shape)
    out = torch.empty_like(Q) if out is None else out
    _check_out(out, Q)
    prep = alloc_prep(shape, params, Q.device) if prep is None else prep
    _check_prep(prep, shape, params, Q.device)
    ws_ptr, ws_bytes = _ws_args(alloc_workspace(shape, params, Q.device) if workspace is None else workspace, Q.device)
    st = lib().vc_attention(Q.data_ptr(), K.data_ptr(), V.data_ptr(), ctypes.byref(_shape(Q)),
                            ctypes.byref(params.c()), ctypes.byref(_prep_struct(prep)), out.data_ptr(),
                            ws_ptr, ws_bytes, _stream(stream))
    _ok(st, "vc_attention")
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20


def attn_fwd_noalloc(Q: torch.Tensor, prep, params: Params, out=None, stream=None) -> torch.Tensor:
    """vc_attn_fwd without a workspace, for callers that cannot allocate at
    call time: the library's static per-device scratch holds the quantised Q.
    Problems larger than the scratch raise VcError(VC_ERR_WORKSPACE); calls
    that overlap on the GPU race on the shared scratch."""
    _check_input(Q, "Q")
    _check_prep(prep, tuple(Q.shape), params, Q.device)
    out = torch.empty_like(Q) if out is None else out
    _check_out(out, Q)
    st = lib().vc_attn_fwd_noalloc(Q.data_ptr(), ctypes.byref(_prep_struct(prep)), ctypes.byref(_shape(Q)),
                                   ctypes.byref(params.c()), out.data_ptr(), _stream(stream))
    _ok(st, "vc_attn_fwd_noalloc")
    return out


def check(workspace: torch.Tensor, stream=None) -> None:
    """Synchronise and raise VcError if a kernel recorded a device-side timeout."""
    ws_ptr, _ = _ws_args(workspace, workspace.device)
    _ok(lib().vc_check(ws_ptr, _stream(stream)), "vc_check")


def e4m3_encode(x: torch.Tensor, stream=None) -> torch.Tensor:
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _ok(lib().vc_e4m3_encode(x.data_ptr(), out.data_ptr(), x.numel(), _stream(stream)), "vc_e4m3_encode")
    return out


def quantize_q(q: torch.Tensor, stream=None):
    """Per-token E4M3 Q as the attention call quantises it: q bf16 [..., d] ->
    (codes uint8 [..., d], scales fp32 [...])."""
    if q.dtype != torch.bfloat16 or not q.is_cuda or not q.is_contiguous() or q.dim() < 1:
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    d = q.shape[-1]
    codes = torch.empty(q.shape, dtype=torch.uint8, device=q.device)
    scales = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    _ok(lib().vc_quantize_q(q.data_ptr(), codes.data_ptr(), scales.data_ptr(), q.numel() // max(d, 1), d,
                            _stream(stream)), "vc_quantize_q")
    return codes, scales


def expcast_bytes(A: torch.Tensor, s: torch.Tensor, cb: torch.Tensor, stream=None) -> torch.Tensor:
    if not A.is_cuda:
        raise ValueError("A, s and cb must be CUDA tensors")
    for t, n in ((A, "A"), (s, "s"), (cb, "cb")):
        _check_like(t, n, A.shape, torch.float32, A.device)
    out = torch.empty(A.shape, dtype=torch.uint8, device=A.device)
    _ok(lib().vc_expcast_bytes(A.data_ptr(), s.data_ptr(), cb.data_ptr(), out.data_ptr(), A.numel(), _stream(stream)),
        "vc_expcast_bytes")
    return out


class _HostSet:
    """One set of device buffers and streams for vc_attention_host."""

    def __init__(self, shape, params: Params, device):
        self.q = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.k = torch.empty_like(self.q)
        self.v = torch.empty_like(self.q)
        self.o = torch.empty_like(self.q)
        self.prep = alloc_prep(shape, params, device)
        self.ws = alloc_workspace(shape, params, device)
        self.streams = [torch.cuda.Stream(device=self.q.device) for _ in range(3)]  # h2d, compute, d2h


class HostAttention:
    """End-to-end call from pinned host buffers (vc_attention_host): the B*H
    problems run in `groups` runs, each one's H2D copy, prep + attention and
    D2H copy on three streams, so the transfers of one run overlap the
    computation of its neighbours.  With `sets` = 2 the calls alternate
    between two independent sets of device buffers, workspaces and streams,
    so the copies of one call also overlap the computation of the previous
    one.  Device memory is allocated once, in the constructor."""

    def __init__(self, shape, params: Params, device="cuda", groups: int = 4, sets: int = 2):
        self.shape, self.params, self.groups = tuple(shape), params, groups
        self.sets = [_HostSet(self.shape, params, device) for _ in range(max(1, sets))]
        self.calls = 0
        n = 1
        for x in self.shape:
            n *= x
        self.h2d_bytes = 3 * n * 2
        self.d2h_bytes = n * 2

    @property
    def ws(self):  # workspace of the set the last call used (for vc_check)
        return self.sets[(self.calls - 1) % len(self.sets)].ws

    def check(self):
        """Synchronise every set and raise VcError on a recorded device error."""
        for st in self.sets:
            _ok(lib().vc_check(st.ws.data_ptr(), ctypes.c_void_p(st.streams[2].cuda_stream)), "vc_check")

    def __call__(self, q_host, k_host, v_host, o_host, stream=None):
        for t, n in ((q_host, "q_host"), (k_host, "k_host"), (v_host, "v_host"), (o_host, "o_host")):
            if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or tuple(t.shape) != self.shape:
                raise ValueError(f"{n} must be a contiguous bf16 host tensor of shape {self.shape}")
        st = self.sets[self.calls % len(self.sets)]
        self.calls += 1
        cur = torch.cuda.current_stream(st.q.device) if stream is None else stream
        for s in st.streams:
            s.wait_stream(cur)
        s_in, s_c, s_out = st.streams
        rc = lib().vc_attention_host(
            q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), o_host.data_ptr(), ctypes.byref(_Shape(*self.shape)),
            ctypes.byref(self.params.c()), self.groups, st.q.data_ptr(), st.k.data_ptr(), st.v.data_ptr(),
            st.o.data_ptr(), ctypes.byref(_prep_struct(st.prep)), st.ws.data_ptr(), st.ws.numel(),
            ctypes.c_void_p(s_in.cuda_stream), ctypes.c_void_p(s_c.cuda_stream), ctypes.c_void_p(s_out.cuda_stream))
        _ok(rc, "vc_attention_host")
        # The caller's stream moves on once O is back; the next call (other
        # set) does not wait for this one.
        return _HostDone(cur, s_out, s_c)


class _HostDone:
    """Returned by HostAttention: `wait()` makes the caller's stream wait for
    the call's output copy (the call itself leaves the caller's stream free,
    so consecutive calls overlap)."""

    def __init__(self, cur, s_out, s_c):
        self._cur, self._s_out, self._s_c = cur, s_out, s_c

    def wait(self):
        self._cur.wait_stream(self._s_out)
        self._cur.wait_stream(self._s_c)
