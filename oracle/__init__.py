"""ctypes front end of the plain C oracle (vc_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check, and the
benchmark's CPU-baseline leg and `--impl reference` arm are the only users.  It takes numpy arrays and
returns numpy arrays; it imports nothing from the CUDA package, and the CUDA
package never imports it.

Every function here is a thin argument marshaller around one C routine; the
arithmetic, and the citation of the passage it follows, live in vc_oracle.c.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# VC_ORACLE_SRC points the tests at another copy of the C source (the mutation
# test plants one mistake in a copy and checks that the pins fail); the
# library builds beside whichever source is used.
_SRC = os.environ.get("VC_ORACLE_SRC") or os.path.join(_HERE, "vc_oracle.c")
_SO = os.path.join(os.path.dirname(os.path.abspath(_SRC)), "_build", "libvcoracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile vc_oracle.c (strict IEEE: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_SO), exist_ok=True)
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
             "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f32, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        sig = {
            "vo_e4m3_value": (f64, [ctypes.c_uint8]),
            "vo_e4m3_encode": (ctypes.c_uint8, [f32]),
            "vo_e4m3_encode_array": (None, [P, i64, P]),
            "vo_e4m3_value_array": (None, [P, i64, P]),
            "vo_expcast_byte": (ctypes.c_uint8, [f32, f32, f32]),
            "vo_expcast_array": (None, [P, P, P, i64, P]),
            "vo_kmeans": (None, [P, i32, i32, i32, i32, P, P]),
            "vo_stable_perm": (None, [P, i32, i32, P]),
            "vo_quant_q": (None, [P, i32, i32, P, P]),
            "vo_quant_k": (None, [P, i32, i32, i32, P, P, P]),
            "vo_smooth_v": (None, [P, i32, i32, i32, P, i32, P, P, P]),
            "vo_e2m1_value": (f64, [ctypes.c_uint8]),
            "vo_e2m1_encode": (ctypes.c_uint8, [f32]),
            "vo_e2m1_value_array": (None, [P, i64, P]),
            "vo_e2m1_encode_array": (None, [P, i64, P]),
            "vo_nvfp4_block_array": (None, [P, i64, i32, P, P]),
            "vo_smooth_v_nvfp4": (None, [P, i32, i32, i32, P, i32, P, P, P, P]),
            "vo_attn_emul": (None, [P, P, i32, P, P, P, P, P, i32, i32, i32, f64, i32, i32, i32, P, P, P, P]),
            "vo_attn_exact": (None, [P, P, P, P, i32, i32, i32, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------- codec
def e4m3_value(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().vo_e4m3_value_array(_p(c), c.size, _p(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().vo_e4m3_encode_array(_p(x), x.size, _p(out))
    return out


def e2m1_value(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().vo_e2m1_value_array(_p(c), c.size, _p(out))
    return out


def e2m1_encode(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().vo_e2m1_encode_array(_p(x), x.size, _p(out))
    return out


def nvfp4_blocks(x) -> tuple[np.ndarray, np.ndarray]:
    """NVFP4 coding of the blocks along the last axis of x (length <= 16):
    returns (E2M1 codes shaped like x, UE4M3 scales shaped x.shape[:-1])."""
    x = _c(x, np.float32)
    n = x.shape[-1]
    assert 1 <= n <= 16
    codes = np.empty(x.shape, np.uint8)
    scales = np.empty(x.shape[:-1], np.uint8)
    lib().vo_nvfp4_block_array(_p(x), x.size // n, n, _p(codes), _p(scales))
    return codes, scales


def expcast_bytes(A, s, cb) -> np.ndarray:
    A, s, cb = np.broadcast_arrays(_c(A, np.float32), _c(s, np.float32), _c(cb, np.float32))
    A, s, cb = _c(A, np.float32), _c(s, np.float32), _c(cb, np.float32)
    out = np.empty(A.shape, np.uint8)
    lib().vo_expcast_array(_p(A), _p(s), _p(cb), A.size, _p(out))
    return out


def kappa(d: int) -> float:
    """fp32 rounding of 8*log2(e)/sqrt(d): the score scale in byte units."""
    return float(np.float32(8.0 / (math.log(2.0) * math.sqrt(d))))


# --------------------------------------------------------------- V-Smooth prep
def kmeans(v_bits: np.ndarray, C: int, iters: int):
    v = _c(v_bits, np.uint16)
    n, d = v.shape
    labels = np.empty(n, np.int32)
    cent = np.empty((C, d), np.float64)
    lib().vo_kmeans(_p(v), n, d, C, iters, _p(labels), _p(cent))
    return labels, cent


def stable_perm(labels: np.ndarray, C: int) -> np.ndarray:
    lab = _c(labels, np.int32)
    perm = np.empty(lab.shape[0], np.int32)
    lib().vo_stable_perm(_p(lab), lab.shape[0], C, _p(perm))
    return perm


def quant_q(q_bits: np.ndarray):
    q = _c(q_bits, np.uint16)
    n, d = q.shape
    qhat = np.empty((n, d), np.uint8)
    sq = np.empty(n, np.float32)
    lib().vo_quant_q(_p(q), n, d, _p(qhat), _p(sq))
    return qhat, sq


def quant_k(k_bits: np.ndarray, perm: np.ndarray, bk: int):
    k = _c(k_bits, np.uint16)
    n, d = k.shape
    T = -(-n // bk)
    khat = np.empty((T * bk, d), np.uint8)
    ksc = np.empty(T, np.float32)
    lib().vo_quant_k(_p(k), n, d, bk, _p(_c(perm, np.int32)), _p(khat), _p(ksc))
    return khat, ksc


def smooth_v(v_bits: np.ndarray, perm: np.ndarray, bk: int, smooth: bool = True):
    v = _c(v_bits, np.uint16)
    n, d = v.shape
    T = -(-n // bk)
    vhat = np.empty((T * bk, d), np.uint8)
    vmu = np.empty((T, d), np.float32)
    vsc = np.empty(d, np.float32)
    lib().vo_smooth_v(_p(v), n, d, bk, _p(_c(perm, np.int32)), int(smooth), _p(vhat), _p(vmu), _p(vsc))
    return vhat, vmu, vsc


def smooth_v_nvfp4(v_bits: np.ndarray, perm: np.ndarray, bk: int, smooth: bool = True):
    """4-bit residual: E2M1 codes vq [T*bk, d], UE4M3 block scales vgs
    [T, bk/16, d], block means vmu [T, d], channel scales vsc [d]."""
    v = _c(v_bits, np.uint16)
    n, d = v.shape
    T = -(-n // bk)
    vq = np.empty((T * bk, d), np.uint8)
    vgs = np.empty((T, bk // 16, d), np.uint8)
    vmu = np.empty((T, d), np.float32)
    vsc = np.empty(d, np.float32)
    lib().vo_smooth_v_nvfp4(_p(v), n, d, bk, _p(_c(perm, np.int32)), int(smooth), _p(vq), _p(vgs), _p(vmu),
                            _p(vsc))
    return vq, vgs, vmu, vsc


def nvfp4_v_values(vq: np.ndarray, vgs: np.ndarray) -> np.ndarray:
    """Residual values in channel-scale units: value(block scale) * value(code)."""
    T, G, d = vgs.shape
    sv = np.repeat(e4m3_value(vgs), 16, axis=1).reshape(T * G * 16, d)
    return sv * e2m1_value(vq)


def prep_head(k_bits, v_bits, *, C: int, iters: int, bk: int, smooth: bool = True, resid_fmt: int = 0):
    """The whole V-Smooth prep of one head, step by step (resid_fmt 1: the
    4-bit residual, whose outputs add vq and vgs in place of vhat)."""
    n = v_bits.shape[0]
    if smooth:
        labels, cent = kmeans(v_bits, C, iters)
        perm = stable_perm(labels, C)
    else:
        labels, cent = np.zeros(n, np.int32), None
        perm = np.arange(n, dtype=np.int32)
    khat, ksc = quant_k(k_bits, perm, bk)
    if resid_fmt == 1:
        vq, vgs, vmu, vsc = smooth_v_nvfp4(v_bits, perm, bk, smooth)
        return dict(labels=labels, centroids=cent, perm=perm, khat=khat, ksc=ksc, vq=vq, vgs=vgs, vmu=vmu,
                    vsc=vsc)
    vhat, vmu, vsc = smooth_v(v_bits, perm, bk, smooth)
    return dict(labels=labels, centroids=cent, perm=perm, khat=khat, ksc=ksc, vhat=vhat, vmu=vmu, vsc=vsc)


# ------------------------------------------------------------------ attention
def _chunks(nrows: int, parts: int):
    step = max(1, -(-nrows // parts))
    return [(a, min(nrows, a + step)) for a in range(0, nrows, step)]


def attn_emul(qv, sq, kv, ksc, rv, vmu, vsc, *, n: int, bk: int, beta: int, exact: bool = False,
              pfmt: int = 0, rowmask=None, kappa_value: float | None = None, threads: int | None = None):
    """Replay of the attention forward over the given query rows (values);
    pfmt 1 re-codes each 16-key block of P to NVFP4 (the 4-bit path);
    rowmask [nrows, T] (0 = drop the key tile for that row) is a block-sparse
    mask."""
    qv, sq = _c(qv, np.float64), _c(sq, np.float32)
    kv, ksc, rv = _c(kv, np.float64), _c(ksc, np.float32), _c(rv, np.float64)
    vmu, vsc = _c(vmu, np.float32), _c(vsc, np.float32)
    nrows, d = qv.shape
    kap = kappa(d) if kappa_value is None else kappa_value
    if exact and kappa_value is None:
        kap = 8.0 / (math.log(2.0) * math.sqrt(d))
    out = np.empty((nrows, d), np.float64)
    M = np.empty(nrows, np.float64)
    l = np.empty(nrows, np.float64)
    T = -(-n // bk)
    if rowmask is not None:
        rowmask = _c(rowmask, np.uint8)
        assert rowmask.shape == (nrows, T)
    L = lib()

    def run(a, b):
        if b <= a:
            return
        rm = None if rowmask is None else _p(rowmask[a:b])
        L.vo_attn_emul(_p(qv[a:b]), _p(sq[a:b]), b - a, _p(kv), _p(ksc), _p(rv), _p(vmu), _p(vsc), n, d, bk,
                       kap, int(beta), int(exact), int(pfmt), rm, _p(out[a:b]), _p(M[a:b]), _p(l[a:b]))

    threads = threads or os.cpu_count() or 1
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda ab: run(*ab), _chunks(nrows, threads)))
    return out, M, l


def attn_exact(q_bits, k_bits, v_bits, rows, threads: int | None = None) -> np.ndarray:
    q, k, v = _c(q_bits, np.uint16), _c(k_bits, np.uint16), _c(v_bits, np.uint16)
    rows = _c(rows, np.int32)
    n, d = k.shape
    out = np.empty((rows.shape[0], d), np.float64)
    L = lib()

    def run(a, b):
        if b > a:
            L.vo_attn_exact(_p(q), _p(k), _p(v), _p(rows[a:b]), b - a, n, d, _p(out[a:b]))

    threads = threads or os.cpu_count() or 1
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda ab: run(*ab), _chunks(rows.shape[0], threads)))
    return out


def forward_head(q_bits, k_bits, v_bits, rows, *, C: int, iters: int, bk: int, beta: int,
                 smooth: bool = True, resid_fmt: int = 0, prep=None, tile_mask=None, bm: int = 128,
                 threads: int | None = None):
    """V-Smooth prep plus the quantised attention replay for selected rows of
    one head (resid_fmt 1: 4-bit residual and NVFP4 P in the PV product)."""
    n, d = k_bits.shape
    if prep is None:
        prep = prep_head(k_bits, v_bits, C=C, iters=iters, bk=bk, smooth=smooth, resid_fmt=resid_fmt)
    rows = np.asarray(rows, dtype=np.int64)
    qhat, sq = quant_q(np.asarray(q_bits)[rows])
    rv = nvfp4_v_values(prep["vq"], prep["vgs"]) if resid_fmt == 1 else e4m3_value(prep["vhat"])
    # a block-sparse mask [Tq, T] over (query tile of bm rows, key tile), per row
    rowmask = None if tile_mask is None else np.asarray(tile_mask, np.uint8)[rows // bm]
    out, M, l = attn_emul(e4m3_value(qhat), sq, e4m3_value(prep["khat"]), prep["ksc"], rv, prep["vmu"],
                          prep["vsc"], n=n, bk=bk, beta=beta, pfmt=resid_fmt, rowmask=rowmask, threads=threads)
    return dict(prep=prep, qhat=qhat, sq=sq, out=out, M=M, l=l)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 -> bf16 (both round-to-nearest-even), returned as float32 values."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)
