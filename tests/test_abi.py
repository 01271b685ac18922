"""The C ABI library builds for sm_100a, loads, and exports every function that
include/*.h declares (no compute calls: this runs without a GPU)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(vc_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def libpath():
    from bit_fp8_attention_smooth_b200 import build

    return build.build()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("vc_smooth_prepare", "vc_attn_fwd", "vc_attention", "vc_workspace_bytes", "vc_prep_buffer_bytes",
              "vc_check", "vc_status_string", "vc_abi_version", "vc_e4m3_encode", "vc_expcast_bytes",
              "vc_quantize_q"):
        assert n in names


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing


def test_library_loads_and_answers_host_queries(libpath):
    L = ctypes.CDLL(libpath)
    assert L.vc_abi_version() == 2
    L.vc_status_string.restype = ctypes.c_char_p
    assert L.vc_status_string(0) == b"ok"
    import bit_fp8_attention_smooth_b200 as vc

    shape = (1, 40, 32768, 128)
    params = vc.Params(C=64, iters=10, block=128)
    sizes = vc.prep_sizes(shape, params)
    assert sizes[2] == 40 * 32768 * 128 and sizes[4] == 40 * 128 * 32768 and sizes[7] == 0
    # the 4-bit residual: two codes a byte, one UE4M3 scale per 16 tokens of a channel
    p4 = vc.Params(C=64, iters=10, block=128, resid_fmt=1)
    s4 = vc.prep_sizes(shape, p4)
    assert s4[4] == 40 * 128 * 32768 // 2 and s4[7] == 40 * 256 * 128 * 8
    with pytest.raises(vc.VcError) as e:  # block 64 has no 4-bit path
        vc.prep_sizes(shape, vc.Params(C=64, iters=10, block=64, resid_fmt=1))
    assert e.value.status == vc.VC_ERR_UNSUPPORTED
    with pytest.raises(vc.VcError) as e:
        vc.prep_sizes(shape, vc.Params(C=64, iters=10, block=128, resid_fmt=2))
    assert e.value.status == vc.VC_ERR_INVALID_ARG
    assert vc.workspace_bytes(shape, params) >= 40 * 32768 * 128
    with pytest.raises(vc.VcError) as e:
        vc.workspace_bytes((1, 1, 100, 96), params)
    assert e.value.status == vc.VC_ERR_UNSUPPORTED


def test_oracle_builds_independently():
    import oracle

    path = oracle.build()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    assert "vo_attn_emul" in out and "vc_" not in out


def test_argument_checks_run_before_any_device_call(libpath):
    """Host-side validation of the entry points answers without a GPU: the
    checks come before any CUDA call (the pointers below are never used)."""
    import bit_fp8_attention_smooth_b200 as vc

    L = vc.lib()
    fake = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced
    shape = vc._Shape(1, 2, 1000, 128)
    prep = vc._Prep(*([fake.value] * 8))
    dense = vc.Params(C=8, iters=2, block=128)

    def masked(params, mask):
        return L.vc_attn_fwd_masked(fake, ctypes.byref(prep), ctypes.byref(shape), ctypes.byref(params.c()), mask,
                                    fake, fake, ctypes.c_size_t(1 << 40), None)

    assert masked(dense, None) == vc.VC_ERR_INVALID_ARG  # a mask is required
    assert masked(vc.Params(C=8, iters=2, block=128, resid_fmt=1), fake) == vc.VC_ERR_UNSUPPORTED
    assert masked(vc.Params(C=8, iters=2, block=96), fake) == vc.VC_ERR_UNSUPPORTED
    assert masked(vc.Params(C=8, iters=2, block=128, smooth=3), fake) == vc.VC_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.vc_attn_fwd_masked(odd, ctypes.byref(prep), ctypes.byref(shape), ctypes.byref(dense.c()), fake, fake,
                                fake, ctypes.c_size_t(1 << 40), None) == vc.VC_ERR_INVALID_ARG
    # the 4-bit prep needs its block-scale buffer
    p4 = vc.Params(C=8, iters=2, block=128, resid_fmt=1)
    no_scales = vc._Prep(*([fake.value] * 7 + [None]))
    assert L.vc_attn_fwd(fake, ctypes.byref(no_scales), ctypes.byref(shape), ctypes.byref(p4.c()), fake, fake,
                         ctypes.c_size_t(1 << 40), None) == vc.VC_ERR_INVALID_ARG
    # the per-token Q quantiser: d, the token count and alignment, before the device
    assert L.vc_quantize_q(fake, fake, fake, 10, 96, None) == vc.VC_ERR_UNSUPPORTED
    assert L.vc_quantize_q(fake, fake, fake, -1, 128, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_quantize_q(odd, fake, fake, 10, 128, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_quantize_q(fake, odd, fake, 10, 128, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_quantize_q(fake, fake, ctypes.c_void_p((1 << 20) + 2), 10, 128, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_quantize_q(None, None, None, 0, 128, None) == vc.VC_OK  # nothing to do


def test_product_path_fails_loudly_without_the_library(monkeypatch, tmp_path):
    """No CPU fallback: with the library absent, the public calls raise."""
    import torch

    import bit_fp8_attention_smooth_b200 as vc

    monkeypatch.setattr(vc, "LIB_PATH", str(tmp_path / "libvcattn.so"))
    monkeypatch.setattr(vc, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        vc.lib()
    params = vc.Params(C=4, iters=2, block=64)
    # the workspace size comes from the library too
    with pytest.raises(RuntimeError, match="missing"):
        vc.alloc_workspace((1, 1, 128, 64), params, "cpu")
    # host tensors are refused, never computed on the CPU
    x = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises((RuntimeError, ValueError), match="missing|CUDA tensor"):
        vc.attention(x, x, x, params)


def test_package_never_loads_the_oracle():
    """The product path (binding and kernels) names no oracle module, file or
    symbol: the oracle is test infrastructure only."""
    pkg = os.path.join(ROOT, "bit_fp8_attention_smooth_b200")
    offenders = []
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                if re.search(r"import\s+oracle|from\s+oracle|vc_oracle|liboracle|\bvo_\w+\(", text):
                    offenders.append(f)
    assert not offenders, offenders


@pytest.mark.parametrize("shape", [(1, 40, 32768, 128), (2, 3, 777, 64), (1, 1, 1, 128), (1, 2, 300, 128)])
@pytest.mark.parametrize("block,resid_fmt", [(64, 0), (128, 0), (128, 1)])
def test_binding_layout_matches_the_library_sizes(libpath, shape, block, resid_fmt):
    """The binding checks buffers against its own table of prep shapes; the
    library sizes them with vc_prep_buffer_bytes.  Both must agree byte for
    byte, field by field, or a buffer the binding accepts could be too small."""
    import torch

    import bit_fp8_attention_smooth_b200 as vc

    params = vc.Params(C=min(16, shape[2]), iters=3, block=block, resid_fmt=resid_fmt)  # C <= N
    sizes = vc.prep_sizes(shape, params)
    layout = vc.prep_layout(shape, params)
    for i, name in enumerate(vc.PREP_FIELDS):
        want = sizes[i]
        if name not in layout:
            assert want == 0, name
            continue
        sh, dt = layout[name]
        n = 1
        for x in sh:
            n *= x
        assert n * torch.empty((), dtype=dt).element_size() == want, (name, sh, dt, want)


def test_shape_and_parameter_checks_of_every_entry_point(libpath):
    """Every entry point rejects a bad shape, parameter, pointer or workspace
    size on the host, before any CUDA call (the pointers are never used)."""
    import bit_fp8_attention_smooth_b200 as vc

    L = vc.lib()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    prep = vc._Prep(*([fake.value] * 8))
    big = ctypes.c_size_t(1 << 40)

    def sh(B=1, H=2, N=1000, d=128):
        return vc._Shape(B, H, N, d)

    def pr(**kw):
        base = dict(C=8, iters=2, block=128)
        base.update(kw)
        return vc.Params(**base).c()

    def prepare(shape, params, K=fake, V=fake, p=prep, ws=fake, nbytes=big):
        return L.vc_smooth_prepare(K, V, ctypes.byref(shape), ctypes.byref(params), ctypes.byref(p) if p else None,
                                   ws, nbytes, None)

    def attention(shape, params, O=fake, ws=fake, nbytes=big):
        return L.vc_attention(fake, fake, fake, ctypes.byref(shape), ctypes.byref(params), ctypes.byref(prep), O,
                              ws, nbytes, None)

    INV, UNS, WS = vc.VC_ERR_INVALID_ARG, vc.VC_ERR_UNSUPPORTED, vc.VC_ERR_WORKSPACE
    cases = [
        (sh(d=96), pr(), UNS), (sh(), pr(block=96), UNS), (sh(), pr(block=64, resid_fmt=1), UNS),
        (sh(N=0), pr(), INV), (sh(B=0), pr(), INV), (sh(N=(1 << 24) + 1), pr(), INV),
        (sh(B=256, H=257), pr(), INV),
        (sh(), pr(resid_fmt=2), INV), (sh(), pr(smooth=3), INV), (sh(), pr(smooth=-1), INV),
        (sh(), pr(beta=71), INV), (sh(), pr(beta=-1), INV), (sh(), pr(wait_limit_ns=-1), INV),
        (sh(), pr(C=0), INV), (sh(), pr(C=257), INV), (sh(N=7), pr(C=8), INV),
        (sh(), pr(iters=0), INV), (sh(), pr(iters=65), INV),
    ]
    for shape, params, want in cases:
        got = (prepare(shape, params), attention(shape, params))
        assert got == (want, want), (shape.B, shape.H, shape.N, shape.d, params.C, params.iters, params.block,
                                     params.beta, params.smooth, params.resid_fmt, got)
    ok_shape, ok = sh(), pr()
    assert prepare(ok_shape, ok, K=None) == INV
    assert prepare(ok_shape, ok, V=odd) == INV
    assert prepare(ok_shape, ok, p=None) == INV
    assert prepare(ok_shape, ok, p=vc._Prep(*([fake.value] * 4 + [odd.value] + [fake.value] * 3))) == INV
    assert prepare(ok_shape, ok, ws=odd) == INV
    assert prepare(ok_shape, ok, nbytes=ctypes.c_size_t(1024)) == WS
    assert attention(ok_shape, ok, O=None) == INV
    assert attention(ok_shape, ok, nbytes=ctypes.c_size_t(1024)) == WS
    # from host buffers: host pointers must be given
    assert L.vc_attention_host(None, fake, fake, fake, ctypes.byref(ok_shape), ctypes.byref(ok), 4, fake, fake,
                               fake, fake, ctypes.byref(prep), fake, big, None, None, None) == INV
    # allocation-free: a problem larger than the static scratch is refused up front
    huge = sh(H=8, N=32768)
    assert L.vc_attn_fwd_noalloc(fake, ctypes.byref(prep), ctypes.byref(huge), ctypes.byref(ok), fake,
                                 None) == WS
    assert L.vc_attn_fwd_noalloc(odd, ctypes.byref(prep), ctypes.byref(ok_shape), ctypes.byref(ok), fake,
                                 None) == INV
    assert L.vc_check(odd, None) == INV


def test_header_is_plain_c_and_a_c_program_links_the_library(libpath, tmp_path):
    """include/vc_attention.h compiles as strict C99 and as C++17, and a plain
    C program links libvcattn.so and answers the host queries (no torch, no
    Python): the boundary is usable from C."""
    inc = os.path.join(ROOT, "include")
    hdr = os.path.join(inc, "vc_attention.h")
    for cmd in (["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-x", "c", hdr],
                ["g++", "-std=c++17", "-Wall", "-Werror", "-fsyntax-only", "-x", "c++", hdr]):
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
    prog = tmp_path / "abi.c"
    prog.write_text(r"""
#include <stdio.h>
#include "vc_attention.h"
int main(void) {
    vc_shape s = {1, 40, 32768, 128};
    vc_params p = {64, 10, 128, 64, 1, 0, 0};
    size_t b[8], ws = 0;
    if (vc_abi_version() != VC_ABI_VERSION) return 1;
    if (vc_prep_buffer_bytes(&s, &p, b) != VC_OK || vc_workspace_bytes(&s, &p, &ws) != VC_OK) return 2;
    p.block = 96;
    if (vc_prep_buffer_bytes(&s, &p, b) != VC_ERR_UNSUPPORTED) return 3;
    printf("%zu %zu %s\n", b[2], ws, vc_status_string(VC_ERR_WORKSPACE));
    return 0;
}
""")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(libpath)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(prog), "-o", str(exe), "-L", libdir,
                        "-lvcattn", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    k_bytes, ws, msg = r.stdout.split(maxsplit=2)
    assert int(k_bytes) == 40 * 32768 * 128 and int(ws) > 0 and msg.strip()
