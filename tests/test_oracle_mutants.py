"""The pins catch plausible mistakes in the oracle.

Each mutant below is a copy of oracle/vc_oracle.c with one planted mistake: a
wrong exponent, bias or tie rule, a dropped term or factor, a wrong sign, a
transposed index, an extra or missing step.  The copy is built in a temporary
folder and the oracle's pin tests run against it (VC_ORACLE_SRC).  Every
mutant must make at least one pin fail.  The mistakes are planted on the CPU,
in the oracle only.

Mutants that do not change any result are left out.  One example: leaving the
scores unrounded before the ExpCast call, whose arguments round them to fp32
anyway.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "vc_oracle.c")
PINS = ["tests/test_oracle_codec.py", "tests/test_oracle_nvfp4.py", "tests/test_oracle_prep.py",
        "tests/test_oracle_attention.py", "tests/test_oracle_sparse.py"]

# (name, text in vc_oracle.c, planted replacement); the first occurrence is replaced
MUTANTS = [
    # E4M3 and E2M1 codecs
    ("e4m3_subnormal_exponent", "v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    ("e4m3_bias", "v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3_ties_down", "code = (lo & 1) ? hi : lo;", "code = lo;"),
    ("e2m1_exponent", "ldexp(1.0 + 0.5 * (double)m, e - 1)", "ldexp(1.0 + 0.5 * (double)m, e)"),
    ("e2m1_ties_up", "code = (lo & 1) ? lo + 1 : lo;", "code = lo + 1;"),
    ("nvfp4_scale_over_4", "vo_e4m3_encode(amax / 6.0f)", "vo_e4m3_encode(amax / 4.0f)"),
    ("nvfp4_exact_division", "codes[i] = vo_e2m1_encode(x[i] * r);", "codes[i] = vo_e2m1_encode(x[i] / sv);"),
    # ExpCast
    ("expcast_ties_up", "if (fr > 0.5)\n        n = fl + 1.0;", "if (fr >= 0.5)\n        n = fl + 1.0;"),
    ("expcast_clamp_at_1", "if (!(t > 0.0)) return 0;", "if (!(t > 1.0)) return 0;"),
    ("expcast_two_roundings", "double d = (double)A * (double)s;", "double d = (double)(A * s);"),
    # k-means and the regroup
    ("kmeans_init_stride", "int64_t src = ((int64_t)k * n) / C;", "int64_t src = ((int64_t)k * (n - 1)) / C;"),
    ("kmeans_ties_high", "if (dist[k] < dist[best]) best = k;", "if (dist[k] <= dist[best]) best = k;"),
    ("kmeans_mean_divisor", "sums[(size_t)k * d + c] / (double)cnt[k];",
     "sums[(size_t)k * d + c] / (double)(cnt[k] + 1);"),
    ("kmeans_l1_distance", "dist[k] += diff * diff;", "dist[k] += fabs(diff);"),
    ("kmeans_extra_update", "if (it == iters - 1) break;", "if (it == iters) break;"),
    ("regroup_reversed", "for (int j = 0; j < n; ++j) perm[start[labels[j]]++] = j;",
     "for (int j = n - 1; j >= 0; --j) perm[start[labels[j]]++] = j;"),
    # quantisers and V-Smooth
    ("qk_scale_over_240", "*scale = amax / 448.0f;", "*scale = amax / 240.0f;"),
    ("block_mean_over_bk", "vmu[(size_t)b * d + c] = smooth ? (float)(s / (double)valid) : 0.0f;",
     "vmu[(size_t)b * d + c] = smooth ? (float)(s / (double)bk) : 0.0f;"),
    ("residual_keeps_mean",
     "                float res = bf16_to_float(v[(size_t)perm[b * bk + r] * d + c]) - vmu[(size_t)b * d + c];\n"
     "                vhat[",
     "                float res = bf16_to_float(v[(size_t)perm[b * bk + r] * d + c]);\n"
     "                vhat["),
    ("nvfp4_channel_scale_448", "vsc[c] = amax[c] > 0.0f ? amax[c] / 2688.0f : 1.0f;",
     "vsc[c] = amax[c] > 0.0f ? amax[c] / 448.0f : 1.0f;"),
    ("nvfp4_block_reversed", "x[i] = y[(size_t)(16 * g + i) * d + c];", "x[i] = y[(size_t)(16 * g + 15 - i) * d + c];"),
    # the attention replay
    ("replay_A_without_q_scale", "A = (double)(aq32 * ksc[b]);", "A = (double)(kappa32 * ksc[b]);"),
    ("replay_M_floor", "double Mc = ceil(x / 8.0);", "double Mc = floor(x / 8.0);"),
    ("replay_M_starts_at_zero", "double Mnew = first ? Mc : (Mc > M ? Mc : M);", "double Mnew = Mc > M ? Mc : M;"),
    ("replay_cb_sign", "double cb = 56.0 + (double)beta - 8.0 * M;", "double cb = 56.0 + (double)beta + 8.0 * M;"),
    ("replay_mean_not_rescaled", "                    omean[c] *= f;\n", ""),
    ("replay_l_not_rescaled", "                l *= f;\n", ""),
    ("replay_restore_without_l", "omean[c] += lb * (double)vmu[(size_t)b * d + c];",
     "omean[c] += (double)vmu[(size_t)b * d + c];"),
    ("replay_p4_without_scale", "p[16 * g + i] = vo_e4m3_value(sc16) * vo_e2m1_value(codes[i]);",
     "p[16 * g + i] = vo_e2m1_value(codes[i]);"),
    ("replay_mask_transposed", "if (rowmask && !rowmask[(size_t)i * T + b]) continue;",
     "if (rowmask && !rowmask[(size_t)b * nrows + i]) continue;"),
    ("replay_output_without_vsc", "((double)vsc[c] * ores[c] + omean[c]) / l", "(ores[c] + omean[c]) / l"),
    ("exact_scale_over_d", "double scale = 1.0 / sqrt((double)d);", "double scale = 1.0 / (double)d;"),
]


def _run_mutant(base, mutant):
    name, old, new = mutant
    src = open(SRC, encoding="utf-8").read()
    if old not in src:
        return name, "missing", f"the text to mutate is no longer in vc_oracle.c: {old!r}"
    folder = os.path.join(base, name)
    os.makedirs(os.path.join(folder, "_build"))
    path = os.path.join(folder, "vc_oracle.c")
    with open(path, "w", encoding="utf-8") as f:
        f.write(src.replace(old, new, 1))
    so = os.path.join(folder, "_build", "libvcoracle.so")
    r = subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                        "-fno-fast-math", "-o", so, path, "-lm"], capture_output=True, text=True)
    if r.returncode:
        return name, "build", r.stderr[-400:]
    env = dict(os.environ, VC_ORACLE_SRC=path, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=900)
    failed = [line for line in r.stdout.splitlines() if line.startswith("FAILED")]
    return name, r.returncode, failed[0] if failed else r.stdout[-400:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    base = str(tmp_path_factory.mktemp("mutants"))
    workers = max(1, min(8, os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as ex:
        return {name: (rc, info) for name, rc, info in ex.map(lambda m: _run_mutant(base, m), MUTANTS)}


def test_unmutated_source_passes_the_pins(tmp_path):
    """The harness itself: the unchanged source, built the same way, passes."""
    name, rc, info = _run_mutant(str(tmp_path), ("unchanged", "#include", "#include"))
    assert rc == 0, info


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_the_mutant(outcomes, name):
    rc, info = outcomes[name]
    # pytest exits 1 when a test failed; anything else (a build or collection
    # error, a missing mutation site) is not a catch
    assert rc == 1 and info.startswith("FAILED"), (name, rc, info)
