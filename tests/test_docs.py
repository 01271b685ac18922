"""The design notes and the README name files that exist: every backticked
repository path in them resolves (bare names are looked up in the package,
its CUDA sources, the tests, the oracle, the header and profile folders)."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SEARCH = ["", "bit_fp8_attention_smooth_b200", "bit_fp8_attention_smooth_b200/csrc", "tests", "oracle", "include",
          "profiles"]


@pytest.mark.parametrize("doc", ["DESIGN.md", "README.md"])
def test_named_files_exist(doc):
    text = open(os.path.join(ROOT, doc), encoding="utf-8").read()
    names = set(re.findall(r"`([A-Za-z0-9_./\-]+\.(?:py|cu|cuh|h|c|md|txt))(?:::[A-Za-z0-9_]+)?`", text))
    assert names
    missing = [n for n in sorted(names) if not any(os.path.exists(os.path.join(ROOT, d, n)) for d in SEARCH)]
    assert not missing, missing
