"""Every source, test, profile or fixture file named in backticks by the repository's
top-level documents exists (a renamed or removed file shows up here)."""

import os
import re

import pytest

from conftest import ROOT

SEARCH = ("", "tests", "tests/golden", "oracle", "profiles", "include", "structured_sparse_attention_b200",
          "structured_sparse_attention_b200/csrc")


@pytest.mark.parametrize("doc", ["DESIGN.md", "README.md"])
def test_named_files_exist(doc):
    text = open(os.path.join(ROOT, doc)).read()
    refs = set(re.findall(r"`([\w./-]+\.(?:py|cu|cuh|h|c|json|md))`", text))
    assert refs
    missing = []
    for ref in sorted(refs):
        names = [ref, os.path.join("structured_sparse_attention_b200", ref)]
        if not any(os.path.exists(os.path.join(ROOT, d, n)) for d in SEARCH for n in names):
            missing.append(ref)
    assert not missing, f"{doc}: named files that do not exist: {missing}"
