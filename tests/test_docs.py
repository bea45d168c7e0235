"""The design notes and README name files of this repository in backticks; every one
must exist, so that the documents cannot drift from the code they describe."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SEARCH = ["", "long_context_attention_fwd_b200", os.path.join("long_context_attention_fwd_b200", "csrc"),
          "tests", "oracle", "profiles"]


@pytest.mark.parametrize("doc", ["DESIGN.md", "README.md"])
def test_named_files_exist(doc):
    text = open(os.path.join(ROOT, doc), encoding="utf-8").read()
    names = set(re.findall(r"`([A-Za-z0-9_./-]+\.(?:py|cu|cuh|h|c|md|json))`", text))
    assert names, "no file names found"
    missing = [n for n in sorted(names)
               if not any(os.path.exists(os.path.join(ROOT, d, n)) for d in SEARCH)]
    assert not missing, missing
