"""Repository checks that need no GPU: the profile summaries run committed files only, and
the oracle stays out of the product path (the package never imports it)."""
from __future__ import annotations

import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _tracked_exists(rel: str) -> bool:
    return os.path.exists(os.path.join(ROOT, rel))


def test_profile_commands_use_committed_files_only():
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        text = open(path, encoding="utf-8").read()
        assert "_work/" not in text, f"{path} names a scratch file"
        for rel in set(re.findall(r"\b((?:tests|adapter_matmul_b200|oracle)/[\w/]+\.py|bench\.py)\b", text)):
            assert _tracked_exists(rel), f"{path} runs {rel}, which is not in the repository"


def test_product_package_never_imports_the_oracle():
    pattern = re.compile(r"^\s*(?:import\s+oracle\b|from\s+oracle\b)", re.M)
    for path in glob.glob(os.path.join(ROOT, "adapter_matmul_b200", "**", "*.py"), recursive=True):
        assert not pattern.search(open(path, encoding="utf-8").read()), f"{path} imports the oracle"
    for path in glob.glob(os.path.join(ROOT, "adapter_matmul_b200", "csrc", "*")):
        assert "oracle" not in os.path.basename(path)
        text = open(path, encoding="utf-8").read()
        assert "sgmv_oracle" not in text and "liboracle" not in text, f"{path} refers to the oracle"
