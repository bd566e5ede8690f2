"""The oracle is plain C11 that compiles without warnings under -Wall -Wextra
-Wpedantic, so a reader can check it against the pages without compiler noise
hiding a real mistake (test infrastructure; it shares nothing with the CUDA
path)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_compiles_cleanly():
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Wpedantic", "-Werror", "-O2", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "oracle"), os.path.join(ROOT, "oracle", "oracle.c")],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr


def test_oracle_shares_nothing_with_the_cuda_path():
    # the oracle includes only the C library and its own header; the CUDA
    # sources include nothing of the oracle; the package imports nothing of it
    import re
    for f in ("oracle.c", "oracle.h"):
        text = open(os.path.join(ROOT, "oracle", f)).read()
        for inc in re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', text):
            assert inc == "oracle.h" or "/" not in inc and not inc.startswith("fa"), (f, inc)
    for f in os.listdir(os.path.join(ROOT, "flash_fwd_b200", "csrc")):
        text = open(os.path.join(ROOT, "flash_fwd_b200", "csrc", f), errors="ignore").read()
        for inc in re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', text):
            assert "oracle" not in inc, (f, inc)
    for f in ("__init__.py", "build.py", "accounting.py", "dist.py", "inputs.py"):
        text = open(os.path.join(ROOT, "flash_fwd_b200", f)).read()
        assert "import oracle" not in text and "from oracle" not in text, f
