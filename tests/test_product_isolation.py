"""The product path never touches the oracle: importing the package, its
binding and the process ring loads no module of ``oracle`` (checked in a
fresh interpreter), and no product source names it."""

import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_product_imports_do_not_load_the_oracle():
    code = ("import sys\n"
            "import long_context_exact_attn_b200 as p\n"
            "from long_context_exact_attn_b200 import ops, ring, workloads\n"
            "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]\n"
            "print(','.join(bad))\n")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == ""


def test_product_sources_do_not_name_the_oracle():
    pkg = os.path.join(ROOT, "long_context_exact_attn_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, f
