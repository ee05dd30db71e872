"""The product path has no CPU fallback: without libq4.so every call raises, CPU tensors
are refused, and no module of the package imports the oracle."""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_missing_library_raises():
    code = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import int4_quantized_b200 as q4
q4.lib_path = "/nonexistent/libq4.so"
for f in (lambda: q4.payload_bytes(4, 8, 4),
          lambda: q4.qgemm_workspace_bytes(1, 64, 64, 4, 32),
          lambda: q4.gptq_prepare(np.eye(4))):
    try:
        f()
    except ImportError:
        continue
    raise SystemExit("no ImportError")
try:
    q4.qpack(torch.zeros(4, 8), 4, 8)   # a CPU tensor
except TypeError:
    pass
else:
    raise SystemExit("CPU tensor accepted")
print("ok")
"""
    r = subprocess.run([sys.executable, "-c", code, ROOT], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def test_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "int4_quantized_b200")
    for fn in sorted(os.listdir(pkg)):
        if not fn.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(pkg, fn)).read())
        for node in ast.walk(tree):
            names = []
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            assert not any(n == "oracle" or n.startswith("oracle.") for n in names), fn
