"""The product path has no CPU fallback: the package never imports the
oracle, and the binding raises when the compiled library is missing instead
of computing anything another way."""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_quantized_lora_blockwise_b200")


def _imports(path):
    tree = ast.parse(open(path, encoding="utf-8").read(), path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            yield from (a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            yield node.module or ""


def test_package_never_imports_the_oracle():
    files = [os.path.join(dp, f) for dp, _, fs in os.walk(PKG) for f in fs if f.endswith(".py")]
    assert files
    for path in files:
        for mod in _imports(path):
            assert mod.split(".")[0] != "oracle", f"{os.path.relpath(path, ROOT)} imports {mod}"


def test_missing_library_raises():
    code = ("from bit_quantized_lora_blockwise_b200 import binding\n"
            "try:\n"
            "    binding.load('/nonexistent/libqlora.so')\n"
            "except OSError as e:\n"
            "    print('raised', 'libqlora.so not found' in str(e))\n")
    p = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == "raised True"
