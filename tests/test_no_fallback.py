"""The product path has no CPU fallback: without libcsa.so every entry point
of the binding raises, and no module of the package imports the oracle."""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "compressed_sparse_attention_compressor_b200")


def test_entry_points_raise_without_the_library():
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from compressed_sparse_attention_compressor_b200 import csa\n"
        "csa.LIB_PATH = '/nonexistent/libcsa.so'\n"
        "failed = []\n"
        "for call in (lambda: csa.csa_topk_workspace_size(1),\n"
        "             lambda: csa.csa_workspace_size(csa.params(4, 512, 128, 64, 64, 64, 128, 128), 1, 1024),\n"
        "             lambda: csa.load()):\n"
        "    try:\n"
        "        call()\n"
        "    except ImportError as e:\n"
        "        failed.append('missing' in str(e))\n"
        "print(failed)\n" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "[True, True, True]", out.stdout + out.stderr


def test_package_never_imports_the_oracle():
    for fn in sorted(os.listdir(PKG)):
        if not fn.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(PKG, fn)).read())
        for node in ast.walk(tree):
            names = []
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            assert not any(n.split(".")[0] == "oracle" for n in names), f"{fn} imports the oracle"
