"""The product path has no fallback (CPU): a missing CUDA library makes the
binding raise, and no module of the package imports the oracle."""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_diffusion_attention_b200")


def test_missing_library_raises():
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from block_diffusion_attention_b200 import flashblock as f\n"
        "f.LIB_PATH = '/nonexistent/libflashblock.so'\n"
        "f._lib = None\n"
        "try:\n"
        "    f.load()\n"
        "except FileNotFoundError as e:\n"
        "    print('raised:', e)\n"
        "else:\n"
        "    print('loaded')\n" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.startswith("raised:") and "build" in out.stdout


def test_product_modules_do_not_import_the_oracle():
    for name in sorted(os.listdir(PKG)):
        if not name.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(PKG, name)).read(), filename=name)
        for node in ast.walk(tree):
            mods = []
            if isinstance(node, ast.Import):
                mods = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                mods = [node.module or ""]
            for m in mods:
                assert not m.split(".")[0] == "oracle", f"{name} imports {m}"
