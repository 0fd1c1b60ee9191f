"""The CUDA path and the CPU oracle are separate: the library never imports,
links or calls the oracle; the oracle never imports the library; the seeded
input generators import neither and hold no arithmetic of the method; and the
binding has no fallback: without libsvdq.so every call raises."""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "w4a4_rank_corrected_svdq_b200")


def _imports(path):
    tree = ast.parse(open(path).read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _py_files(d):
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith(".py")]


def test_library_never_imports_the_oracle():
    for f in _py_files(PKG):
        assert "oracle" not in _imports(f), f
    for f in os.listdir(os.path.join(PKG, "csrc")):
        src = open(os.path.join(PKG, "csrc", f)).read()
        assert "oracle/" not in src and "oracle." not in src, f


def test_oracle_never_imports_the_library():
    for f in _py_files(os.path.join(ROOT, "oracle")):
        assert "w4a4_rank_corrected_svdq_b200" not in _imports(f), f


def test_input_generators_import_neither_side():
    names = _imports(os.path.join(ROOT, "workloads.py"))
    assert "oracle" not in names and "w4a4_rank_corrected_svdq_b200" not in names
    src = open(os.path.join(ROOT, "workloads.py")).read()
    for word in ("linalg.svd", "quantize", "e2m1", "e4m3", "gelu", "rms", "residual"):
        assert word not in src.lower(), word


def test_binding_raises_without_the_library():
    code = ("import sys; sys.path.insert(0, %r)\n"
            "import w4a4_rank_corrected_svdq_b200._lib as L\n"
            "L.LIB_PATH = '/nonexistent/libsvdq.so'\n"
            "try:\n"
            "    L.svdq_weight_sizes(256, 512, 32)\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n"
            "else:\n"
            "    print('no error')\n") % ROOT
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120).stdout
    assert out.startswith("raised:") and "not built" in out, out
