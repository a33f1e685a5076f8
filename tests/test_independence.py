"""The oracle and the CUDA path share no code (CPU only).

The oracle is test infrastructure: the package ``linear_attention_positive_b200`` (the Python
binding and the seeded input generators) never imports it, and the oracle never imports the
package. Only the input generators serve both sides, and they hold none of the method's
arithmetic: no exponential, feature map, prefix sum or feature draw. The CUDA sources do not
include anything from the oracle's folder either.
"""

import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "linear_attention_positive_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _py_files(top):
    for dirpath, _, names in os.walk(top):
        for n in names:
            if n.endswith(".py"):
                yield os.path.join(dirpath, n)


def _imported_modules(path):
    tree = ast.parse(open(path).read(), path)
    out = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out.update(a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            if node.level == 0 and node.module:
                out.add(node.module)
    return out


def test_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        mods = _imported_modules(path)
        assert not any(m == "oracle" or m.startswith("oracle.") for m in mods), path


def test_oracle_never_imports_the_package():
    for path in _py_files(ORACLE):
        mods = _imported_modules(path)
        assert not any(m.startswith("linear_attention_positive_b200") for m in mods), path


def test_cuda_sources_do_not_reach_into_the_oracle():
    csrc = os.path.join(PKG, "csrc")
    for n in os.listdir(csrc):
        text = open(os.path.join(csrc, n), errors="replace").read()
        assert "oracle" not in text.lower(), n


def test_input_generators_hold_no_method_arithmetic():
    path = os.path.join(PKG, "inputs.py")
    tree = ast.parse(open(path).read(), path)
    called = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Call):
            f = node.func
            called.add(f.attr if isinstance(f, ast.Attribute) else getattr(f, "id", ""))
    # A library QR may rotate the synthetic inputs (input structure); the feature map, the causal
    # prefix sums and the feature draw itself must not appear.
    forbidden = {"exp", "exp2", "expm1", "log", "cumsum", "tril", "triu", "einsum"}
    assert not (called & forbidden), called & forbidden
    names = {n.id for n in ast.walk(tree) if isinstance(n, ast.Name)}
    assert not (names & {"phi", "draw_W", "philox4x64_10", "gaussians"})
