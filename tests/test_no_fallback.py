"""The product path has no CPU fallback and never touches the oracle: the
package's sources import nothing from oracle/, and the binding refuses host
tensors (it only marshals device pointers into the CUDA library) instead of
computing anything itself."""
import ast
import os

import pytest
import torch

from block_sparse_kv_spattn_b200 import spattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_kv_spattn_b200")


def _imports(path):
    tree = ast.parse(open(path, encoding="utf-8").read(), filename=path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom) and node.module:
            yield node.module


def test_package_never_imports_the_oracle():
    found = []
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                p = os.path.join(dirpath, f)
                found += [(p, m) for m in _imports(p) if m == "oracle" or m.startswith("oracle.")]
    assert not found, found


def test_package_sources_do_not_name_the_oracle_directory():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".map")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle/" not in text and "import oracle" not in text, f


def test_binding_refuses_host_tensors():
    q = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16)
    kc = torch.zeros(4, 2, 64, 128, dtype=torch.bfloat16)
    bt = torch.zeros(1, 4, dtype=torch.int32)
    sl = torch.full((1,), 256, dtype=torch.int32)
    sel = torch.zeros(1, 2, 4, dtype=torch.int32)
    cnt = torch.zeros(1, 2, dtype=torch.int32)
    out = torch.zeros(1, 1, 8, 128)
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    if not os.path.exists(spattn.LIB_PATH):
        pytest.skip("library not built")
    with pytest.raises(ValueError, match="CUDA tensors"):
        spattn.decode_selected(q, kc, kc, None, None, bt, sl, sel, cnt, out, ws, spattn.Params(top_k=1))
