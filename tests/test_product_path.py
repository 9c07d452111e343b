"""The product path has no CPU fallback and never reaches the oracle: the
package's modules import nothing from oracle/, and every compute entry of
the binding rejects host tensors instead of computing on the CPU."""
import ast
import os

import pytest
import torch

from w8a8_smoothquant_int8_02_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "w8a8_smoothquant_int8_02_b200")


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom):
            yield node.module or ""


def test_package_never_imports_the_oracle():
    for name in os.listdir(PKG):
        if name.endswith(".py"):
            for mod in _imports(os.path.join(PKG, name)):
                assert not mod.split(".")[0] == "oracle", (name, mod)
    for name in os.listdir(os.path.join(PKG, "csrc")):
        text = open(os.path.join(PKG, "csrc", name)).read()
        assert "sq_oracle" not in text and "sqo_" not in text, name


def _host(shape, dtype):
    return torch.zeros(shape, dtype=dtype)


@pytest.mark.parametrize("call", [
    lambda: ops.quantize_act(_host((4, 64), torch.bfloat16), None, "i8"),
    lambda: ops.quantize_act_tensor(_host((4, 64), torch.bfloat16), None, "e4m3"),
    lambda: ops.quantize_weight(_host((64, 32), torch.bfloat16), None, "i8"),
    lambda: ops.calibrate_amax(_host((4, 64), torch.bfloat16), "column"),
    lambda: ops.fold_smoothing(_host(64, torch.float32), _host(64, torch.float32)),
    lambda: ops.gemm_w8a8(_host((4, 64), torch.int8), _host(4, torch.float32),
                          _host((32, 64), torch.int8), _host(32, torch.float32)),
    lambda: ops.gemm_fp8(_host((4, 64), torch.uint8), _host(4, torch.float32),
                         _host((32, 64), torch.uint8), _host(32, torch.float32)),
    lambda: ops.linear(_host((4, 64), torch.bfloat16), None, _host((32, 64), torch.int8),
                       _host(32, torch.float32)),
])
def test_host_tensors_are_rejected(call):
    with pytest.raises(ValueError):
        call()


def test_non_contiguous_tensors_are_rejected():
    x = torch.zeros((64, 4), dtype=torch.bfloat16).t()
    assert not x.is_contiguous()
    with pytest.raises(ValueError):
        ops._cuda(x)


def test_missing_library_raises(monkeypatch, tmp_path):
    """Without libsq.so the binding raises instead of computing anything."""
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops._build, "LIB", str(tmp_path / "libsq.so"))
    with pytest.raises(RuntimeError, match="libsq.so not found"):
        ops.load(build_if_needed=False)
