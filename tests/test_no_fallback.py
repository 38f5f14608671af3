"""The product path has no CPU fallback: without librq.so the binding does not
import, and with it every compute call refuses host tensors instead of
computing anything on the CPU."""

import importlib.util
import os
import shutil

import pytest
import torch

from conftest import ROOT

PKG = os.path.join(ROOT, "rotation_w4a4_quantization_b200")


def test_binding_without_the_library_raises(tmp_path):
    # a copy of the binding next to no librq.so
    shutil.copy(os.path.join(PKG, "rq.py"), tmp_path / "rq.py")
    spec = importlib.util.spec_from_file_location("rq_without_lib", tmp_path / "rq.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="librq.so not built"):
        spec.loader.exec_module(mod)


def test_host_tensors_are_refused():
    rq = pytest.importorskip("rotation_w4a4_quantization_b200.rq")
    x = torch.zeros((4, 512), dtype=torch.bfloat16)
    s = torch.ones(512, dtype=torch.int8)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        rq.rotate_quantize(x, s)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        rq.prepare_weights(x, s)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        rq.rotate_f32(x, s)
    codes = torch.zeros((4, 256), dtype=torch.uint8)
    scales = torch.ones(4, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        rq.w4a4_gemm((codes, scales, None), (codes, scales, None))
    kv = torch.zeros((1, 1, 4, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        rq.kv_rotate_quantize(kv, torch.ones(128, dtype=torch.int8))


def test_product_modules_do_not_import_the_oracle():
    for name in os.listdir(PKG):
        if name.endswith(".py"):
            with open(os.path.join(PKG, name)) as f:
                text = f.read()
            assert "import oracle" not in text and "from oracle" not in text, name
