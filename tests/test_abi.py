"""The C-ABI library loads, exports every symbol include/lf_decode.h
declares, and rejects bad arguments on the host before touching the GPU
(CPU only: no kernel is launched here)."""
import ctypes
import os
import re
import subprocess

import pytest

from attention_lf_decode_b200 import binding
from attention_lf_decode_b200 import build as lfbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    lfbuild.build()
    return binding.load_library()


def declared_functions():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"^\s*(?:LF_API\s+)?(?:int|const char\s*\*)\s+(lf_\w+)\s*\(", src, re.M)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(binding.EXPORTS) <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", lfbuild.LIB],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(\w+)$", out, re.M))
    for n in names:
        assert n in exported, n
        assert getattr(lib, n) is not None
    # nothing else leaks out of the library but the C ABI
    assert all(e.startswith("lf_") for e in exported), sorted(exported)


def test_version_and_strerror(lib):
    assert binding.lf_version() >> 16 == 1
    for code in (0, -1, -2, -3, -4, -5):
        assert binding.lf_strerror(code).startswith("LF_")
    assert "unknown" in binding.lf_strerror(-99)


def test_host_validation_before_cuda(lib):
    h = ctypes.c_void_p()
    bad = [(0, 8, 2, 128, 64), (1, 8, 3, 128, 64), (1, 8, 2, 96, 64), (1, 18, 2, 128, 64),
           (1, 8, 2, 128, 0), (40000, 8, 2, 128, 64)]
    for args in bad:
        assert lib.lf_init(ctypes.byref(h), *args, None) == binding.LF_EINVAL, args
        assert not h.value
    assert lib.lf_init(None, 1, 8, 2, 128, 64, None) == binding.LF_EINVAL
    # a null handle is refused by every call that takes one
    n = None
    assert lib.lf_decode_step(n, n, n, n, n, n, n, 64, 4, 8, n, n) == binding.LF_ENOTINIT
    assert lib.lf_decode_attention(n, n, n, n, n, n, n, 64, n) == binding.LF_ENOTINIT
    assert lib.lf_prefill_cache(n, n, n, 0, n, n, n, 64) == binding.LF_ENOTINIT
    assert lib.lf_get_status(n) == binding.LF_ENOTINIT
    assert lib.lf_set_split(n, 2) == binding.LF_ENOTINIT
    assert lib.lf_destroy(n) == binding.LF_ENOTINIT


def test_init_without_a_device_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    h = ctypes.c_void_p()
    assert lib.lf_init(ctypes.byref(h), 1, 8, 2, 128, 64, None) == binding.LF_ECUDA
    assert not h.value


def test_product_path_has_no_oracle_or_cpu_fallback():
    """The library package never imports the oracle."""
    pkg = os.path.join(ROOT, "attention_lf_decode_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", src, re.M), f


def test_binding_rejects_a_tensor_on_another_device():
    """A call on a handle checks that every tensor is on the handle's device
    before anything reaches the library (tensors faked on the CPU)."""
    import torch

    class OnCuda1(torch.Tensor):
        @property
        def is_cuda(self):
            return True

        @property
        def device(self):
            return torch.device("cuda", 1)

    t = torch.Tensor._make_subclass(OnCuda1, torch.zeros(4, dtype=torch.bfloat16))
    h = binding.Handle(None, 1, 1, 1, 64, 4, device=0)
    with pytest.raises(ValueError, match="cuda:1, expected cuda:0"):
        binding._hptr(h, t, torch.bfloat16, (4,), "q")
    h1 = binding.Handle(None, 1, 1, 1, 64, 4, device=1)
    assert binding._hptr(h1, t, torch.bfloat16, (4,), "q").value == t.data_ptr()
