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


def _fake_cuda(shape, dtype, index=0):
    """A CPU tensor that reports itself as living on cuda:<index>; only its
    metadata is read (the library is never called with it)."""
    import torch

    class FakeCuda(torch.Tensor):
        @property
        def is_cuda(self):
            return True

        @property
        def device(self):
            return torch.device("cuda", index)

        def get_device(self):
            return index

    return torch.Tensor._make_subclass(FakeCuda, torch.zeros(shape, dtype=dtype))


def test_binding_rejects_a_tensor_on_another_device():
    """A call on a handle checks that every tensor is on the handle's device
    before anything reaches the library."""
    import torch
    t = _fake_cuda((4,), torch.bfloat16, index=1)
    h = binding.Handle(None, 1, 1, 1, 64, 4, device=0)
    with pytest.raises(ValueError, match="cuda:1, expected cuda:0"):
        binding._hptr(h, t, torch.bfloat16, (4,), "q")
    h1 = binding.Handle(None, 1, 1, 1, 64, 4, device=1)
    assert binding._hptr(h1, t, torch.bfloat16, (4,), "q").value == t.data_ptr()


def test_every_wrapper_marshals_its_arguments(lib, monkeypatch):
    """Each Python wrapper calls its C function with as many arguments as the
    ctypes signature declares, pointers as c_void_p (or None where the header
    allows NULL); a recording stand-in replaces the library, so no CUDA call
    is made."""
    import torch
    calls = []

    class Recorder:
        def __getattr__(self, name):
            real = getattr(lib, name)

            def fn(*args):
                assert len(args) == len(real.argtypes), (name, len(args), len(real.argtypes))
                for a, t in zip(args, real.argtypes):
                    if t is ctypes.c_void_p:
                        assert a is None or isinstance(a, ctypes.c_void_p), (name, a)
                calls.append(name)
                return 2 if name == "lf_get_split" else 0
            return fn

    monkeypatch.setattr(binding, "_lib", Recorder())
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    mk = _fake_cuda
    B, Hq, Hkv, D, N, n = 2, 8, 2, 64, 32, 16
    bf, u8, i32, f32 = torch.bfloat16, torch.uint8, torch.int32, torch.float32
    h = binding.Handle(ctypes.c_void_p(1), B, Hq, Hkv, D, N, device=0)
    q, kn, vn = mk((B, Hq, D), bf), mk((B, Hkv, D), bf), mk((B, Hkv, D), bf)
    kc, vc = mk((B, Hkv, N, D), bf), mk((B, Hkv, N, D), bf)
    kc8, vc8 = mk((B, Hkv, N, D), u8), mk((B, Hkv, N, D), u8)
    pos, out, ev = mk((B, Hkv, N), i32), mk((B, Hq, D), f32), mk((B, Hkv), i32)
    kp, vp, nb = mk((B, Hkv, n, D), bf), mk((B, Hkv, n, D), bf), mk((B,), i32)

    binding.lf_set_stream(h, 0)
    binding.lf_set_split(h, 2)
    assert binding.lf_get_split(h, N) == 2
    binding.lf_set_score(h, binding.LF_SCORE_ALPHA_L1V)
    binding.lf_get_score(h)
    binding.lf_prefill_cache(h, kp, vp, n, kc, vc, pos, N)
    binding.lf_prefill_cache(h, None, None, 0, kc, vc, pos, N)
    binding.lf_decode_step(h, q, kn, vn, kc, vc, pos, N, 4, 8, out, ev)
    binding.lf_decode_attention(h, q, kn, vn, kc, vc, pos, N, out)
    binding.lf_decode_step_ragged(h, q, kn, vn, kc, vc, pos, N, nb, 4, 8, out, ev)
    binding.lf_decode_attention_ragged(h, q, kn, vn, kc, vc, pos, N, nb, out)
    binding.lf_prefill_cache_fp8(h, kp, vp, n, kc8, vc8, pos, N, 0.5, 2.0)
    for seq in (None, nb):
        binding.lf_decode_step_fp8(h, q, kn, vn, kc8, vc8, pos, N, 4, 8, 0.5, 2.0, out, ev, seq)
        binding.lf_decode_attention_fp8(h, q, kn, vn, kc8, vc8, pos, N, 0.5, 2.0, out, seq)
    binding.lf_decode_step_noalloc(q, kn, vn, kc, vc, pos, N, 4, 8, out, ev, stream=0)
    assert binding.lf_get_status(h) == binding.LF_OK
    binding.lf_status_bits(h)
    binding.lf_destroy(h)
    assert h.ptr is None
    assert set(calls) >= set(binding.EXPORTS) - {"lf_init", "lf_strerror", "lf_version"}

    # a wrongly shaped or typed tensor is refused before the library is called
    n_calls = len(calls)
    h = binding.Handle(ctypes.c_void_p(1), B, Hq, Hkv, D, N, device=0)
    with pytest.raises(ValueError, match="shape"):
        binding.lf_decode_step(h, q, kn, vn, kc, vc, pos, N + 1, 4, 8, out, ev)
    with pytest.raises(TypeError, match="uint8"):
        binding.lf_decode_step_fp8(h, q, kn, vn, kc, vc, pos, N, 4, 8, 1.0, 1.0, out, ev)
    assert len(calls) == n_calls
    h.ptr = None
