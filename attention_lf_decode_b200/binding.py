"""Python binding of the C ABI in ``include/lf_decode.h`` (ctypes).

Argument marshalling only: every step of the decode runs in the CUDA kernels
of ``liblf_decode.so``.  Tensors are torch CUDA tensors (PyTorch provides
device memory and streams); they are checked for device, dtype, shape and
contiguity, and their data pointers are passed through.  There is no CPU
fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblf_decode.so")

LF_OK = 0
LF_EINVAL = -1
LF_ENOTINIT = -2
LF_ECUDA = -3
LF_EDEVICE = -4
LF_EUNSUPPORTED = -5
LF_STATUS_WAIT_TIMEOUT = 1
LF_STATUS_NO_CANDIDATE = 2
LF_STATUS_BAD_SEQ_BUDGET = 4
LF_SCORE_MEAN_PROB = 0
LF_SCORE_ALPHA_L1V = 1

EXPORTS = ("lf_init", "lf_set_stream", "lf_prefill_cache", "lf_decode_step",
           "lf_decode_attention", "lf_decode_step_ragged", "lf_decode_attention_ragged",
           "lf_prefill_cache_fp8", "lf_decode_step_fp8", "lf_decode_attention_fp8",
           "lf_set_split", "lf_get_split", "lf_set_score", "lf_get_score", "lf_get_status",
           "lf_status_bits", "lf_destroy", "lf_strerror", "lf_version",
           "lf_decode_step_noalloc")


class LFError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {lf_strerror(code)} ({code})")
        self.code = code


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblf_decode.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} is missing: build it with `python -m attention_lf_decode_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, VP, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_float
    sig = {
        "lf_init": ([ctypes.POINTER(P), I, I, I, I, I, VP], I),
        "lf_set_stream": ([P, VP], I),
        "lf_prefill_cache": ([P, VP, VP, I, VP, VP, VP, I], I),
        "lf_decode_step": ([P, VP, VP, VP, VP, VP, VP, I, I, I, VP, VP], I),
        "lf_decode_attention": ([P, VP, VP, VP, VP, VP, VP, I, VP], I),
        "lf_decode_step_ragged": ([P, VP, VP, VP, VP, VP, VP, I, VP, I, I, VP, VP], I),
        "lf_decode_attention_ragged": ([P, VP, VP, VP, VP, VP, VP, I, VP, VP], I),
        "lf_prefill_cache_fp8": ([P, VP, VP, I, VP, VP, VP, I, F, F], I),
        "lf_decode_step_fp8": ([P, VP, VP, VP, VP, VP, VP, I, VP, I, I, F, F, VP, VP], I),
        "lf_decode_attention_fp8": ([P, VP, VP, VP, VP, VP, VP, I, VP, F, F, VP], I),
        "lf_set_split": ([P, I], I),
        "lf_get_split": ([P, I], I),
        "lf_set_score": ([P, I], I),
        "lf_get_score": ([P], I),
        "lf_get_status": ([P], I),
        "lf_status_bits": ([P], I),
        "lf_destroy": ([P], I),
        "lf_strerror": ([I], ctypes.c_char_p),
        "lf_version": ([], I),
        "lf_decode_step_noalloc": ([VP, VP, VP, VP, VP, VP, I, I, I, I, I, I, I, VP, VP, VP], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def lf_strerror(code: int) -> str:
    return load_library().lf_strerror(int(code)).decode()


def lf_version() -> int:
    return load_library().lf_version()


def _check(code: int, what: str) -> int:
    if code < 0:
        raise LFError(code, what)
    return code


_Tensor = None  # torch.Tensor, looked up on first use


def _ptr(t, dtype, shape, name, device: Optional[int] = None):
    """Data pointer of a contiguous CUDA tensor of the given dtype/shape (on
    CUDA device ``device`` when it is given).  Runs for every tensor of every
    call, so it keeps to cheap attribute reads (no torch.device objects, no
    tuple copies)."""
    global _Tensor
    if t is None:
        return None
    if _Tensor is None:
        import torch
        _Tensor = torch.Tensor
    if not isinstance(t, _Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.get_device() != device:
        raise ValueError(f"{name} is on cuda:{t.get_device()}, expected cuda:{device}")
    if t.dtype is not dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and t.shape != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _hptr(h, t, dtype, shape, name):
    """_ptr for a call on handle h: the tensor must be on the handle's device."""
    return _ptr(t, dtype, shape, name, h.device)


class Handle:
    """An ``lf_handle`` plus the shape it was created for."""

    def __init__(self, ptr: ctypes.c_void_p, B, Hq, Hkv, D, max_budget, device: int):
        self.ptr = ptr
        self.B, self.Hq, self.Hkv, self.D, self.max_budget = B, Hq, Hkv, D, max_budget
        self.device = device  # the CUDA device index the handle was made on

    def __del__(self):
        try:
            if self.ptr:
                lf_destroy(self)
        except Exception:
            pass


def lf_init(B: int, Hq: int, Hkv: int, D: int, max_budget: int, stream=None) -> Handle:
    """Create a handle on the current CUDA device.  ``stream``: a torch
    stream, a raw cudaStream_t integer, or None for torch's current stream."""
    import torch
    lib = load_library()
    h = ctypes.c_void_p()
    _check(lib.lf_init(ctypes.byref(h), B, Hq, Hkv, D, max_budget, _stream_ptr(stream)), "lf_init")
    return Handle(h, B, Hq, Hkv, D, max_budget, torch.cuda.current_device())


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def lf_set_stream(h: Handle, stream=None) -> None:
    _check(load_library().lf_set_stream(h.ptr, _stream_ptr(stream)), "lf_set_stream")


def lf_set_split(h: Handle, split: int) -> None:
    _check(load_library().lf_set_split(h.ptr, split), "lf_set_split")


def lf_get_split(h: Handle, budget: int) -> int:
    return _check(load_library().lf_get_split(h.ptr, budget), "lf_get_split")


def lf_set_score(h: Handle, score: int) -> None:
    """LF_SCORE_MEAN_PROB (default) or LF_SCORE_ALPHA_L1V (the page's form)."""
    _check(load_library().lf_set_score(h.ptr, score), "lf_set_score")


def lf_get_score(h: Handle) -> int:
    return _check(load_library().lf_get_score(h.ptr), "lf_get_score")


def lf_prefill_cache(h: Handle, k, v, n: int, kcache, vcache, pos, budget: int) -> None:
    import torch
    bf = torch.bfloat16
    cshape = (h.B, h.Hkv, budget, h.D)
    kp = _hptr(h, k, bf, (h.B, h.Hkv, n, h.D), "k") if n > 0 else None
    vp = _hptr(h, v, bf, (h.B, h.Hkv, n, h.D), "v") if n > 0 else None
    _check(load_library().lf_prefill_cache(
        h.ptr, kp, vp, n, _hptr(h, kcache, bf, cshape, "kcache"),
        _hptr(h, vcache, bf, cshape, "vcache"),
        _hptr(h, pos, torch.int32, (h.B, h.Hkv, budget), "pos"), budget), "lf_prefill_cache")


def lf_decode_step(h: Handle, q, k_new, v_new, kcache, vcache, pos, budget: int, sink: int,
                   window: int, out, evicted_idx) -> None:
    import torch
    bf = torch.bfloat16
    cshape = (h.B, h.Hkv, budget, h.D)
    _check(load_library().lf_decode_step(
        h.ptr, _hptr(h, q, bf, (h.B, h.Hq, h.D), "q"),
        _hptr(h, k_new, bf, (h.B, h.Hkv, h.D), "k_new"),
        _hptr(h, v_new, bf, (h.B, h.Hkv, h.D), "v_new"),
        _hptr(h, kcache, bf, cshape, "kcache"), _hptr(h, vcache, bf, cshape, "vcache"),
        _hptr(h, pos, torch.int32, (h.B, h.Hkv, budget), "pos"), budget, sink, window,
        _hptr(h, out, torch.float32, (h.B, h.Hq, h.D), "out"),
        _hptr(h, evicted_idx, torch.int32, (h.B, h.Hkv), "evicted_idx")), "lf_decode_step")


def lf_decode_attention(h: Handle, q, k_new, v_new, kcache, vcache, pos, budget: int, out) -> None:
    import torch
    bf = torch.bfloat16
    cshape = (h.B, h.Hkv, budget, h.D)
    _check(load_library().lf_decode_attention(
        h.ptr, _hptr(h, q, bf, (h.B, h.Hq, h.D), "q"),
        _hptr(h, k_new, bf, (h.B, h.Hkv, h.D), "k_new"),
        _hptr(h, v_new, bf, (h.B, h.Hkv, h.D), "v_new"),
        _hptr(h, kcache, bf, cshape, "kcache"), _hptr(h, vcache, bf, cshape, "vcache"),
        _hptr(h, pos, torch.int32, (h.B, h.Hkv, budget), "pos"), budget,
        _hptr(h, out, torch.float32, (h.B, h.Hq, h.D), "out")), "lf_decode_attention")


def lf_decode_step_ragged(h: Handle, q, k_new, v_new, kcache, vcache, pos, budget: int,
                          seq_budget, sink: int, window: int, out, evicted_idx) -> None:
    """lf_decode_step with a per-sequence budget: seq_budget is a CUDA int32
    tensor [B] (see include/lf_decode.h)."""
    import torch
    bf = torch.bfloat16
    cshape = (h.B, h.Hkv, budget, h.D)
    _check(load_library().lf_decode_step_ragged(
        h.ptr, _hptr(h, q, bf, (h.B, h.Hq, h.D), "q"),
        _hptr(h, k_new, bf, (h.B, h.Hkv, h.D), "k_new"),
        _hptr(h, v_new, bf, (h.B, h.Hkv, h.D), "v_new"),
        _hptr(h, kcache, bf, cshape, "kcache"), _hptr(h, vcache, bf, cshape, "vcache"),
        _hptr(h, pos, torch.int32, (h.B, h.Hkv, budget), "pos"), budget,
        _hptr(h, seq_budget, torch.int32, (h.B,), "seq_budget"), sink, window,
        _hptr(h, out, torch.float32, (h.B, h.Hq, h.D), "out"),
        _hptr(h, evicted_idx, torch.int32, (h.B, h.Hkv), "evicted_idx")), "lf_decode_step_ragged")


def lf_decode_attention_ragged(h: Handle, q, k_new, v_new, kcache, vcache, pos, budget: int,
                               seq_budget, out) -> None:
    import torch
    bf = torch.bfloat16
    cshape = (h.B, h.Hkv, budget, h.D)
    _check(load_library().lf_decode_attention_ragged(
        h.ptr, _hptr(h, q, bf, (h.B, h.Hq, h.D), "q"),
        _hptr(h, k_new, bf, (h.B, h.Hkv, h.D), "k_new"),
        _hptr(h, v_new, bf, (h.B, h.Hkv, h.D), "v_new"),
        _hptr(h, kcache, bf, cshape, "kcache"), _hptr(h, vcache, bf, cshape, "vcache"),
        _hptr(h, pos, torch.int32, (h.B, h.Hkv, budget), "pos"), budget,
        _hptr(h, seq_budget, torch.int32, (h.B,), "seq_budget"),
        _hptr(h, out, torch.float32, (h.B, h.Hq, h.D), "out")), "lf_decode_attention_ragged")


def lf_prefill_cache_fp8(h: Handle, k, v, n: int, kcache, vcache, pos, budget: int,
                         k_scale: float, v_scale: float) -> None:
    """Prefill an E4M3 cache (kcache / vcache: CUDA uint8 [B, Hkv, budget, D])
    from bf16 prompt K/V [B, Hkv, n, D]."""
    import torch
    bf, u8 = torch.bfloat16, torch.uint8
    cshape = (h.B, h.Hkv, budget, h.D)
    kp = _hptr(h, k, bf, (h.B, h.Hkv, n, h.D), "k") if n > 0 else None
    vp = _hptr(h, v, bf, (h.B, h.Hkv, n, h.D), "v") if n > 0 else None
    _check(load_library().lf_prefill_cache_fp8(
        h.ptr, kp, vp, n, _hptr(h, kcache, u8, cshape, "kcache"),
        _hptr(h, vcache, u8, cshape, "vcache"),
        _hptr(h, pos, torch.int32, (h.B, h.Hkv, budget), "pos"), budget, k_scale, v_scale),
        "lf_prefill_cache_fp8")


def lf_decode_step_fp8(h: Handle, q, k_new, v_new, kcache, vcache, pos, budget: int, sink: int,
                       window: int, k_scale: float, v_scale: float, out, evicted_idx,
                       seq_budget=None) -> None:
    """The decode step on an E4M3 cache (see include/lf_decode.h)."""
    import torch
    bf, u8 = torch.bfloat16, torch.uint8
    cshape = (h.B, h.Hkv, budget, h.D)
    _check(load_library().lf_decode_step_fp8(
        h.ptr, _hptr(h, q, bf, (h.B, h.Hq, h.D), "q"),
        _hptr(h, k_new, bf, (h.B, h.Hkv, h.D), "k_new"),
        _hptr(h, v_new, bf, (h.B, h.Hkv, h.D), "v_new"),
        _hptr(h, kcache, u8, cshape, "kcache"), _hptr(h, vcache, u8, cshape, "vcache"),
        _hptr(h, pos, torch.int32, (h.B, h.Hkv, budget), "pos"), budget,
        None if seq_budget is None
        else _hptr(h, seq_budget, torch.int32, (h.B,), "seq_budget"),
        sink, window, k_scale, v_scale,
        _hptr(h, out, torch.float32, (h.B, h.Hq, h.D), "out"),
        _hptr(h, evicted_idx, torch.int32, (h.B, h.Hkv), "evicted_idx")), "lf_decode_step_fp8")


def lf_decode_attention_fp8(h: Handle, q, k_new, v_new, kcache, vcache, pos, budget: int,
                            k_scale: float, v_scale: float, out, seq_budget=None) -> None:
    import torch
    bf, u8 = torch.bfloat16, torch.uint8
    cshape = (h.B, h.Hkv, budget, h.D)
    _check(load_library().lf_decode_attention_fp8(
        h.ptr, _hptr(h, q, bf, (h.B, h.Hq, h.D), "q"),
        _hptr(h, k_new, bf, (h.B, h.Hkv, h.D), "k_new"),
        _hptr(h, v_new, bf, (h.B, h.Hkv, h.D), "v_new"),
        _hptr(h, kcache, u8, cshape, "kcache"), _hptr(h, vcache, u8, cshape, "vcache"),
        _hptr(h, pos, torch.int32, (h.B, h.Hkv, budget), "pos"), budget,
        None if seq_budget is None
        else _hptr(h, seq_budget, torch.int32, (h.B,), "seq_budget"),
        k_scale, v_scale, _hptr(h, out, torch.float32, (h.B, h.Hq, h.D), "out")),
        "lf_decode_attention_fp8")


def lf_decode_step_noalloc(q, k_new, v_new, kcache, vcache, pos, budget: int, sink: int,
                           window: int, out, evicted_idx, stream=None) -> None:
    """lf_decode_step without a handle and without any device allocation
    (for callers that cannot allocate; see include/lf_decode.h).  Shapes are
    taken from the tensors: q [B, Hq, D], kcache [B, Hkv, budget, D]."""
    import torch
    bf = torch.bfloat16
    B, Hq, D = q.shape
    Hkv = kcache.shape[1]
    cshape = (B, Hkv, budget, D)
    dev = torch.cuda.current_device()  # the call runs on the current device
    _check(load_library().lf_decode_step_noalloc(
        _ptr(q, bf, (B, Hq, D), "q", dev), _ptr(k_new, bf, (B, Hkv, D), "k_new", dev),
        _ptr(v_new, bf, (B, Hkv, D), "v_new", dev), _ptr(kcache, bf, cshape, "kcache", dev),
        _ptr(vcache, bf, cshape, "vcache", dev),
        _ptr(pos, torch.int32, (B, Hkv, budget), "pos", dev),
        B, Hq, Hkv, D, budget, sink, window,
        _ptr(out, torch.float32, (B, Hq, D), "out", dev),
        _ptr(evicted_idx, torch.int32, (B, Hkv), "evicted_idx", dev), _stream_ptr(stream)),
        "lf_decode_step_noalloc")


def lf_get_status(h: Handle) -> int:
    """LF_OK, or LF_EDEVICE (bits from lf_status_bits); raises on LF_ECUDA."""
    code = load_library().lf_get_status(h.ptr)
    if code not in (LF_OK, LF_EDEVICE):
        raise LFError(code, "lf_get_status")
    return code


def lf_status_bits(h: Handle) -> int:
    return _check(load_library().lf_status_bits(h.ptr), "lf_status_bits")


def lf_destroy(h: Handle) -> None:
    if h.ptr:
        code = load_library().lf_destroy(h.ptr)
        h.ptr = None
        _check(code, "lf_destroy")


# ---------------------------------------------------------------- helpers

def bf16_from_bits(bits, device="cuda"):
    """torch bf16 tensor on ``device`` from a numpy uint16 bit array."""
    import numpy as np
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def bits_from_bf16(t):
    """numpy uint16 bits of a bf16 tensor (copied to the host)."""
    import numpy as np
    return t.detach().contiguous().view(__import__("torch").int16).cpu().numpy().view(np.uint16)
