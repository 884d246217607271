"""The allocation-free entry point, lf_decode_step_noalloc.

It serves callers that cannot allocate device memory (runtimes that reserve
the device memory in a pool of their own, hosts that pass only buffers and a
stream): it takes no handle, and its scratch (the kernel's status word) is a
fixed array inside the library.  Here it is called through the C ABI on two
steps in a row and checked against lf_decode_step on an identical copy of the
cache, within the tolerance the other GPU tests use.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process (it builds all of its own state).
"""
import ctypes

import numpy as np
import pytest

from attention_lf_decode_b200 import binding, synth

pytestmark = pytest.mark.gpu

OUT_ATOL = 2e-3


def test_noalloc_matches_handle_path_two_calls(cuda_ok):
    import torch
    lib = binding.load_library()
    cfg = synth.CONFIGS["llama3_8b"].with_(batch=2, budget=1024, prefill=1024, window=32)
    gen = synth.SynthDecode(cfg)
    kpre, vpre = gen.prefill()
    caches = []
    for _ in range(2):
        kc = binding.bf16_from_bits(synth.prefill_layout(kpre, vpre, cfg.budget)[0])
        vc = binding.bf16_from_bits(synth.prefill_layout(kpre, vpre, cfg.budget)[1])
        pos = torch.from_numpy(synth.prefill_layout(kpre, vpre, cfg.budget)[2]).cuda()
        caches.append((kc, vc, pos))
    h = binding.lf_init(cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim, cfg.budget)
    stream = torch.cuda.current_stream()
    shape_o = (cfg.batch, cfg.hq, cfg.head_dim)
    for s in range(2):
        qb, knb, vnb = gen.step_inputs(s)
        q, kn, vn = (binding.bf16_from_bits(x) for x in (qb, knb, vnb))
        out_a = torch.full(shape_o, float("nan"), dtype=torch.float32, device="cuda")
        out_b = torch.full(shape_o, float("nan"), dtype=torch.float32, device="cuda")
        ev_a = torch.full((cfg.batch, cfg.hkv), -9, dtype=torch.int32, device="cuda")
        ev_b = torch.full((cfg.batch, cfg.hkv), -9, dtype=torch.int32, device="cuda")
        kc, vc, pos = caches[0]
        binding.lf_decode_step(h, q, kn, vn, kc, vc, pos, cfg.budget, cfg.sink, cfg.window,
                               out_a, ev_a)
        kc, vc, pos = caches[1]
        P = ctypes.c_void_p
        rc = lib.lf_decode_step_noalloc(
            P(q.data_ptr()), P(kn.data_ptr()), P(vn.data_ptr()), P(kc.data_ptr()),
            P(vc.data_ptr()), P(pos.data_ptr()), cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim,
            cfg.budget, cfg.sink, cfg.window, P(out_b.data_ptr()), P(ev_b.data_ptr()),
            P(stream.cuda_stream))
        assert rc == binding.LF_OK, binding.lf_strerror(rc)
        torch.cuda.synchronize()
        a, b = out_a.cpu().numpy(), out_b.cpu().numpy()
        assert np.isfinite(b).all()
        assert np.abs(a - b).max() <= OUT_ATOL
        assert np.array_equal(ev_a.cpu().numpy(), ev_b.cpu().numpy())
        assert (ev_b.cpu().numpy() >= 0).all()
        for x, y in zip(caches[0], caches[1]):
            assert torch.equal(x, y)
    assert binding.lf_get_status(h) == binding.LF_OK
    binding.lf_destroy(h)


def test_noalloc_rejects_bad_shapes_on_host(cuda_ok):
    lib = binding.load_library()
    n = None
    # Hq not a multiple of Hkv; unsupported head dim; budget too large
    assert lib.lf_decode_step_noalloc(n, n, n, n, n, n, 1, 6, 4, 128, 64, 4, 8, n, n, n) == binding.LF_EINVAL
    assert lib.lf_decode_step_noalloc(n, n, n, n, n, n, 1, 8, 2, 96, 64, 4, 8, n, n, n) == binding.LF_EINVAL
    assert lib.lf_decode_step_noalloc(n, n, n, n, n, n, 1, 8, 2, 128, (1 << 22) + 1, 4, 8, n, n, n) == binding.LF_EINVAL
    # null pointers are rejected by the same checks as lf_decode_step
    assert lib.lf_decode_step_noalloc(n, n, n, n, n, n, 1, 8, 2, 128, 64, 4, 8, n, n, n) == binding.LF_EINVAL
