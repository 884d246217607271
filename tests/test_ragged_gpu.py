"""GPU parity of ragged batches (a budget per sequence) against the oracle's
``seq_budget``: lf_decode_step_ragged and lf_decode_attention_ragged.

Each sequence b owns slots 0 .. n_b - 1; the slots beyond hold junk (NaN
values, positions far ahead) that must be neither read nor written.
Sequences at different fill levels share a batch (some append, some
evict).  Covered: every split, both scores, the configured ragged workload
at full size on sampled rows, a CUDA graph replaying ragged steps (the row
counter of the dynamic schedule must be back at zero after every launch),
split changes between calls, out-of-range budgets (status bit, nothing
written) and the attention-only call.
"""
import numpy as np
import pytest

import oracle
from attention_lf_decode_b200 import binding, synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu
NAN_BF16 = 0x7FC0


@pytest.fixture(autouse=True)
def _cuda(cuda_ok):
    binding.load_library()


def _bits(rng, shape, scale=1.0):
    return synth.to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _custom(B, Hq, Hkv, D, N, sink, window, seed=0):
    return synth.DecodeConfig("custom", batch=B, hq=Hq, hkv=Hkv, head_dim=D, budget=N,
                              sink=sink, window=window, prefill=N, steps=8, seed=seed)


def ragged_state(rng, B, Hkv, D, N, nb, fill_frac):
    """Host state: sequence b has fill_frac[b] * nb[b] filled slots (scattered
    inside its budget, unique positions); junk beyond nb[b]."""
    kb = _bits(rng, (B, Hkv, N, D))
    vb = _bits(rng, (B, Hkv, N, D))
    pos = np.full((B, Hkv, N), -1, np.int32)
    for b in range(B):
        n = int(nb[b])
        f = int(round(fill_frac[b] * n))
        for g in range(Hkv):
            slots = rng.permutation(n)[:f]
            pos[b, g, slots] = rng.permutation(f) + 3
            pos[b, g, n:] = 1_000_000 + np.arange(N - n)
        kb[b, :, n:] = NAN_BF16
        vb[b, :, n:] = NAN_BF16
    return kb, vb, pos


class RaggedRun:
    """Device state plus the per-sequence budgets, stepped through the C ABI."""

    def __init__(self, cfg, nb, kb, vb, pos, split=0, score="mean_prob"):
        import torch
        self.torch = torch
        self.cfg = cfg
        self.g = H.GpuCache(cfg, n=0, split=split, score=score)
        self.g.set_state(kb, vb, pos)
        self.nb_host = np.asarray(nb, np.int32)
        self.nb = torch.from_numpy(self.nb_host.copy()).cuda()
        self.score = score

    def step(self, qb, knb, vnb, attention_only=False):
        c, g = self.cfg, self.g
        q, kn, vn = (binding.bf16_from_bits(x) for x in (qb, knb, vnb))
        if attention_only:
            binding.lf_decode_attention_ragged(g.h, q, kn, vn, g.kcache, g.vcache, g.pos,
                                               c.budget, self.nb, g.out)
        else:
            binding.lf_decode_step_ragged(g.h, q, kn, vn, g.kcache, g.vcache, g.pos, c.budget,
                                          self.nb, c.sink, c.window, g.out, g.evicted)


def run_teacher_forced(cfg, nb, kb, vb, pos, steps, rng, split=0, score="mean_prob"):
    r = RaggedRun(cfg, nb, kb, vb, pos, split=split, score=score)
    stats = H.Stats()
    B, Hq, Hkv, D = cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim
    for s in range(steps):
        qb, knb, vnb = _bits(rng, (B, Hq, D)), _bits(rng, (B, Hkv, D)), _bits(rng, (B, Hkv, D))
        r.step(qb, knb, vnb)
        res = oracle.decode_step(*H.oracle_state(kb, vb, pos), synth.bf16_bits_to_f64(qb),
                                 synth.bf16_bits_to_f64(knb), synth.bf16_bits_to_f64(vnb),
                                 cfg.sink, cfg.window, score=score, seq_budget=nb)
        kb, vb, pos = H.check_step(res, pos, r.g.host_rows(), stats, kb, vb, knb, vnb, f"s{s}")
    code, bits = r.g.status()
    assert code == binding.LF_OK, bits
    return stats, r


@pytest.mark.parametrize("split", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("score", ["mean_prob", "alpha_l1v"])
def test_ragged_budgets_every_split(split, score):
    rng = np.random.default_rng(100 + split)
    B, Hq, Hkv, D, N, sink, window = 7, 8, 2, 128, 1000, 4, 8
    nb = rng.integers(sink + window + 1, N + 1, size=B)
    nb[0], nb[1] = N, sink + window + 1
    fill = np.where(rng.random(B) < 0.6, 1.0, rng.random(B))
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=split)
    kb, vb, pos = ragged_state(rng, B, Hkv, D, N, nb, fill)
    st, _ = run_teacher_forced(cfg, nb, kb, vb, pos, 4, rng, split=split, score=score)
    assert st.rows == 4 * B * Hkv


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 4, 64), (7, 1, 128), (16, 2, 128)])
def test_ragged_group_sizes(Hq, Hkv, D):
    rng = np.random.default_rng(Hq + D)
    B, N, sink, window = 5, 700, 4, 16
    nb = rng.integers(sink + window + 1, N + 1, size=B)
    fill = np.ones(B)
    fill[2] = 0.5
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=Hq)
    kb, vb, pos = ragged_state(rng, B, Hkv, D, N, nb, fill)
    run_teacher_forced(cfg, nb, kb, vb, pos, 3, rng)


def test_ragged_appends_until_each_budget_is_full():
    """Every sequence starts with 4 free slots inside its budget: 4 appends
    each, then evictions, each at its own budget."""
    rng = np.random.default_rng(7)
    B, Hq, Hkv, D, N, sink, window = 6, 8, 2, 128, 300, 4, 8
    nb = np.array([300, 13, 100, 257, 64, 199])
    fill = (nb - 4) / nb
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=7)
    kb, vb, pos = ragged_state(rng, B, Hkv, D, N, nb, fill)
    st, _ = run_teacher_forced(cfg, nb, kb, vb, pos, 8, rng)
    assert st.appends == 4 * B * Hkv


def test_ragged_workload_full_size_sampled_rows():
    """The configured ragged workload (batch 64, budget 4096, per-sequence
    budgets in [1024, 4096]) in the launch configuration the bench times."""
    cfg = synth.CONFIGS["ragged"]
    gen = synth.SynthDecode(cfg)
    nb = gen.seq_budgets()
    kpre, vpre = gen.prefill()
    r = RaggedRun(cfg, nb, *synth.prefill_layout(kpre, vpre, cfg.budget))
    sel = [0, 17, 63]
    kb, vb, pos = synth.prefill_layout(kpre[sel], vpre[sel], cfg.budget)
    del kpre, vpre
    stats = H.Stats()
    for s in range(3):
        qb, knb, vnb = gen.step_inputs(s)
        r.step(qb, knb, vnb)
        res = oracle.decode_step(*H.oracle_state(kb, vb, pos), synth.bf16_bits_to_f64(qb[sel]),
                                 synth.bf16_bits_to_f64(knb[sel]), synth.bf16_bits_to_f64(vnb[sel]),
                                 cfg.sink, cfg.window, seq_budget=nb[sel])
        kb, vb, pos = H.check_step(res, pos, r.g.host_rows(sel), stats, kb, vb, knb[sel],
                                   vnb[sel], f"s{s}")
    assert r.g.status()[0] == binding.LF_OK


def test_ragged_graph_replay_resets_the_row_counter():
    """Three ragged steps captured in one CUDA graph, replayed four times:
    every launch must see the counter at zero again, or rows would be
    skipped.  Compared with the oracle after each replay."""
    import torch
    rng = np.random.default_rng(9)
    B, Hq, Hkv, D, N, sink, window = 9, 8, 2, 128, 600, 4, 8
    nb = rng.integers(sink + window + 1, N + 1, size=B)
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=9)
    kb, vb, pos = ragged_state(rng, B, Hkv, D, N, nb, np.ones(B))
    r = RaggedRun(cfg, nb, kb, vb, pos)
    ins = [(_bits(rng, (B, Hq, D)), _bits(rng, (B, Hkv, D)), _bits(rng, (B, Hkv, D))) for _ in range(3)]
    dev = [tuple(binding.bf16_from_bits(x) for x in t) for t in ins]
    g = r.g
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    binding.lf_set_stream(g.h, stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for q, kn, vn in dev:
            binding.lf_decode_step_ragged(g.h, q, kn, vn, g.kcache, g.vcache, g.pos, N, r.nb,
                                          sink, window, g.out, g.evicted)
    binding.lf_set_stream(g.h, torch.cuda.current_stream())
    torch.cuda.synchronize()
    # capture does not run the kernels: the state is still the initial one
    stats = H.Stats()
    for rep in range(4):
        graph.replay()
        torch.cuda.synchronize()
        for i, (qb, knb, vnb) in enumerate(ins):
            res = oracle.decode_step(*H.oracle_state(kb, vb, pos), synth.bf16_bits_to_f64(qb),
                                     synth.bf16_bits_to_f64(knb), synth.bf16_bits_to_f64(vnb),
                                     sink, window, seq_budget=nb)
            # only the last step of a replay is visible; follow the oracle
            if i < 2:
                kb = synth.to_bf16_bits(res.kcache.astype(np.float32))
                vb = synth.to_bf16_bits(res.vcache.astype(np.float32))
                pos = res.pos.astype(np.int32)
                continue
            kb, vb, pos = H.check_step(res, pos, g.host_rows(), stats, kb, vb, knb, vnb,
                                       f"replay {rep}")
    assert g.status()[0] == binding.LF_OK


def test_ragged_split_changes_between_calls():
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, N, sink, window = 5, 8, 2, 128, 900, 4, 8
    nb = rng.integers(sink + window + 1, N + 1, size=B)
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=11)
    kb, vb, pos = ragged_state(rng, B, Hkv, D, N, nb, np.ones(B))
    r = RaggedRun(cfg, nb, kb, vb, pos)
    stats = H.Stats()
    for s, split in enumerate([2, 8, 1, 16, 4, 0, 2]):
        binding.lf_set_split(r.g.h, split)
        qb, knb, vnb = _bits(rng, (B, Hq, D)), _bits(rng, (B, Hkv, D)), _bits(rng, (B, Hkv, D))
        r.step(qb, knb, vnb)
        res = oracle.decode_step(*H.oracle_state(kb, vb, pos), synth.bf16_bits_to_f64(qb),
                                 synth.bf16_bits_to_f64(knb), synth.bf16_bits_to_f64(vnb),
                                 sink, window, seq_budget=nb)
        kb, vb, pos = H.check_step(res, pos, r.g.host_rows(), stats, kb, vb, knb, vnb, f"s{s}")


def test_ragged_attention_only():
    rng = np.random.default_rng(13)
    B, Hq, Hkv, D, N = 6, 8, 2, 128, 800
    nb = rng.integers(1, N + 1, size=B)
    cfg = _custom(B, Hq, Hkv, D, N, 4, 8, seed=13)
    kb, vb, pos = ragged_state(rng, B, Hkv, D, N, nb, rng.random(B))
    r = RaggedRun(cfg, nb, kb, vb, pos)
    qb, knb, vnb = _bits(rng, (B, Hq, D)), _bits(rng, (B, Hkv, D)), _bits(rng, (B, Hkv, D))
    r.step(qb, knb, vnb, attention_only=True)
    out, _, kb2, vb2, pos2 = r.g.host_rows()
    ref = oracle.decode_attention(*H.oracle_state(kb, vb, pos), synth.bf16_bits_to_f64(qb),
                                  synth.bf16_bits_to_f64(knb), synth.bf16_bits_to_f64(vnb),
                                  seq_budget=nb)
    assert np.max(np.abs(out - ref)) <= H.OUT_ATOL
    assert np.array_equal(kb2, kb) and np.array_equal(vb2, vb) and np.array_equal(pos2, pos)


def test_ragged_bad_budget_flags_status_and_writes_nothing():
    rng = np.random.default_rng(15)
    B, Hq, Hkv, D, N, sink, window = 4, 8, 2, 128, 256, 4, 8
    nb = np.array([256, 0, 300, 100])
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=15)
    kb, vb, pos = ragged_state(rng, B, Hkv, D, N, np.clip(nb, 1, N), np.ones(B))
    r = RaggedRun(cfg, nb, kb, vb, pos)
    qb, knb, vnb = _bits(rng, (B, Hq, D)), _bits(rng, (B, Hkv, D)), _bits(rng, (B, Hkv, D))
    r.step(qb, knb, vnb)
    code, bits = r.g.status()
    assert code == binding.LF_EDEVICE and bits & binding.LF_STATUS_BAD_SEQ_BUDGET
    _, ev, kb2, vb2, pos2 = r.g.host_rows()
    assert (ev[1] == -2).all() and (ev[2] == -2).all()
    for b in (1, 2):
        assert np.array_equal(kb2[b], kb[b]) and np.array_equal(pos2[b], pos[b])
    # the valid sequences were stepped normally
    res = oracle.decode_step(*H.oracle_state(kb[[0, 3]], vb[[0, 3]], pos[[0, 3]]),
                             synth.bf16_bits_to_f64(qb[[0, 3]]), synth.bf16_bits_to_f64(knb[[0, 3]]),
                             synth.bf16_bits_to_f64(vnb[[0, 3]]), sink, window, seq_budget=nb[[0, 3]])
    np.testing.assert_array_equal(ev[[0, 3]], res.evicted)


def test_ragged_host_checks():
    import torch
    h = binding.lf_init(2, 4, 2, 128, 256)
    try:
        lib = binding.load_library()
        z = torch.zeros(1 << 16, dtype=torch.int32, device="cuda")
        p = z.data_ptr()
        assert lib.lf_decode_step_ragged(h.ptr, p, p, p, p, p, p, 256, None, 4, 8, p, p) == binding.LF_EINVAL
        assert lib.lf_decode_step_ragged(h.ptr, p, p, p, p, p, p, 256, p + 2, 4, 8, p, p) == binding.LF_EINVAL
        assert lib.lf_decode_attention_ragged(h.ptr, p, p, p, p, p, p, 256, None, p) == binding.LF_EINVAL
    finally:
        binding.lf_destroy(h)
