"""GPU parity: the fused decode kernel (through the C ABI) against the oracle.

Teacher-forced: every step starts from the same state on both sides.
Workloads: the five configured decode workloads (full sizes on sampled rows,
or all rows with fewer steps), plus edge cases: ragged budgets, every split,
free slots, empty cache, minimum budget, uniform keys (ties), planted near
ties, G = 1/7/8, D = 64/128, the no-eviction control.
"""
import numpy as np
import pytest

import oracle
from attention_lf_decode_b200 import binding, synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda(cuda_ok):
    binding.load_library()


def _bits(rng, shape, scale=1.0, shift=None):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    if shift is not None:
        x = x + shift.astype(np.float32)
    return synth.to_bf16_bits(x)


# ------------------------------------------------------- configured workloads

def test_tiny_all_steps():
    st = H.teacher_forced(synth.CONFIGS["tiny"], steps=64)
    assert st.exact_evictions + st.accepted_ties == 64 * 2


def test_llama3_8b_shape_all_rows():
    st = H.teacher_forced(synth.CONFIGS["llama3_8b"], steps=12)
    assert st.rows == 12 * 64


def test_llama3_8b_shape_sampled_rows_long():
    st = H.teacher_forced(synth.CONFIGS["llama3_8b"], steps=96, batch_idx=[0, 5])
    assert st.max_abs < 1e-4


def test_throughput_full_size_sampled_rows():
    """Batch 64, budget 4096, in the launch configuration the bench times."""
    cfg = synth.CONFIGS["throughput"]
    st = H.teacher_forced(cfg, steps=4, batch_idx=[0, 31, 63])
    assert st.rows == 4 * 3 * 8


def test_long_reasoning_g7_sampled_rows():
    cfg = synth.CONFIGS["long_reasoning"]
    st = H.teacher_forced(cfg, steps=6, batch_idx=[0, 15])
    assert st.rows == 6 * 2 * 4


@pytest.mark.parametrize("budget", [1024, 2048, 4096, 8192])
def test_budget_sweep_sampled_rows(budget):
    cfg = synth.CONFIGS[f"sweep_n{budget}"]
    H.teacher_forced(cfg, steps=3, batch_idx=[0, 31])


def test_sweep_control_no_eviction_and_plain_attention():
    """Budget 16384 with 8192 prefilled: no eviction (append), and the fused
    step's output equals the plain attention kernel's bit for bit."""
    cfg = synth.CONFIGS["sweep_control"].with_(batch=4)
    gen = synth.SynthDecode(cfg)
    kpre, vpre = gen.prefill()
    g = H.GpuCache(cfg, kpre, vpre)
    kb, vb, pos = synth.prefill_layout(kpre, vpre, cfg.budget)
    stats = H.Stats()
    for s in range(3):
        qb, knb, vnb = gen.step_inputs(s)
        g.step(qb, knb, vnb, attention_only=True)
        ctrl = g.out.cpu().numpy().copy()
        g.step(qb, knb, vnb)
        K, V, P = H.oracle_state(kb, vb, pos)
        qf, knf, vnf = (synth.bf16_bits_to_f64(x) for x in (qb, knb, vnb))
        plain = oracle.decode_attention(K, V, P, qf, knf, vnf)
        assert np.abs(ctrl - plain).max() <= H.OUT_ATOL
        res = oracle.decode_step(K, V, P, qf, knf, vnf, cfg.sink, cfg.window)
        gpu = g.host_rows()
        np.testing.assert_array_equal(ctrl, gpu[0])
        assert (gpu[1] == -1).all()
        kb, vb, pos = H.check_step(res, pos, gpu, stats, kb, vb, knb, vnb, f"control {s}")
    assert stats.appends == 3 * cfg.rows


# ------------------------------------------------------------- edge cases

def _custom(B, Hq, Hkv, D, N, sink, window, seed=0, **kw):
    return synth.DecodeConfig("custom", batch=B, hq=Hq, hkv=Hkv, head_dim=D, budget=N,
                              sink=sink, window=window, prefill=N, steps=8, seed=seed, **kw)


@pytest.mark.parametrize("N", [300, 301, 97, 1000])
@pytest.mark.parametrize("split", [1, 2, 4, 8, 16])
def test_ragged_budgets_every_split(N, split):
    cfg = _custom(2, 8, 2, 128, N, 4, 8, seed=N)
    H.teacher_forced(cfg, steps=3, split=split)


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 4, 128), (7, 1, 128), (8, 1, 64), (6, 2, 64),
                                      (16, 8, 64), (24, 8, 128), (3, 1, 128), (10, 2, 128)])
def test_group_sizes_and_head_dims(Hq, Hkv, D):
    cfg = _custom(3, Hq, Hkv, D, 520, 4, 16, seed=Hq * 10 + D)
    H.teacher_forced(cfg, steps=4)


def test_minimum_budget_single_candidate():
    cfg = _custom(2, 8, 2, 128, 4 + 8 + 1, 4, 8, seed=9)
    H.teacher_forced(cfg, steps=10)


def test_budget_covers_length_appends_then_evicts():
    """Prefill 40 of 48 slots: 8 appends (no eviction), then evictions."""
    cfg = _custom(2, 8, 2, 128, 48, 4, 8, seed=11).with_(prefill=40)
    st = H.teacher_forced(cfg, steps=14)
    assert st.appends == 8 * 4


@pytest.mark.parametrize("D,prefill", [(128, 150), (64, 310)])
def test_appends_across_every_tile_tail(D, prefill):
    """One CTA per row, the filled prefix growing one slot per step across the
    last 32 slots of the first tile (176 slots at D = 128, 352 at D = 64):
    the free tail of a partly filled tile must stay masked."""
    cfg = _custom(2, 8, 2, D, 600, 4, 8, seed=D).with_(prefill=prefill)
    st = H.teacher_forced(cfg, steps=50, split=1)
    assert st.appends == 50 * 4


def test_budget_beyond_shared_memory_is_rejected_on_the_host():
    """A budget whose per-CTA logits cannot fit in shared memory even at
    16 CTAs per row is rejected with LF_EINVAL before anything is launched;
    a large feasible budget gets a split."""
    h = binding.lf_init(1, 8, 2, 128, 1 << 21)
    try:
        lib = binding.load_library()
        assert lib.lf_get_split(h.ptr, 1 << 21) == binding.LF_EINVAL
        assert lib.lf_get_split(h.ptr, 16384) in (1, 2, 4, 8, 16)
    finally:
        binding.lf_destroy(h)


def test_empty_cache_first_step_returns_v_new():
    cfg = _custom(1, 4, 2, 64, 64, 4, 8, seed=12).with_(prefill=0)
    st = H.teacher_forced(cfg, steps=5)
    assert st.appends == 5 * 2


def test_scattered_free_slots_lowest_first():
    rng = np.random.default_rng(21)
    cfg = _custom(2, 8, 2, 128, 200, 4, 8, seed=21)
    kb = _bits(rng, (2, 2, 200, 128))
    vb = _bits(rng, (2, 2, 200, 128))
    pos = np.full((2, 2, 200), -1, np.int32)
    for b in range(2):
        for g in range(2):
            slots = rng.permutation(200)[:150]
            pos[b, g, slots] = rng.permutation(150)
    g_ = H.GpuCache(cfg, n=0)
    g_.set_state(kb, vb, pos)
    stats = H.Stats()
    for s in range(60):  # fills the 50 free slots, then evicts
        qb, knb, vnb = _bits(rng, (2, 8, 128)), _bits(rng, (2, 2, 128)), _bits(rng, (2, 2, 128))
        g_.step(qb, knb, vnb)
        res = oracle.decode_step(*H.oracle_state(kb, vb, pos), synth.bf16_bits_to_f64(qb),
                                 synth.bf16_bits_to_f64(knb), synth.bf16_bits_to_f64(vnb),
                                 cfg.sink, cfg.window)
        kb, vb, pos = H.check_step(res, pos, g_.host_rows(), stats, kb, vb, knb, vnb, f"s{s}")
    assert stats.appends == 50 * 4


@pytest.mark.parametrize("N,sink,window,G", [(64, 4, 6, 1), (256, 4, 16, 4), (1000, 4, 32, 7)])
def test_uniform_keys_ties_go_to_lowest_slot(N, sink, window, G):
    """All keys equal: every score ties, the fp64 rescoring runs on every
    candidate, and the evictions cycle through slots sink..sink+window."""
    rng = np.random.default_rng(N)
    cfg = _custom(2, 2 * G, 2, 128, N, sink, window, seed=N)
    k0 = _bits(rng, (2, 2, 1, 128))
    kb = np.broadcast_to(k0, (2, 2, N, 128)).copy()
    vb = _bits(rng, (2, 2, N, 128))
    pos = np.broadcast_to(np.arange(N, dtype=np.int32), (2, 2, N)).copy()
    g_ = H.GpuCache(cfg, n=0)
    g_.set_state(kb, vb, pos)
    for k in range(2 * (window + 1) + 3):
        qb = _bits(rng, (2, 2 * G, 128))
        vnb = _bits(rng, (2, 2, 128))
        g_.step(qb, k0[:, :, 0], vnb)
        _, ev, _, _, _ = g_.host_rows()
        assert (ev == sink + (k % (window + 1))).all(), (k, ev)


def test_planted_near_ties_match_exact_ranking():
    """Pairs of keys that differ by one bf16 ulp in the dimension where the
    group's queries are smallest give scores within ~1e-4..1e-8 relative: the
    fp64 rescoring must pick the oracle's slot whenever the oracle's gap is at
    least 1e-6 relative (the harness enforces it)."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, D, N, sink, window = 4, 16, 4, 128, 512, 4, 16
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=5)
    kb = _bits(rng, (B, Hkv, N, D))
    vb = _bits(rng, (B, Hkv, N, D))
    pos = np.broadcast_to(np.arange(N, dtype=np.int32), (B, Hkv, N)).copy()
    g_ = H.GpuCache(cfg, n=0)
    stats = H.Stats()
    for s in range(20):
        qb = _bits(rng, (B, Hq, D))
        qf = synth.bf16_bits_to_f64(qb)
        # plant: the two lowest-logit keys of each row become near copies
        for b in range(B):
            for g in range(Hkv):
                qg = qf[b, g * (Hq // Hkv):(g + 1) * (Hq // Hkv)]
                base = -np.sign(qg.mean(axis=0)) * 2.0
                d = int(np.argmin(np.abs(qg).max(axis=0)))
                base[d] = 2.0 ** -int(rng.choice([1, 4, 8, 12]))
                k1 = synth.to_bf16_bits(base.astype(np.float32))
                k2 = k1.copy()
                k2[d] = k2[d] + 1
                j1, j2 = 100 + s, 300 + s
                kb[b, g, j1], kb[b, g, j2] = k1, k2
        g_.set_state(kb, vb, pos)
        knb, vnb = _bits(rng, (B, Hkv, D)), _bits(rng, (B, Hkv, D))
        g_.step(qb, knb, vnb)
        res = oracle.decode_step(*H.oracle_state(kb, vb, pos), qf, synth.bf16_bits_to_f64(knb),
                                 synth.bf16_bits_to_f64(vnb), sink, window)
        kb, vb, pos = H.check_step(res, pos, g_.host_rows(), stats, kb, vb, knb, vnb, f"s{s}")
    assert stats.exact_evictions + stats.accepted_ties == 20 * B * Hkv


def test_no_candidate_flags_status():
    """A corrupt position table (all positions equal) leaves no candidate:
    the kernel flags it, writes evicted = -2 and changes nothing."""
    rng = np.random.default_rng(3)
    cfg = _custom(1, 4, 2, 128, 64, 4, 8, seed=3)
    kb = _bits(rng, (1, 2, 64, 128))
    vb = _bits(rng, (1, 2, 64, 128))
    pos = np.full((1, 2, 64), 70, np.int32)
    g_ = H.GpuCache(cfg, n=0)
    g_.set_state(kb, vb, pos)
    g_.step(_bits(rng, (1, 4, 128)), _bits(rng, (1, 2, 128)), _bits(rng, (1, 2, 128)))
    code, bits = g_.status()
    assert code == binding.LF_EDEVICE and bits & binding.LF_STATUS_NO_CANDIDATE
    out, ev, k2, v2, p2 = g_.host_rows()
    assert (ev == -2).all()
    assert np.array_equal(k2, kb) and np.array_equal(p2, pos)
    assert g_.status() == (binding.LF_OK, 0)


def test_invalid_arguments_rejected_on_host():
    import torch
    cfg = _custom(1, 4, 2, 128, 64, 4, 8)
    g_ = H.GpuCache(cfg, n=0)
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device="cuda")
    lib = binding.load_library()
    P = lambda t: t.data_ptr()  # noqa: E731
    args = [P(q), P(kn), P(kn), P(g_.kcache), P(g_.vcache), P(g_.pos)]
    for budget, sink, window in [(64, 4, 60), (64, 0, 0), (65, 4, 8), (0, 0, 1), (64, -1, 8)]:
        assert lib.lf_decode_step(g_.h.ptr, *args, budget, sink, window, P(g_.out),
                                  P(g_.evicted)) == binding.LF_EINVAL
    # misaligned q
    assert lib.lf_decode_step(g_.h.ptr, P(q) + 2, *args[1:], 64, 4, 8, P(g_.out),
                              P(g_.evicted)) == binding.LF_EINVAL
    assert lib.lf_prefill_cache(g_.h.ptr, None, None, 65, P(g_.kcache), P(g_.vcache),
                                P(g_.pos), 64) == binding.LF_EINVAL
    assert g_.status() == (binding.LF_OK, 0)


def test_repeatable_bit_for_bit():
    cfg = synth.CONFIGS["llama3_8b"].with_(batch=2)
    gen = synth.SynthDecode(cfg)
    kpre, vpre = gen.prefill()
    outs = []
    for _ in range(2):
        g_ = H.GpuCache(cfg, kpre, vpre)
        for s in range(3):
            g_.step(*gen.step_inputs(s))
        outs.append(g_.host_rows())
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


# ------------------------------------------------------- free running

def test_free_running_trajectory_matches_oracle():
    """The long-reasoning shape (G = 7, AR(1) queries), reduced to budget 512,
    run free on both sides from the same prefill: the eviction sequences
    must agree step for step."""
    cfg = synth.CONFIGS["long_reasoning"].with_(batch=2, budget=512, prefill=512, window=32)
    gen = synth.SynthDecode(cfg)
    kpre, vpre = gen.prefill()
    g_ = H.GpuCache(cfg, kpre, vpre)
    kb, vb, pos = synth.prefill_layout(kpre, vpre, cfg.budget)
    K, V, P = H.oracle_state(kb, vb, pos)
    for s in range(200):
        qb, knb, vnb = gen.step_inputs(s)
        g_.step(qb, knb, vnb)
        res = oracle.decode_step(K, V, P, synth.bf16_bits_to_f64(qb), synth.bf16_bits_to_f64(knb),
                                 synth.bf16_bits_to_f64(vnb), cfg.sink, cfg.window)
        K, V, P = res.kcache, res.vcache, res.pos
        ev = g_.evicted.cpu().numpy()
        assert np.array_equal(ev, res.evicted), f"step {s}: gpu {ev} oracle {res.evicted}"
        assert np.abs(g_.out.cpu().numpy() - res.out).max() <= H.OUT_ATOL
    _, _, kb2, _, p2 = g_.host_rows()
    assert np.array_equal(p2, P.astype(np.int32))
    assert np.array_equal(synth.bf16_bits_to_f64(kb2), K)
