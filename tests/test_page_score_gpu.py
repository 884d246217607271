"""GPU parity of the page-form eviction score (attention weight times the L1
norm of the value vector, LongFlow summary page §2B) against the oracle's
``score="alpha_l1v"``.

Teacher-forced runs on the configured workloads (full sizes on sampled
rows), ragged budgets under every split, group sizes and head dims, and the
degenerate cases of this score: zero-norm values (score exactly 0, lowest
slot first), equal keys with equal-norm values (every score ties: the
evictions cycle through sink .. sink + window), and switching the score
between steps on one handle.
"""
import numpy as np
import pytest

import oracle
from attention_lf_decode_b200 import binding, synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu
L1V = "alpha_l1v"


@pytest.fixture(autouse=True)
def _cuda(cuda_ok):
    binding.load_library()


def _bits(rng, shape, scale=1.0):
    return synth.to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _custom(B, Hq, Hkv, D, N, sink, window, seed=0, **kw):
    return synth.DecodeConfig("custom", batch=B, hq=Hq, hkv=Hkv, head_dim=D, budget=N,
                              sink=sink, window=window, prefill=N, steps=8, seed=seed, **kw)


def test_tiny_all_steps():
    st = H.teacher_forced(synth.CONFIGS["tiny"], steps=64, score=L1V)
    assert st.exact_evictions + st.accepted_ties == 64 * 2


def test_throughput_full_size_sampled_rows():
    cfg = synth.CONFIGS["throughput"]
    st = H.teacher_forced(cfg, steps=3, batch_idx=[1, 40, 63], score=L1V)
    assert st.rows == 3 * 3 * 8


def test_llama3_8b_shape_all_rows():
    st = H.teacher_forced(synth.CONFIGS["llama3_8b"], steps=8, score=L1V)
    assert st.rows == 8 * 64


def test_long_reasoning_g7_sampled_rows():
    st = H.teacher_forced(synth.CONFIGS["long_reasoning"], steps=4, batch_idx=[3], score=L1V)
    assert st.rows == 4 * 4


@pytest.mark.parametrize("N", [301, 1000])
@pytest.mark.parametrize("split", [1, 2, 4, 8, 16])
def test_ragged_budgets_every_split(N, split):
    H.teacher_forced(_custom(2, 8, 2, 128, N, 4, 8, seed=N + 7), steps=3, split=split, score=L1V)


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 4, 128), (7, 1, 128), (8, 1, 64), (6, 2, 64),
                                      (24, 8, 128), (3, 1, 128)])
def test_group_sizes_and_head_dims(Hq, Hkv, D):
    H.teacher_forced(_custom(3, Hq, Hkv, D, 520, 4, 16, seed=Hq * 10 + D + 1), steps=4, score=L1V)


def test_budget_covers_length_appends_then_evicts():
    cfg = _custom(2, 8, 2, 128, 48, 4, 8, seed=31).with_(prefill=40)
    st = H.teacher_forced(cfg, steps=14, score=L1V)
    assert st.appends == 8 * 4


def test_zero_norm_values_are_evicted_first():
    """Value rows of zeros score exactly 0 whatever their attention weight:
    the lowest such candidate goes first (zeroed rows are refilled with
    nonzero values, so the next one goes at the following step)."""
    rng = np.random.default_rng(41)
    B, Hq, Hkv, D, N, sink, window = 2, 8, 2, 128, 400, 4, 16
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=41)
    kb = _bits(rng, (B, Hkv, N, D))
    vb = _bits(rng, (B, Hkv, N, D))
    zero_slots = [2, 57, 58, 203, 390]  # 2 is a sink, 390 is inside the window
    vb[:, :, zero_slots] = 0
    pos = np.broadcast_to(np.arange(N, dtype=np.int32), (B, Hkv, N)).copy()
    g_ = H.GpuCache(cfg, n=0, score=L1V)
    g_.set_state(kb, vb, pos)
    stats = H.Stats()
    for s in range(5):
        qb, knb, vnb = _bits(rng, (B, Hq, D)), _bits(rng, (B, Hkv, D)), _bits(rng, (B, Hkv, D))
        g_.step(qb, knb, vnb)
        res = oracle.decode_step(*H.oracle_state(kb, vb, pos), synth.bf16_bits_to_f64(qb),
                                 synth.bf16_bits_to_f64(knb), synth.bf16_bits_to_f64(vnb),
                                 sink, window, score=L1V)
        gpu = g_.host_rows()
        if s < 3:
            assert (gpu[1] == [57, 58, 203][s]).all(), (s, gpu[1])
        kb, vb, pos = H.check_step(res, pos, gpu, stats, kb, vb, knb, vnb, f"s{s}")
    assert H.binding.lf_get_status(g_.h) == binding.LF_OK


@pytest.mark.parametrize("N,sink,window,G", [(64, 4, 6, 1), (256, 4, 16, 4), (1000, 4, 32, 7)])
def test_equal_keys_equal_norms_cycle(N, sink, window, G):
    """Equal keys and values of one L1 norm (signed permutations of one
    vector): every page score ties, the fp64 rescoring runs on every
    candidate, and the evictions cycle through slots sink..sink+window."""
    rng = np.random.default_rng(N + 1)
    D = 128
    cfg = _custom(2, 2 * G, 2, D, N, sink, window, seed=N)
    k0 = _bits(rng, (2, 2, 1, D))
    base = synth.bf16_bits_to_f64(_bits(rng, (D,)))

    def signed_perms(n):
        rows = [base[rng.permutation(D)] * rng.choice([-1.0, 1.0], size=D) for _ in range(n)]
        return synth.to_bf16_bits(np.array(rows, np.float32))

    kb = np.broadcast_to(k0, (2, 2, N, D)).copy()
    vb = signed_perms(4 * N).reshape(2, 2, N, D)
    pos = np.broadcast_to(np.arange(N, dtype=np.int32), (2, 2, N)).copy()
    g_ = H.GpuCache(cfg, n=0, score=L1V)
    g_.set_state(kb, vb, pos)
    for k in range(2 * (window + 1) + 3):
        qb = _bits(rng, (2, 2 * G, D))
        vnb = signed_perms(4).reshape(2, 2, D)
        g_.step(qb, k0[:, :, 0], vnb)
        _, ev, _, _, _ = g_.host_rows()
        assert (ev == sink + (k % (window + 1))).all(), (k, ev)


def test_switching_score_between_steps():
    """One handle, the score switched every step: each step matches the
    oracle under the score it ran with."""
    rng = np.random.default_rng(51)
    B, Hq, Hkv, D, N, sink, window = 2, 8, 2, 128, 700, 4, 32
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=51)
    kb = _bits(rng, (B, Hkv, N, D))
    # spread the value norms so that the two scores often disagree
    vf = synth.bf16_bits_to_f64(_bits(rng, (B, Hkv, N, D)))
    vb = synth.to_bf16_bits((vf * np.exp2(rng.integers(-4, 5, size=(B, Hkv, N, 1)))).astype(np.float32))
    pos = np.broadcast_to(np.arange(N, dtype=np.int32), (B, Hkv, N)).copy()
    g_ = H.GpuCache(cfg, n=0)
    g_.set_state(kb, vb, pos)
    stats = H.Stats()
    differ = 0
    for s in range(12):
        score = L1V if s % 2 else "mean_prob"
        binding.lf_set_score(g_.h, H.SCORE_CODES[score])
        assert binding.lf_get_score(g_.h) == H.SCORE_CODES[score]
        qb, knb, vnb = _bits(rng, (B, Hq, D)), _bits(rng, (B, Hkv, D)), _bits(rng, (B, Hkv, D))
        g_.step(qb, knb, vnb)
        args = (*H.oracle_state(kb, vb, pos), synth.bf16_bits_to_f64(qb),
                synth.bf16_bits_to_f64(knb), synth.bf16_bits_to_f64(vnb), sink, window)
        res = oracle.decode_step(*args, score=score)
        other = oracle.decode_step(*args, score="mean_prob" if s % 2 else L1V)
        differ += int((res.evicted != other.evicted).sum())
        kb, vb, pos = H.check_step(res, pos, g_.host_rows(), stats, kb, vb, knb, vnb, f"s{s}")
    assert differ > 0  # the test would not notice a score that is ignored


def test_invalid_score_rejected():
    h = binding.lf_init(1, 4, 2, 128, 256)
    try:
        lib = binding.load_library()
        assert lib.lf_set_score(h.ptr, 2) == binding.LF_EINVAL
        assert lib.lf_set_score(h.ptr, -1) == binding.LF_EINVAL
        assert binding.lf_get_score(h) == binding.LF_SCORE_MEAN_PROB
        binding.lf_set_score(h, binding.LF_SCORE_ALPHA_L1V)
        assert binding.lf_get_score(h) == binding.LF_SCORE_ALPHA_L1V
    finally:
        binding.lf_destroy(h)
