"""Pins of the CPU oracle to things other than itself (CPU only).

* a library routine: torch's scaled_dot_product_attention in float64 (GQA
  mapping, scale, softmax over cache + new token, output);
* a pure-Python scalar brute force on tiny caches (tests/brute_force.py);
* closed forms: one query head => evict the lowest exact dot product
  (computed in exact rational arithmetic); uniform keys => evictions cycle
  through slots sink .. sink + window;
* hand-derived cases (tests/golden/hand_cases.json);
* invariants of a whole trajectory and permutation equivariance.

The page-form score (alpha times ||v||_1) has its own pins: the brute force,
a hand case where it and the head-averaged probability disagree, a one-head
closed form in the log domain (exact dot products, no softmax), zero-norm
values, and equal-norm values (where it must rank exactly like the default).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from attention_lf_decode_b200 import synth
from tests.brute_force import brute_row

HERE = os.path.dirname(os.path.abspath(__file__))


def _bf16(rng, shape, scale=1.0):
    return synth.bf16_bits_to_f64(synth.to_bf16_bits(
        (rng.standard_normal(shape) * scale).astype(np.float32)))


def random_state(rng, B, Hq, Hkv, D, N, fill, permute=True):
    """A bf16-exact random cache state: `fill` filled slots with unique
    positions 0..fill-1, scattered over the slots when `permute`."""
    K = _bf16(rng, (B, Hkv, N, D))
    V = _bf16(rng, (B, Hkv, N, D))
    pos = np.full((B, Hkv, N), -1, np.int64)
    for b in range(B):
        for g in range(Hkv):
            slots = rng.permutation(N)[:fill] if permute else np.arange(fill)
            pos[b, g, slots] = np.arange(fill)
    q = _bf16(rng, (B, Hq, D))
    kn = _bf16(rng, (B, Hkv, D))
    vn = _bf16(rng, (B, Hkv, D))
    return K, V, pos, q, kn, vn


def sdpa_reference(K, V, pos, q, kn, vn):
    """torch SDPA (float64, CPU, enable_gqa) over filled slots + new token."""
    B, Hkv, N, D = K.shape
    Hq = q.shape[1]
    out = np.zeros((B, Hq, D))
    for b in range(B):
        # each KV head may have a different filled set: run them one by one
        G = Hq // Hkv
        for g in range(Hkv):
            f = pos[b, g] >= 0
            k = torch.from_numpy(np.concatenate([K[b, g][f], kn[b, g][None]]))[None, None]
            v = torch.from_numpy(np.concatenate([V[b, g][f], vn[b, g][None]]))[None, None]
            qq = torch.from_numpy(q[b, g * G:(g + 1) * G])[None, :, None, :]
            o = F.scaled_dot_product_attention(qq, k, v, enable_gqa=True)
            out[b, g * G:(g + 1) * G] = o[0, :, 0].numpy()
    return out


def sdpa_batched(K, V, q, kn, vn):
    """Same, for a cache whose slots are all filled: one batched SDPA call,
    where torch's own GQA mapping decides which KV head each query head uses."""
    k = torch.from_numpy(np.concatenate([K, kn[:, :, None]], axis=2))
    v = torch.from_numpy(np.concatenate([V, vn[:, :, None]], axis=2))
    qq = torch.from_numpy(q)[:, :, None, :]
    return F.scaled_dot_product_attention(qq, k, v, enable_gqa=True)[:, :, 0].numpy()


# ------------------------------------------------------------------ P1: SDPA

@pytest.mark.parametrize("B,Hq,Hkv,D,N,fill", [
    (2, 4, 2, 8, 12, 12), (1, 8, 2, 64, 40, 17), (3, 3, 3, 16, 9, 0),
    (2, 6, 2, 32, 33, 33), (1, 7, 1, 128, 64, 50)])
def test_output_matches_library_attention(B, Hq, Hkv, D, N, fill):
    rng = np.random.default_rng(100 + N)
    K, V, pos, q, kn, vn = random_state(rng, B, Hq, Hkv, D, N, fill)
    res = oracle.decode_step(K, V, pos, q, kn, vn, sink=1, window=2)
    ref = sdpa_reference(K, V, pos, q, kn, vn)
    np.testing.assert_allclose(res.out, ref, rtol=0, atol=1e-12)
    if fill == N:
        np.testing.assert_allclose(res.out, sdpa_batched(K, V, q, kn, vn), rtol=0, atol=1e-12)
    ctrl = oracle.decode_attention(K, V, pos, q, kn, vn)
    np.testing.assert_allclose(ctrl, ref, rtol=0, atol=1e-12)


def test_no_eviction_while_budget_covers_length():
    """budget >= prefill + steps: append-only cache, evicted == -1, output is
    plain decode attention at every step."""
    rng = np.random.default_rng(7)
    B, Hq, Hkv, D, N, n0, steps = 2, 4, 2, 16, 24, 5, 19
    K, V, pos, _, _, _ = random_state(rng, B, Hq, Hkv, D, N, n0, permute=False)
    for s in range(steps):
        q = _bf16(rng, (B, Hq, D))
        kn = _bf16(rng, (B, Hkv, D))
        vn = _bf16(rng, (B, Hkv, D))
        ref = sdpa_reference(K, V, pos, q, kn, vn)
        res = oracle.decode_step(K, V, pos, q, kn, vn, sink=4, window=3)
        np.testing.assert_allclose(res.out, ref, rtol=0, atol=1e-12)
        assert (res.evicted == -1).all()
        assert (res.pos[..., n0 + s] == n0 + s).all()
        np.testing.assert_array_equal(res.kcache[..., n0 + s, :], kn)
        K, V, pos = res.kcache, res.vcache, res.pos


# ------------------------------------------------------- P2: probabilities

def test_probabilities_sum_to_one():
    rng = np.random.default_rng(3)
    K, V, pos, q, kn, vn = random_state(rng, 2, 8, 2, 64, 300, 300)
    res = oracle.decode_step(K, V, pos, q, kn, vn, sink=4, window=16)
    for r in res.rows:
        tot = r.p.sum(axis=1) + r.p_new
        np.testing.assert_allclose(tot, 1.0, rtol=0, atol=1e-12)
        assert (r.p >= 0).all() and (r.p_new > 0).all()
        np.testing.assert_allclose(r.score, r.p.mean(axis=0), rtol=0, atol=0)


# ------------------------------------------------------- P3: brute force

@pytest.mark.parametrize("seed,score", [(s, "mean_prob") for s in range(40)]
                         + [(s, "alpha_l1v") for s in range(100, 130)])
def test_matches_scalar_brute_force(seed, score):
    rng = np.random.default_rng(seed)
    Hkv = int(rng.integers(1, 3))
    G = int(rng.integers(1, 4))
    D = int(rng.choice([2, 4, 8]))
    N = int(rng.integers(3, 13))
    sink = int(rng.integers(0, 3))
    window = int(rng.integers(1, 4))
    fill = N if seed % 3 else int(rng.integers(0, N + 1))
    if fill == N and N <= sink + window:
        N = sink + window + 2
        fill = N
    K, V, pos, q, kn, vn = random_state(rng, 1, G * Hkv, Hkv, D, N, fill)
    res = oracle.decode_step(K, V, pos, q, kn, vn, sink, window, score=score)
    for g in range(Hkv):
        out, ev, slot, t = brute_row(K[0, g].tolist(), V[0, g].tolist(), pos[0, g].tolist(),
                                     q[0, g * G:(g + 1) * G].tolist(), kn[0, g].tolist(),
                                     vn[0, g].tolist(), sink, window, score=score)
        assert res.evicted[0, g] == ev
        assert res.rows[g].slot == slot and res.rows[g].t == t
        np.testing.assert_allclose(res.out[0, g * G:(g + 1) * G], np.array(out),
                                   rtol=0, atol=1e-12)
        # new state: exactly one slot changed, to the new token
        changed = np.flatnonzero((res.pos[0, g] != pos[0, g]))
        assert changed.tolist() == [slot]
        assert res.pos[0, g, slot] == t
        np.testing.assert_array_equal(res.kcache[0, g, slot], kn[0, g])
        np.testing.assert_array_equal(res.vcache[0, g, slot], vn[0, g])
        others = np.arange(N) != slot
        np.testing.assert_array_equal(res.kcache[0, g][others], K[0, g][others])


# ------------------------------------------------ P4: one head, exact dot

def _exact_dot(a, b):
    return sum(Fraction(float(x)) * Fraction(float(y)) for x, y in zip(a, b))


@pytest.mark.parametrize("seed", range(12))
def test_single_head_evicts_lowest_exact_dot(seed):
    """G = 1: the softmax is monotone, so the evicted slot is the candidate
    with the lowest exact dot product q.K_j (lowest index among equals)."""
    rng = np.random.default_rng(1000 + seed)
    N, D, sink, window = 48, 16, 4, 8
    K, V, pos, q, kn, vn = random_state(rng, 1, 1, 1, D, N, N)
    if seed % 2:  # plant exact duplicates of the best keys to exercise ties
        K[0, 0, 20] = K[0, 0, 30] = K[0, 0, 40] = -np.abs(K[0, 0, 20])
    res = oracle.decode_step(K, V, pos, q, kn, vn, sink, window)
    t = int(pos.max()) + 1
    best = None
    for j in range(N):
        if j < sink or pos[0, 0, j] >= t - window:
            continue
        d = _exact_dot(q[0, 0], K[0, 0, j])
        if best is None or d < best[0]:
            best = (d, j)
    assert res.evicted[0, 0] == best[1]


# ------------------------------------------- P5: uniform keys, closed form

@pytest.mark.parametrize("N,sink,window,G", [(32, 4, 6, 1), (20, 0, 1, 2), (64, 4, 16, 4)])
def test_uniform_keys_evict_in_a_cycle(N, sink, window, G):
    """All keys equal => all scores equal => the lowest candidate slot goes.
    From a full prefill (slot j at position j), step k evicts slot
    sink + (k mod (window + 1)): the slot refilled at step k - window - 1 is
    the first to leave the window again."""
    rng = np.random.default_rng(5)
    D = 8
    k0 = _bf16(rng, (D,))
    K = np.broadcast_to(k0, (1, 1, N, D)).copy()
    V = _bf16(rng, (1, 1, N, D))
    pos = np.arange(N)[None, None].astype(np.int64)
    for k in range(3 * (window + 1) + 2):
        q = _bf16(rng, (1, G, D))
        vn = _bf16(rng, (1, 1, D))
        res = oracle.decode_step(K, V, pos, q, k0[None, None], vn, sink, window)
        assert res.evicted[0, 0] == sink + (k % (window + 1)), k
        K, V, pos = res.kcache, res.vcache, res.pos


# --------------------------------------------------- hand-derived cases

def test_hand_cases():
    with open(os.path.join(HERE, "golden", "hand_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        K = np.array(c["K"], float)[None, None]
        V = np.array(c["V"], float)[None, None]
        pos = np.array(c["pos"])[None, None]
        q = np.array(c["q"], float)[None]
        kn = np.array(c["k_new"], float)[None, None]
        vn = np.array(c["v_new"], float)[None, None]
        res = oracle.decode_step(K, V, pos, q, kn, vn, c["sink"], c["window"],
                                 score=c.get("score", "mean_prob"))
        exp = c["expected"]
        r = res.rows[0]
        assert (res.evicted[0, 0], r.slot, r.t) == (exp["evicted"], exp["slot"], exp["t"]), c["name"]
        assert res.pos[0, 0, exp["slot"]] == exp["t"]
        if "out" in exp:
            np.testing.assert_array_equal(res.out[0], np.array(exp["out"]))


# ------------------------------------------- P6: trajectory invariants

def test_trajectory_invariants():
    cfg = synth.CONFIGS["tiny"].with_(budget=64, prefill=64, window=8, steps=160)
    gen = synth.SynthDecode(cfg)
    kb, vb = gen.prefill()
    kc, vc, pos = synth.prefill_layout(kb, vb, cfg.budget)
    K, V = synth.bf16_bits_to_f64(kc), synth.bf16_bits_to_f64(vc)
    pos = pos.astype(np.int64)
    sink_k = K[..., :cfg.sink, :].copy()
    for s, (qb, knb, vnb) in gen.iter_steps():
        q, kn, vn = (synth.bf16_bits_to_f64(x) for x in (qb, knb, vnb))
        res = oracle.decode_step(K, V, pos, q, kn, vn, cfg.sink, cfg.window)
        t = cfg.prefill + s
        for b in range(cfg.batch):
            for g in range(cfg.hkv):
                r = res.rows[b * cfg.hkv + g]
                assert r.t == t
                e = res.evicted[b, g]
                assert e >= cfg.sink and pos[b, g, e] < t - cfg.window
                p_after = res.pos[b, g]
                assert len(set(p_after.tolist())) == cfg.budget  # unique
                assert set(range(t - cfg.window, t + 1)) <= set(p_after.tolist())
        np.testing.assert_array_equal(res.kcache[..., :cfg.sink, :], sink_k)
        assert (res.pos[..., :cfg.sink] == np.arange(cfg.sink)).all()
        K, V, pos = res.kcache, res.vcache, res.pos


# ------------------------------------- P7: permutation equivariance

@pytest.mark.parametrize("seed", range(6))
def test_permutation_equivariance(seed):
    """Shuffling non-sink slots (K, V and pos together) moves the evicted
    slot with them and leaves the output unchanged."""
    rng = np.random.default_rng(200 + seed)
    B, Hq, Hkv, D, N, sink, window = 1, 4, 2, 16, 40, 4, 6
    K, V, pos, q, kn, vn = random_state(rng, B, Hq, Hkv, D, N, N, permute=False)
    res = oracle.decode_step(K, V, pos, q, kn, vn, sink, window)
    perm = np.concatenate([np.arange(sink), sink + rng.permutation(N - sink)])
    inv = np.argsort(perm)
    res2 = oracle.decode_step(K[..., perm, :], V[..., perm, :], pos[..., perm],
                              q, kn, vn, sink, window)
    np.testing.assert_allclose(res2.out, res.out, rtol=0, atol=1e-12)
    for g in range(Hkv):
        e, e2 = res.evicted[0, g], res2.evicted[0, g]
        sc = res.rows[g].score
        order = np.sort(sc[res.rows[g].candidates])
        if order[1] - order[0] > 1e-9 * order[0]:  # no near tie
            assert inv[e] == e2


# ------------------------------------------------------------ generator

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 7,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 1e-30], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(synth.to_bf16_bits(x), ref)
    back = synth.bf16_bits_to_f32(ref)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(
        torch.bfloat16).float().numpy())


def test_generator_rows_and_steps_regenerate():
    cfg = synth.CONFIGS["tiny"].with_(batch=3)
    g1, g2 = synth.SynthDecode(cfg), synth.SynthDecode(cfg)
    k_all, v_all = g1.prefill()
    k_sub, v_sub = g2.prefill([2])
    np.testing.assert_array_equal(k_all[2:3], k_sub)
    np.testing.assert_array_equal(v_all[2:3], v_sub)
    a = g1.step_inputs(5)
    b = g2.step_inputs(5)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    # AR(1) queries: in-order and restarted draws agree
    ar = synth.CONFIGS["long_reasoning"].with_(batch=1, budget=64, prefill=64)
    g3, g4 = synth.SynthDecode(ar), synth.SynthDecode(ar)
    seq = [g3.step_inputs(s)[0] for s in range(4)]
    np.testing.assert_array_equal(g4.step_inputs(3)[0], seq[3])
    np.testing.assert_array_equal(g4.step_inputs(1)[0], seq[1])


def test_generator_outlier_structure():
    """About frac of the prefill keys carry the +mag*u outlier: their
    projection on u is far above the N(0,1) bulk."""
    cfg = synth.CONFIGS["throughput"].with_(batch=1, budget=4096)
    gen = synth.SynthDecode(cfg)
    k, _ = gen.prefill_row(0)
    proj = synth.bf16_bits_to_f64(k) @ gen.u.astype(np.float64)
    frac = np.mean(proj > 2.0)
    assert 0.01 < frac < 0.05
    q, _, _ = gen.step_inputs(0)
    qp = synth.bf16_bits_to_f64(q) @ gen.u.astype(np.float64)
    assert abs(qp.mean() - 1.0) < 0.2


def test_prefill_rejects_over_budget():
    with pytest.raises(ValueError):
        oracle.prefill(np.zeros((1, 1, 5, 4)), np.zeros((1, 1, 5, 4)), 5, 4)
    kc, vc, pos = oracle.prefill(np.ones((1, 1, 3, 4)), np.ones((1, 1, 3, 4)), 3, 6)
    assert pos.tolist() == [[[0, 1, 2, -1, -1, -1]]]


# ------------------------------------- the page-form score alpha * ||v||_1

@pytest.mark.parametrize("seed", range(12))
def test_page_score_single_head_log_domain(seed):
    """G = 1: p_j = e^(s_j - m) / l with the same m and l for every slot, so
    the page score p_j * ||v_j||_1 is lowest where s_j + ln ||v_j||_1 is
    lowest.  s_j is an exact rational dot product; only the log is rounded."""
    rng = np.random.default_rng(2000 + seed)
    N, D, sink, window = 40, 16, 4, 8
    K, V, pos, q, kn, vn = random_state(rng, 1, 1, 1, D, N, N)
    V[0, 0] *= np.exp2(rng.integers(-3, 4, size=(N, 1)))  # spread the norms (exact in bf16)
    res = oracle.decode_step(K, V, pos, q, kn, vn, sink, window, score="alpha_l1v")
    t = int(pos.max()) + 1
    scale = 1.0 / math.sqrt(D)
    keyed = []
    for j in range(N):
        if j < sink or pos[0, 0, j] >= t - window:
            continue
        l1 = sum(Fraction(abs(float(x))) for x in V[0, 0, j])
        keyed.append((float(_exact_dot(q[0, 0], K[0, 0, j])) * scale + math.log(float(l1)), j))
    keyed.sort()
    assert keyed[1][0] - keyed[0][0] > 1e-9  # no near tie in these draws
    assert res.evicted[0, 0] == keyed[0][1]


def test_page_score_zero_norm_values_go_first():
    """A candidate whose value vector is all zeros scores exactly 0: the
    lowest-index such candidate is evicted, whatever its probability."""
    rng = np.random.default_rng(77)
    N, D, sink, window = 24, 8, 2, 4
    K, V, pos, q, kn, vn = random_state(rng, 1, 3, 1, D, N, N, permute=False)
    V[0, 0, [1, 9, 14]] = 0.0   # slot 1 is a sink and may not go
    K[0, 0, 14] = -K[0, 0, 14]  # whatever the logits
    res = oracle.decode_step(K, V, pos, q, kn, vn, sink, window, score="alpha_l1v")
    assert res.evicted[0, 0] == 9
    assert res.rows[0].score[9] == 0.0 and res.rows[0].score[14] == 0.0


def test_page_score_equal_norms_rank_like_mean_prob():
    """With every ||v_j||_1 equal (values are signed permutations of one
    vector) the two scores differ by one common factor, so a whole
    trajectory evicts the same slots under both."""
    rng = np.random.default_rng(78)
    N, D, sink, window, G = 32, 8, 4, 6, 4
    base = _bf16(rng, (D,))

    def signed_perm():
        return base[rng.permutation(D)] * rng.choice([-1.0, 1.0], size=D)

    K = _bf16(rng, (1, 1, N, D))
    V = np.stack([signed_perm() for _ in range(N)])[None, None]
    pos = np.arange(N)[None, None].astype(np.int64)
    Ka, Va, pa = K, V, pos
    for k in range(60):
        q = _bf16(rng, (1, G, D))
        kn = _bf16(rng, (1, 1, D))
        vn = signed_perm()[None, None]
        ra = oracle.decode_step(Ka, Va, pa, q, kn, vn, sink, window, score="alpha_l1v")
        rb = oracle.decode_step(Ka, Va, pa, q, kn, vn, sink, window, score="mean_prob")
        assert ra.evicted[0, 0] == rb.evicted[0, 0], k
        np.testing.assert_array_equal(ra.out, rb.out)
        Ka, Va, pa = ra.kcache, ra.vcache, ra.pos


def test_unknown_score_is_rejected():
    rng = np.random.default_rng(3)
    K, V, pos, q, kn, vn = random_state(rng, 1, 2, 1, 4, 8, 8)
    with pytest.raises(ValueError):
        oracle.decode_step(K, V, pos, q, kn, vn, 1, 2, score="l2")


# ------------------------------------------ ragged batches (per-sequence budget)

def _ragged_state(rng, B, Hq, Hkv, D, N, sink, window):
    """Per batch entry b a budget n_b; slots 0..n_b-1 hold a cache that is
    full or partly free; the slots beyond hold junk that must be ignored:
    NaN values and positions far above the prefix's."""
    K, V, pos, q, kn, vn = random_state(rng, B, Hq, Hkv, D, N, N)
    nb = rng.integers(sink + window + 1, N + 1, size=B)
    for b in range(B):
        n = int(nb[b])
        full = rng.random() < 0.7
        fill = n if full else int(rng.integers(0, n))
        for g in range(Hkv):
            pos[b, g, :n] = -1
            slots = rng.permutation(n)[:fill]
            pos[b, g, slots] = rng.permutation(fill) + int(rng.integers(0, 50))
            pos[b, g, n:] = 10_000 + np.arange(N - n)
            K[b, g, n:] = np.nan
            V[b, g, n:] = np.nan
    return K, V, pos, q, kn, vn, nb


@pytest.mark.parametrize("seed", range(24))
def test_ragged_matches_brute_force(seed):
    rng = np.random.default_rng(3000 + seed)
    B, Hkv, G = 3, int(rng.integers(1, 3)), int(rng.integers(1, 4))
    D, N, sink, window = int(rng.choice([2, 4, 8])), int(rng.integers(8, 15)), 1, 2
    score = "alpha_l1v" if seed % 2 else "mean_prob"
    K, V, pos, q, kn, vn, nb = _ragged_state(rng, B, G * Hkv, Hkv, D, N, sink, window)
    res = oracle.decode_step(K, V, pos, q, kn, vn, sink, window, score=score, seq_budget=nb)
    for b in range(B):
        n = int(nb[b])
        for g in range(Hkv):
            out, ev, slot, t = brute_row(K[b, g, :n].tolist(), V[b, g, :n].tolist(),
                                         pos[b, g, :n].tolist(),
                                         q[b, g * G:(g + 1) * G].tolist(), kn[b, g].tolist(),
                                         vn[b, g].tolist(), sink, window, score=score)
            assert res.evicted[b, g] == ev and res.rows[b * Hkv + g].t == t
            np.testing.assert_allclose(res.out[b, g * G:(g + 1) * G], np.array(out),
                                       rtol=0, atol=1e-12)
            assert res.pos[b, g, slot] == t
            # the junk beyond the budget is untouched (NaN stays NaN)
            np.testing.assert_array_equal(res.pos[b, g, n:], pos[b, g, n:])
            assert np.isnan(res.kcache[b, g, n:]).all() and np.isnan(res.vcache[b, g, n:]).all()


def test_ragged_outputs_match_library_attention():
    rng = np.random.default_rng(3100)
    B, Hq, Hkv, D, N = 4, 8, 2, 16, 40
    K, V, pos, q, kn, vn, nb = _ragged_state(rng, B, Hq, Hkv, D, N, 2, 4)
    res = oracle.decode_step(K, V, pos, q, kn, vn, 2, 4, seq_budget=nb)
    att = oracle.decode_attention(K, V, pos, q, kn, vn, seq_budget=nb)
    for b in range(B):
        n = int(nb[b])
        ref = sdpa_reference(K[b:b + 1, :, :n], V[b:b + 1, :, :n], pos[b:b + 1, :, :n],
                             q[b:b + 1], kn[b:b + 1], vn[b:b + 1])
        np.testing.assert_allclose(res.out[b:b + 1], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(att[b:b + 1], ref, rtol=0, atol=1e-12)
    assert not np.isnan(res.out).any()


def test_ragged_budget_equal_to_slots_is_the_plain_step():
    rng = np.random.default_rng(3200)
    K, V, pos, q, kn, vn = random_state(rng, 3, 6, 2, 8, 20, 20)
    a = oracle.decode_step(K, V, pos, q, kn, vn, 2, 3)
    b = oracle.decode_step(K, V, pos, q, kn, vn, 2, 3, seq_budget=[20, 20, 20])
    np.testing.assert_array_equal(a.out, b.out)
    np.testing.assert_array_equal(a.evicted, b.evicted)
    np.testing.assert_array_equal(a.pos, b.pos)


@pytest.mark.parametrize("nb", [[0, 5], [5, 21], [5]])
def test_ragged_budget_validation(nb):
    rng = np.random.default_rng(3300)
    K, V, pos, q, kn, vn = random_state(rng, 2, 2, 1, 4, 20, 20)
    with pytest.raises(ValueError):
        oracle.decode_step(K, V, pos, q, kn, vn, 1, 2, seq_budget=nb)
