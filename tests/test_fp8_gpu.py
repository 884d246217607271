"""GPU parity of the E4M3 (FP8) KV cache against oracle/kvfp8.py:
lf_prefill_cache_fp8, lf_decode_step_fp8 (plain and ragged) and
lf_decode_attention_fp8.

The stored codes are compared bit for bit: the prefill's, and after every
step the new token's codes in the chosen slot (fp32 quotient by the scale,
round to nearest even, saturation).  Outputs within the usual 2e-3; the
evicted slot exact except oracle near ties.  Covered: the configured
workloads at full size on sampled rows, every split, both scores, group
sizes and head dims, non-unit scales, saturating values, equal keys (every
score ties: fp64 rescoring from E4M3 codes), a ragged batch, attention only,
and the host checks of the scales.
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


def _bits(rng, shape, scale=1.0):
    return synth.to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _f64(bits):
    return synth.bf16_bits_to_f64(bits)


def _custom(B, Hq, Hkv, D, N, sink, window, seed=0, **kw):
    return synth.DecodeConfig("custom", batch=B, hq=Hq, hkv=Hkv, head_dim=D, budget=N,
                              sink=sink, window=window, prefill=N, steps=8, seed=seed, **kw)


class Fp8Cache:
    """An E4M3 cache on the device, driven through the C ABI."""

    def __init__(self, cfg, ks, vs, split=0, score="mean_prob", seq_budget=None):
        import torch
        self.torch, self.cfg, self.ks, self.vs = torch, cfg, ks, vs
        c = cfg
        self.h = binding.lf_init(c.batch, c.hq, c.hkv, c.head_dim, c.budget)
        if split:
            binding.lf_set_split(self.h, split)
        binding.lf_set_score(self.h, H.SCORE_CODES[score])
        shape = (c.batch, c.hkv, c.budget, c.head_dim)
        self.kcache = torch.zeros(shape, dtype=torch.uint8, device="cuda")
        self.vcache = torch.zeros(shape, dtype=torch.uint8, device="cuda")
        self.pos = torch.full(shape[:3], -1, dtype=torch.int32, device="cuda")
        self.out = torch.empty((c.batch, c.hq, c.head_dim), dtype=torch.float32, device="cuda")
        self.evicted = torch.empty((c.batch, c.hkv), dtype=torch.int32, device="cuda")
        self.nb = None if seq_budget is None else torch.from_numpy(np.asarray(seq_budget, np.int32)).cuda()

    def prefill(self, kbits, vbits, n):
        k = binding.bf16_from_bits(kbits) if n else None
        v = binding.bf16_from_bits(vbits) if n else None
        binding.lf_prefill_cache_fp8(self.h, k, v, n, self.kcache, self.vcache, self.pos,
                                     self.cfg.budget, self.ks, self.vs)

    def set_state(self, kc, vc, pos):
        t = self.torch
        self.kcache.copy_(t.from_numpy(np.ascontiguousarray(kc, np.uint8)))
        self.vcache.copy_(t.from_numpy(np.ascontiguousarray(vc, np.uint8)))
        self.pos.copy_(t.from_numpy(np.ascontiguousarray(pos, np.int32)))

    def step(self, qb, knb, vnb, attention_only=False):
        c = self.cfg
        q, kn, vn = (binding.bf16_from_bits(x) for x in (qb, knb, vnb))
        if attention_only:
            binding.lf_decode_attention_fp8(self.h, q, kn, vn, self.kcache, self.vcache, self.pos,
                                            c.budget, self.ks, self.vs, self.out, self.nb)
        else:
            binding.lf_decode_step_fp8(self.h, q, kn, vn, self.kcache, self.vcache, self.pos,
                                       c.budget, c.sink, c.window, self.ks, self.vs, self.out,
                                       self.evicted, self.nb)

    def host_rows(self, sel=None):
        t = self.torch
        t.cuda.synchronize()
        arrs = (self.out, self.evicted, self.kcache, self.vcache, self.pos)
        if sel is not None:
            idx = t.tensor(list(sel), device="cuda")
            arrs = tuple(a.index_select(0, idx) for a in arrs)
        return tuple(a.cpu().numpy() for a in arrs)

    def status(self):
        return binding.lf_get_status(self.h), binding.lf_status_bits(self.h)


def run_steps(c, cfg, kc, vc, pos, steps, rng, sel=None, gen=None, score="mean_prob",
              seq_budget=None, key_scale=1.0):
    """Teacher-forced steps; the oracle runs on the rows of `sel` (all if None)."""
    stats = H.Stats()
    B, Hq, Hkv, D = cfg.batch, cfg.hq, cfg.hkv, cfg.head_dim
    bs = list(range(B)) if sel is None else list(sel)
    nb = None if seq_budget is None else np.asarray(seq_budget)[bs]
    for s in range(steps):
        if gen is not None:
            qb, knb, vnb = gen.step_inputs(s)
        else:
            qb, knb, vnb = (_bits(rng, (B, Hq, D)), _bits(rng, (B, Hkv, D), key_scale),
                            _bits(rng, (B, Hkv, D)))
        c.step(qb, knb, vnb)
        res = oracle.decode_step_fp8(kc, vc, pos, _f64(qb[bs]), _f64(knb[bs]), _f64(vnb[bs]),
                                     cfg.sink, cfg.window, c.ks, c.vs, score=score, seq_budget=nb)
        kq = oracle.quantize(_f64(knb[bs]), c.ks)
        vq = oracle.quantize(_f64(vnb[bs]), c.vs)
        kc, vc, pos = H.check_step(res, pos, c.host_rows(sel), stats, kc, vc, kq, vq, f"s{s}")
    code, bits = c.status()
    assert code == binding.LF_OK, bits
    return stats


def _prefilled(cfg, ks, vs, rng, n=None, **kw):
    n = cfg.prefill if n is None else n
    kb = _bits(rng, (cfg.batch, cfg.hkv, n, cfg.head_dim))
    vb = _bits(rng, (cfg.batch, cfg.hkv, n, cfg.head_dim))
    c = Fp8Cache(cfg, ks, vs, **kw)
    c.prefill(kb, vb, n)
    kc, vc, pos = oracle.prefill_fp8(_f64(kb), _f64(vb), n, cfg.budget, ks, vs)
    return c, kc, vc, pos.astype(np.int32)


def test_prefill_codes_bit_exact():
    rng = np.random.default_rng(1)
    cfg = _custom(3, 8, 2, 128, 300, 4, 8)
    c, kc, vc, pos = _prefilled(cfg, 0.37, 2.5, rng, n=257)
    _, _, gk, gv, gp = c.host_rows()
    assert np.array_equal(gk, kc) and np.array_equal(gv, vc) and np.array_equal(gp, pos)


@pytest.mark.parametrize("ks,vs", [(1.0, 1.0), (0.5, 1.5), (0.0625, 3.0)])
def test_tiny_all_steps(ks, vs):
    cfg = synth.CONFIGS["tiny"]
    rng = np.random.default_rng(2)
    c, kc, vc, pos = _prefilled(cfg, ks, vs, rng)
    st = run_steps(c, cfg, kc, vc, pos, 48, rng)
    assert st.exact_evictions + st.accepted_ties == 48 * 2


def test_throughput_full_size_sampled_rows():
    cfg = synth.CONFIGS["throughput"]
    gen = synth.SynthDecode(cfg)
    kpre, vpre = gen.prefill()
    c = Fp8Cache(cfg, 1.0, 1.0)
    c.prefill(kpre, vpre, cfg.prefill)
    sel = [0, 33, 63]
    kc, vc, pos = oracle.prefill_fp8(_f64(kpre[sel]), _f64(vpre[sel]), cfg.prefill, cfg.budget, 1.0, 1.0)
    del kpre, vpre
    st = run_steps(c, cfg, kc, vc, pos.astype(np.int32), 3, None, sel=sel, gen=gen)
    assert st.rows == 3 * 3 * 8


@pytest.mark.parametrize("split", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("score", ["mean_prob", "alpha_l1v"])
def test_every_split_both_scores(split, score):
    rng = np.random.default_rng(10 + split)
    cfg = _custom(2, 8, 2, 128, 1000, 4, 8, seed=split)
    c, kc, vc, pos = _prefilled(cfg, 0.75, 1.25, rng, split=split, score=score)
    run_steps(c, cfg, kc, vc, pos, 3, rng, score=score)


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 4, 64), (7, 1, 128), (8, 1, 64), (6, 2, 64),
                                      (24, 8, 128), (3, 1, 128)])
def test_group_sizes_and_head_dims(Hq, Hkv, D):
    rng = np.random.default_rng(Hq * 7 + D)
    cfg = _custom(3, Hq, Hkv, D, 520, 4, 16, seed=Hq)
    c, kc, vc, pos = _prefilled(cfg, 0.5, 0.5, rng)
    run_steps(c, cfg, kc, vc, pos, 4, rng)


def test_appends_across_the_tile_tail():
    """E4M3 tiles hold 352 slots at D = 128: the filled prefix grows across
    slots 320..351 of the first tile while the rest stays free."""
    rng = np.random.default_rng(21)
    cfg = _custom(2, 8, 2, 128, 700, 4, 8, seed=21)
    c, kc, vc, pos = _prefilled(cfg, 1.0, 1.0, rng, n=310, split=1)
    st = run_steps(c, cfg, kc, vc, pos, 50, rng)
    assert st.appends == 50 * 4


def test_appends_then_evicts_and_saturating_values():
    """Prefill 40 of 48 slots; new keys 300x larger than the key scale
    allows, and a value scale of 1/256 (values beyond +-1.75 saturate), so
    both caches get saturated codes (+-448) while outputs stay O(1)."""
    rng = np.random.default_rng(5)
    cfg = _custom(2, 8, 2, 128, 48, 4, 8, seed=5)
    c, kc, vc, pos = _prefilled(cfg, 1.0, 1.0 / 256, rng, n=40)
    st = run_steps(c, cfg, kc, vc, pos, 12, rng, key_scale=300.0)
    assert st.appends == 8 * 4
    _, _, gk, gv, _ = c.host_rows()
    assert ((gk & 0x7F) == 0x7E).any() and ((gv & 0x7F) == 0x7E).any()


@pytest.mark.parametrize("score", ["mean_prob", "alpha_l1v"])
def test_equal_keys_cycle(score):
    """Every key holds the same codes and every value the same codes: all
    scores tie, and the evictions cycle through sink .. sink + window."""
    rng = np.random.default_rng(6)
    N, sink, window, D = 300, 4, 16, 128
    cfg = _custom(2, 8, 2, D, N, sink, window, seed=6)
    k0 = oracle.quantize(_f64(_bits(rng, (D,))), 1.0)
    v0 = oracle.quantize(_f64(_bits(rng, (D,))), 1.0)
    kc = np.broadcast_to(k0, (2, 2, N, D)).copy()
    vc = np.broadcast_to(v0, (2, 2, N, D)).copy()
    pos = np.broadcast_to(np.arange(N, dtype=np.int32), (2, 2, N)).copy()
    c = Fp8Cache(cfg, 1.0, 1.0, score=score)
    c.set_state(kc, vc, pos)
    kn = synth.to_bf16_bits(oracle.e4m3_decode(k0).astype(np.float32))
    vn = synth.to_bf16_bits(oracle.e4m3_decode(v0).astype(np.float32))
    for k in range(2 * (window + 1) + 3):
        qb = _bits(rng, (2, 8, D))
        c.step(qb, np.broadcast_to(kn, (2, 2, D)).copy(), np.broadcast_to(vn, (2, 2, D)).copy())
        ev = c.host_rows()[1]
        assert (ev == sink + (k % (window + 1))).all(), (k, ev)


def test_ragged_fp8():
    rng = np.random.default_rng(7)
    B, Hq, Hkv, D, N, sink, window = 6, 8, 2, 128, 800, 4, 8
    nb = rng.integers(sink + window + 1, N + 1, size=B)
    cfg = _custom(B, Hq, Hkv, D, N, sink, window, seed=7)
    c, kc, vc, pos = _prefilled(cfg, 0.5, 2.0, rng, seq_budget=nb)
    # junk beyond each budget: NaN codes and far-ahead positions
    for b in range(B):
        kc[b, :, nb[b]:] = 0x7F
        vc[b, :, nb[b]:] = 0xFF
        pos[b, :, nb[b]:] = 10_000_000
    c.set_state(kc, vc, pos)
    run_steps(c, cfg, kc, vc, pos, 4, rng, seq_budget=nb)


def test_attention_only():
    rng = np.random.default_rng(8)
    cfg = _custom(3, 8, 2, 128, 400, 4, 8, seed=8)
    c, kc, vc, pos = _prefilled(cfg, 0.25, 4.0, rng, n=333)
    qb, knb, vnb = _bits(rng, (3, 8, 128)), _bits(rng, (3, 2, 128)), _bits(rng, (3, 2, 128))
    c.step(qb, knb, vnb, attention_only=True)
    out, _, gk, gv, gp = c.host_rows()
    ref = oracle.decode_attention(oracle.dequantize(kc, 0.25), oracle.dequantize(vc, 4.0), pos,
                                  _f64(qb), _f64(knb), _f64(vnb))
    assert np.max(np.abs(out - ref)) <= H.OUT_ATOL
    assert np.array_equal(gk, kc) and np.array_equal(gv, vc) and np.array_equal(gp, pos)


def test_bad_scales_rejected_on_host():
    import torch
    h = binding.lf_init(1, 4, 2, 128, 256)
    try:
        lib = binding.load_library()
        z = torch.zeros(1 << 16, dtype=torch.int32, device="cuda")
        p = z.data_ptr()
        for ks, vs in [(0.0, 1.0), (1.0, -1.0), (float("inf"), 1.0), (1.0, float("nan"))]:
            assert lib.lf_decode_step_fp8(h.ptr, p, p, p, p, p, p, 256, None, 4, 8, ks, vs, p, p) \
                == binding.LF_EINVAL
            assert lib.lf_prefill_cache_fp8(h.ptr, p, p, 4, p, p, p, 256, ks, vs) == binding.LF_EINVAL
    finally:
        binding.lf_destroy(h)
