"""Pins of the FP8 (E4M3) cache oracle (CPU only).

* decoding: every one of the 256 codes against torch's float8_e4m3fn;
* encoding: round to nearest, ties to even, against torch's conversion on
  random values over the whole range, exact halfway points and subnormals;
  saturation to +-448 beyond (where torch gives NaN instead, by its own
  definition), and the NaN code;
* scales: with a power-of-two scale the fp32 quotient is exact, so the
  codes equal torch's conversion of x / scale;
* the step: the scalar brute force on the dequantised cache, torch SDPA on
  the dequantised cache plus the exact new token, and the new token's codes.
"""

import numpy as np
import pytest
import torch

import oracle
from attention_lf_decode_b200 import synth
from tests.brute_force import brute_row
from tests.test_oracle import sdpa_reference

F8 = torch.float8_e4m3fn


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(F8).to(torch.float64).numpy()


def _torch_encode(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(F8).view(torch.uint8).numpy()


def test_decode_all_codes_match_torch():
    c = np.arange(256)
    a, b = oracle.e4m3_decode(c), _torch_decode(c)
    assert np.array_equal(np.isnan(a), np.isnan(b))
    ok = ~np.isnan(a)
    assert np.array_equal(a[ok], b[ok]) and np.array_equal(np.signbit(a[ok]), np.signbit(b[ok]))
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6 and oracle.e4m3_decode(0x38) == 1.0


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(100_000) * np.exp2(rng.uniform(-12, 9, 100_000)),
        rng.uniform(-463.99, 463.99, 20_000),
    ]).astype(np.float32)
    x = x[np.abs(x) < 464]
    assert np.array_equal(oracle.e4m3_encode(x), _torch_encode(x))


def test_encode_exact_halfway_points_and_subnormals():
    mags = oracle.e4m3_decode(np.arange(0x7F))
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)   # exact in fp32
    x = np.concatenate([mids, -mids, mags.astype(np.float32)])
    enc = oracle.e4m3_encode(x)
    assert np.array_equal(enc, _torch_encode(x))
    # ties go to the even code
    assert (oracle.e4m3_encode(mids) % 2 == 0).all()
    assert oracle.e4m3_encode(2.0 ** -10) == 0 and oracle.e4m3_encode(1.5 * 2.0 ** -9) == 2


def test_encode_saturates_and_keeps_nan():
    x = np.array([464.0, 1e6, -465.0, -1e30, np.inf, -np.inf], np.float32)
    assert list(oracle.e4m3_encode(x)) == [0x7E, 0x7E, 0xFE, 0xFE, 0x7E, 0xFE]
    assert oracle.e4m3_encode(np.nan) == 0x7F
    # round trip of every finite code
    c = np.array([k for k in range(256) if (k & 0x7F) != 0x7F])
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(c)), c.astype(np.uint8))


@pytest.mark.parametrize("k", [-3, 0, 2, 5])
def test_power_of_two_scale_is_an_exact_division(k):
    rng = np.random.default_rng(k + 10)
    x = synth.bf16_bits_to_f32(synth.to_bf16_bits(rng.standard_normal(5000).astype(np.float32) * 4))
    codes = oracle.quantize(x, 2.0 ** k)
    ref = _torch_encode(x / np.float32(2.0 ** k))
    ok = np.abs(x / 2.0 ** k) < 464
    assert np.array_equal(codes[ok], ref[ok])
    np.testing.assert_array_equal(oracle.dequantize(codes, 2.0 ** k), oracle.e4m3_decode(codes) * 2.0 ** k)


def _fp8_state(rng, B, Hq, Hkv, D, N, fill, ks, vs):
    kc = rng.integers(0, 256, size=(B, Hkv, N, D)).astype(np.uint8)
    vc = rng.integers(0, 256, size=(B, Hkv, N, D)).astype(np.uint8)
    # no NaN codes in the cache
    kc[(kc & 0x7F) == 0x7F] = 0x3F
    vc[(vc & 0x7F) == 0x7F] = 0x3F
    pos = np.full((B, Hkv, N), -1, np.int64)
    for b in range(B):
        for g in range(Hkv):
            slots = rng.permutation(N)[:fill]
            pos[b, g, slots] = np.arange(fill)
    bf = lambda s: synth.bf16_bits_to_f64(synth.to_bf16_bits(rng.standard_normal(s).astype(np.float32)))
    return kc, vc, pos, bf((B, Hq, D)) * 0.05, bf((B, Hkv, D)), bf((B, Hkv, D))


@pytest.mark.parametrize("seed", range(16))
def test_fp8_step_matches_brute_force(seed):
    rng = np.random.default_rng(4000 + seed)
    Hkv, G = int(rng.integers(1, 3)), int(rng.integers(1, 4))
    D, N = int(rng.choice([2, 4, 8])), int(rng.integers(6, 13))
    sink, window = 1, 2
    fill = N if seed % 3 else int(rng.integers(0, N + 1))
    ks, vs = float(np.float32(rng.uniform(0.05, 3.0))), float(np.float32(rng.uniform(0.05, 3.0)))
    score = "alpha_l1v" if seed % 2 else "mean_prob"
    kc, vc, pos, q, kn, vn = _fp8_state(rng, 1, G * Hkv, Hkv, D, N, fill, ks, vs)
    res = oracle.decode_step_fp8(kc, vc, pos, q, kn, vn, sink, window, ks, vs, score=score)
    Kd = oracle.e4m3_decode(kc) * ks
    Vd = oracle.e4m3_decode(vc) * vs
    for g in range(Hkv):
        out, ev, slot, t = brute_row(Kd[0, g].tolist(), Vd[0, g].tolist(), pos[0, g].tolist(),
                                     q[0, g * G:(g + 1) * G].tolist(), kn[0, g].tolist(),
                                     vn[0, g].tolist(), sink, window, score=score)
        assert res.evicted[0, g] == ev
        np.testing.assert_allclose(res.out[0, g * G:(g + 1) * G], np.array(out), rtol=0, atol=1e-12)
        # the new token is stored quantised: torch's codes of x / scale (in range)
        kq, vq = _torch_encode(kn[0, g] / np.float32(ks)), _torch_encode(vn[0, g] / np.float32(vs))
        np.testing.assert_array_equal(res.kcache[0, g, slot], kq)
        np.testing.assert_array_equal(res.vcache[0, g, slot], vq)
        assert res.pos[0, g, slot] == t
        others = np.arange(N) != slot
        np.testing.assert_array_equal(res.kcache[0, g][others], kc[0, g][others])


def test_fp8_output_is_attention_over_dequantised_cache_and_exact_new_token():
    rng = np.random.default_rng(4100)
    ks, vs = 0.75, 1.25
    kc, vc, pos, q, kn, vn = _fp8_state(rng, 2, 8, 2, 16, 30, 30, ks, vs)
    res = oracle.decode_step_fp8(kc, vc, pos, q, kn, vn, 2, 4, ks, vs)
    ref = sdpa_reference(oracle.dequantize(kc, ks), oracle.dequantize(vc, vs), pos, q, kn, vn)
    np.testing.assert_allclose(res.out, ref, rtol=0, atol=1e-12)


def test_fp8_prefill_layout():
    rng = np.random.default_rng(4200)
    k = synth.bf16_bits_to_f64(synth.to_bf16_bits(rng.standard_normal((2, 2, 5, 8)).astype(np.float32)))
    v = synth.bf16_bits_to_f64(synth.to_bf16_bits(rng.standard_normal((2, 2, 5, 8)).astype(np.float32)))
    kq, vq, pos = oracle.prefill_fp8(k, v, 5, 9, 0.5, 2.0)
    np.testing.assert_array_equal(kq[..., :5, :], _torch_encode(k / np.float32(0.5)))
    np.testing.assert_array_equal(vq[..., :5, :], _torch_encode(v / np.float32(2.0)))
    assert (kq[..., 5:, :] == 0).all() and (pos[..., 5:] == -1).all()
    assert (pos[..., :5] == np.arange(5)).all()
