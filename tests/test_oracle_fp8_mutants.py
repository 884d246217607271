"""The FP8 pins must catch plausible mistakes in the FP8 oracle: each mutant
is a copy of oracle/kvfp8.py with one planted mistake (CPU only)."""
import inspect
import sys
import types

import pytest

import oracle
import oracle.kvfp8 as real
from tests import test_oracle_fp8 as pins

MUTANTS = {
    "exponent_bias": ("np.exp2(e - 7.0)", "np.exp2(e - 8.0)"),
    "subnormal_scale": ("sub = sign * (m / 8.0) * 2.0 ** -6", "sub = sign * (m / 8.0) * 2.0 ** -7"),
    "ties_away_from_zero": ("pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))",
                            "pick_hi = (dhi <= dlo)"),
    "no_saturation": ("code = np.where(a >= _MAGS[-1], len(_MAGS) - 1,",
                      "code = np.where(a >= 2 * _MAGS[-1], len(_MAGS),"),
    "scale_ignored": ("return e4m3_decode(codes) * float(np.float32(scale))",
                      "return e4m3_decode(codes) * 1.0"),
    "new_token_quantised_in_attention": (
        "res = longflow.decode_step(K, V, pos, q, k_new, v_new,",
        "res = longflow.decode_step(K, V, pos, q, dequantize(quantize(k_new, k_scale), k_scale), v_new,"),
    "stored_unscaled": ("kq[b, g, slot] = quantize(k_new[b, g], k_scale)",
                        "kq[b, g, slot] = quantize(k_new[b, g], 1.0)"),
}
NAMES = ("e4m3_decode", "e4m3_encode", "quantize", "dequantize", "decode_step_fp8", "prefill_fp8")


def _mutant(name, old, new):
    src = inspect.getsource(real)
    assert src.count(old) == 1, name
    mod = types.ModuleType("oracle.kvfp8_mutant_" + name)
    mod.__package__ = "oracle"
    sys.modules[mod.__name__] = mod
    try:
        exec(compile(src.replace(old, new), mod.__name__, "exec"), mod.__dict__)
    finally:
        sys.modules.pop(mod.__name__, None)
    return mod


def _pin_calls():
    calls = [(pins.test_decode_all_codes_match_torch, {}),
             (pins.test_encode_matches_torch_in_range, {}),
             (pins.test_encode_exact_halfway_points_and_subnormals, {}),
             (pins.test_encode_saturates_and_keeps_nan, {}),
             (pins.test_fp8_output_is_attention_over_dequantised_cache_and_exact_new_token, {}),
             (pins.test_fp8_prefill_layout, {})]
    calls += [(pins.test_power_of_two_scale_is_an_exact_division, dict(k=k)) for k in (-3, 2)]
    calls += [(pins.test_fp8_step_matches_brute_force, dict(seed=s)) for s in range(6)]
    return calls


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8_pins_catch_mutant(name, monkeypatch):
    mod = _mutant(name, *MUTANTS[name])
    for n in NAMES:
        monkeypatch.setattr(oracle, n, getattr(mod, n))
    for fn, kw in _pin_calls():
        try:
            fn(**kw)
        except (AssertionError, ValueError, IndexError):
            return
    pytest.fail(f"no pin caught the mutant {name}")


def test_fp8_unmutated_copy_passes(monkeypatch):
    mod = _mutant("identity", "E4M3_MAX = 448.0", "E4M3_MAX = 448.0")
    for n in NAMES:
        monkeypatch.setattr(oracle, n, getattr(mod, n))
    for fn, kw in _pin_calls():
        fn(**kw)
