"""The pins must catch plausible mistakes in the oracle.

Each mutant is a copy of the oracle's source with one planted mistake (an
off-by-one in a mask, a dropped softmax term, a wrong scale, a transposed
head mapping, a wrong reduction, a wrong tie-break); it runs on the CPU
only.  The test asserts that at least one pin of tests/test_oracle.py fails
on every mutant.
"""
import inspect
import sys
import types

import pytest

import oracle.longflow as real
from tests import test_oracle as pins

MUTANTS = {
    "window_off_by_one": ("cand = (j >= sink) & (pos < t - window)",
                          "cand = (j >= sink) & (pos <= t - window)"),
    "sink_off_by_one": ("cand = (j >= sink) & (pos < t - window)",
                        "cand = (j > sink) & (pos < t - window)"),
    "sink_by_position": ("cand = (j >= sink) & (pos < t - window)",
                         "cand = (pos >= sink) & (pos < t - window)"),
    "window_by_slot": ("cand = (j >= sink) & (pos < t - window)",
                       "cand = (j >= sink) & (j < N - window)"),
    "new_token_not_in_denominator": ("l = e.sum(axis=1) + e_new", "l = e.sum(axis=1) + 0 * e_new"),
    "new_token_not_in_max": ("m = np.maximum(s.max(axis=1), s_new)", "m = s.max(axis=1)"),
    "scale_1_over_d": ("scale = 1.0 / math.sqrt(D)", "scale = 1.0 / D"),
    "gqa_strided_heads": ("q[b, g * G:(g + 1) * G], k_new[b, g]", "q[b, g::Hkv], k_new[b, g]"),
    "score_max_over_heads": ("alpha = p.mean(axis=0)", "alpha = p.max(axis=0)"),
    "score_first_head_only": ("alpha = p.mean(axis=0)", "alpha = p[0]"),
    "l1v_signed_sum": ("sc = alpha * np.abs(V).sum(axis=1)", "sc = alpha * V.sum(axis=1)"),
    "l1v_l2_norm": ("sc = alpha * np.abs(V).sum(axis=1)", "sc = alpha * np.sqrt((V * V).sum(axis=1))"),
    "l1v_key_norm": ("sc = alpha * np.abs(V).sum(axis=1)", "sc = alpha * np.abs(K).sum(axis=1)"),
    "l1v_divides": ("sc = alpha * np.abs(V).sum(axis=1)", "sc = alpha / np.abs(V).sum(axis=1)"),
    "l1v_dropped": ('if score == "alpha_l1v":', 'if score == "no such score":'),
    "l1v_max_norm": ("sc = alpha * np.abs(V).sum(axis=1)", "sc = alpha * np.abs(V).max(axis=1)"),
    "ragged_budget_ignored": ("        n = nb[b]\n        for g in range(Hkv):\n            r = decode_row(",
                              "        n = N\n        for g in range(Hkv):\n            r = decode_row("),
    "ragged_budget_minus_one": ("        n = nb[b]\n        for g in range(Hkv):\n            r = decode_row(",
                                "        n = max(1, nb[b] - 1)\n        for g in range(Hkv):\n            r = decode_row("),
    "ties_to_highest_slot": (
        "slot = int(np.argmin(np.where(cand, sc, np.inf)))",
        "slot = int(N - 1 - np.argmin(np.where(cand, sc, np.inf)[::-1]))"),
    "t_is_max_pos": ("t = int(pos[filled].max()) + 1", "t = int(pos[filled].max())"),
    "append_to_highest_free": ("slot = int(np.flatnonzero(~filled)[0])",
                               "slot = int(np.flatnonzero(~filled)[-1])"),
    "out_drops_new_value": ("+ p_new[:, None] * v_new[None, :]", "+ 0 * v_new[None, :]"),
}


def _mutant(name, old, new):
    src = inspect.getsource(real)
    assert src.count(old) >= 1, name
    mod = types.ModuleType("oracle_mutant_" + name)
    mod.__file__ = "<mutant>"
    sys.modules[mod.__name__] = mod
    try:
        exec(compile(src.replace(old, new, 1), mod.__name__, "exec"), mod.__dict__)
    finally:
        sys.modules.pop(mod.__name__, None)
    return mod


def _pin_calls():
    calls = [(pins.test_output_matches_library_attention, dict(B=2, Hq=4, Hkv=2, D=8, N=12, fill=12)),
             (pins.test_output_matches_library_attention, dict(B=1, Hq=8, Hkv=2, D=64, N=40, fill=17)),
             (pins.test_no_eviction_while_budget_covers_length, {}),
             (pins.test_hand_cases, {}),
             (pins.test_trajectory_invariants, {}),
             (pins.test_uniform_keys_evict_in_a_cycle, dict(N=32, sink=4, window=6, G=1))]
    calls += [(pins.test_matches_scalar_brute_force, dict(seed=s, score="mean_prob")) for s in range(40)]
    calls += [(pins.test_single_head_evicts_lowest_exact_dot, dict(seed=s)) for s in range(4)]
    calls += [(pins.test_matches_scalar_brute_force, dict(seed=s, score="alpha_l1v"))
              for s in range(100, 130)]
    calls += [(pins.test_page_score_single_head_log_domain, dict(seed=s)) for s in range(2)]
    calls += [(pins.test_ragged_matches_brute_force, dict(seed=s)) for s in range(6)]
    calls += [(pins.test_ragged_outputs_match_library_attention, {})]
    calls += [(pins.test_page_score_zero_norm_values_go_first, {}),
              (pins.test_page_score_equal_norms_rank_like_mean_prob, {})]
    return calls


# a planted mistake may overflow (e.g. a max that misses the new token's
# logit makes exp() overflow): the pins must fail on it, quietly
@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    mod = _mutant(name, *MUTANTS[name])
    monkeypatch.setattr(pins, "oracle", mod)
    for fn, kw in _pin_calls():
        try:
            fn(**kw)
        except (AssertionError, ValueError, IndexError):
            return
    pytest.fail(f"no pin caught the mutant {name}")


def test_unmutated_copy_passes(monkeypatch):
    mod = _mutant("identity", "import math", "import math")
    monkeypatch.setattr(pins, "oracle", mod)
    for fn, kw in _pin_calls():
        fn(**kw)
