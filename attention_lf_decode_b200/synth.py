"""Seeded synthetic inputs for the LongFlow decode step.

This module only draws numbers: it holds none of the decode step's arithmetic
(no logits, softmax, scores or eviction).  Both the CUDA path (through the
tests and ``bench.py``) and the CPU oracle are fed from it, so both see the
same bf16 bits.

Workloads stand in for the long chain-of-thought decode the LongFlow pages
describe ("LongFlow: Efficient KV Cache Compression for Reasoning Models",
section 4 "Resultados Experimentales": reasoning models, budget 3,200 for
16,000 generated tokens; and the Russian blog page "Долгая память",
Qwen3-8B at batch 128 and length 3200).  No dataset is used.

Recipe (every tensor is drawn in fp32 and rounded once to bf16,
round-to-nearest-even):

* ``u``: a seeded unit vector in R^D (the "query-correlated direction").
* keys, values, new values: N(0, 1).
* key outliers: a Bernoulli(frac) mask per (row, slot) adds ``mag * u``.
  Prefill keys always get them; new keys only when ``new_key_outliers``.
* queries: ``u + N(0, 1)`` per head (``query_mode="shift"``), or
  ``u + z_t`` with z an AR(1) walk of coefficient rho that is stationary
  N(0, 1) (``query_mode="ar1"``), so the important slots drift.

Every draw is keyed by ``SeedSequence([seed, step_key, tensor_id, row])``
on a Philox generator, so any step or any row can be regenerated alone
(the oracle runs on row subsets of the large workloads).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Iterable, Optional, Sequence

import numpy as np

# tensor ids inside the seed sequence
_T_U = 1
_T_KPRE = 2
_T_VPRE = 3
_T_KPRE_MASK = 4
_T_Q = 5
_T_KNEW = 6
_T_VNEW = 7
_T_KNEW_MASK = 8
_T_AR_INIT = 9
_T_SEQ_BUDGET = 10
_PREFILL_KEY = 0  # step_key of prefill draws; decode step s uses s + 1


@dataclass(frozen=True)
class DecodeConfig:
    """Shape and data recipe of one decode workload."""

    name: str
    batch: int
    hq: int
    hkv: int
    head_dim: int
    budget: int
    sink: int
    window: int
    prefill: int
    steps: int
    seed: int
    key_outlier_frac: float = 0.05
    key_outlier_mag: float = 3.0
    new_key_outliers: bool = False
    query_mode: str = "shift"  # "shift" or "ar1"
    ar_rho: float = 0.95
    # ragged batch: per-sequence budgets drawn uniformly in
    # [seq_budget_min, budget] (0 = every sequence uses all slots)
    seq_budget_min: int = 0

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def rows(self) -> int:
        return self.batch * self.hkv

    def with_(self, **kw) -> "DecodeConfig":
        return dataclasses.replace(self, **kw)


def _budget_sweep(budget: int, seed: int, prefill: Optional[int] = None,
                  name: Optional[str] = None) -> DecodeConfig:
    return DecodeConfig(
        name=name or f"sweep_n{budget}", batch=32, hq=32, hkv=8, head_dim=128,
        budget=budget, sink=4, window=128,
        prefill=budget if prefill is None else prefill, steps=512, seed=seed)


CONFIGS = {
    # tiny decode: the small case the oracle finishes in seconds
    "tiny": DecodeConfig("tiny", batch=1, hq=8, hkv=2, head_dim=64, budget=256,
                         sink=4, window=16, prefill=256, steps=64, seed=1),
    # Llama-3-8B layer shape
    "llama3_8b": DecodeConfig("llama3_8b", batch=8, hq=32, hkv=8, head_dim=128,
                              budget=2048, sink=4, window=64, prefill=2048,
                              steps=1024, seed=2),
    # throughput point: batch 64, budget 4096, full cache
    "throughput": DecodeConfig("throughput", batch=64, hq=32, hkv=8, head_dim=128,
                               budget=4096, sink=4, window=128, prefill=4096,
                               steps=256, seed=3, key_outlier_frac=0.02,
                               key_outlier_mag=4.0, new_key_outliers=True),
    # long-reasoning trajectory: AR(1) queries, free-running
    "long_reasoning": DecodeConfig("long_reasoning", batch=16, hq=28, hkv=4,
                                   head_dim=128, budget=8192, sink=4, window=256,
                                   prefill=8192, steps=16384, seed=4,
                                   query_mode="ar1"),
    # ragged serving batch: the throughput shape with per-sequence budgets
    # drawn in [1024, 4096], each sequence's cache full at its own budget
    "ragged": DecodeConfig("ragged", batch=64, hq=32, hkv=8, head_dim=128,
                           budget=4096, sink=4, window=128, prefill=4096, steps=256,
                           seed=5, key_outlier_frac=0.02, key_outlier_mag=4.0,
                           new_key_outliers=True, seq_budget_min=1024),
    # budget sweep (full caches) and the no-eviction control
    "sweep_n1024": _budget_sweep(1024, 50),
    "sweep_n2048": _budget_sweep(2048, 51),
    "sweep_n4096": _budget_sweep(4096, 52),
    "sweep_n8192": _budget_sweep(8192, 53),
    "sweep_control": _budget_sweep(16384, 54, prefill=8192, name="sweep_control"),
}


# ---------------------------------------------------------------- bf16 bits

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits.

    Inputs are finite draws; NaN handling is not needed here.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
    return (b >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


# ---------------------------------------------------------------- generator

def _rng(seed: int, step_key: int, tensor_id: int, row: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(
        np.random.SeedSequence([seed, step_key, tensor_id, row])))


class SynthDecode:
    """Draws the prefill cache and the per-step (q, k_new, v_new) of a config.

    All arrays are bf16 bit patterns (``uint16``) in the layouts the library
    uses: prefill K/V ``[B, Hkv, n, D]``, q ``[B, Hq, D]``, k_new and v_new
    ``[B, Hkv, D]``.
    """

    def __init__(self, cfg: DecodeConfig):
        self.cfg = cfg
        g = _rng(cfg.seed, _PREFILL_KEY, _T_U)
        u = g.standard_normal(cfg.head_dim)
        self.u = (u / np.linalg.norm(u)).astype(np.float32)
        self._ar_step = -1
        self._ar_z: Optional[np.ndarray] = None

    # -- prefill ------------------------------------------------------------
    def prefill_row(self, row: int, n: Optional[int] = None):
        """Prefill K and V of one flat row ``row = b * Hkv + g``: ([n, D], [n, D])."""
        c = self.cfg
        n = c.prefill if n is None else n
        D = c.head_dim
        k = _rng(c.seed, _PREFILL_KEY, _T_KPRE, row).standard_normal((n, D), dtype=np.float32)
        v = _rng(c.seed, _PREFILL_KEY, _T_VPRE, row).standard_normal((n, D), dtype=np.float32)
        mask = _rng(c.seed, _PREFILL_KEY, _T_KPRE_MASK, row).random(n) < c.key_outlier_frac
        if mask.any():
            k[mask] += np.float32(c.key_outlier_mag) * self.u
        return to_bf16_bits(k), to_bf16_bits(v)

    def prefill(self, batch_idx: Optional[Sequence[int]] = None, n: Optional[int] = None):
        """Prefill K/V for the given batch entries (all KV heads): [b', Hkv, n, D]."""
        c = self.cfg
        n = c.prefill if n is None else n
        bs = range(c.batch) if batch_idx is None else list(batch_idx)
        k = np.empty((len(bs), c.hkv, n, c.head_dim), np.uint16)
        v = np.empty_like(k)
        for i, b in enumerate(bs):
            for g in range(c.hkv):
                k[i, g], v[i, g] = self.prefill_row(b * c.hkv + g, n)
        return k, v

    # -- decode steps -------------------------------------------------------
    def _ar_state(self, step: int) -> np.ndarray:
        c = self.cfg
        shape = (c.batch, c.hq, c.head_dim)
        if self._ar_z is None or step < self._ar_step:
            self._ar_z = _rng(c.seed, _PREFILL_KEY, _T_AR_INIT).standard_normal(
                shape, dtype=np.float32)
            self._ar_step = -1
        rho = np.float32(c.ar_rho)
        sig = np.float32(np.sqrt(1.0 - c.ar_rho * c.ar_rho))
        while self._ar_step < step:
            self._ar_step += 1
            eps = _rng(c.seed, self._ar_step + 1, _T_Q).standard_normal(shape, dtype=np.float32)
            if self._ar_step > 0:
                self._ar_z = rho * self._ar_z + sig * eps
        return self._ar_z

    def step_inputs(self, step: int):
        """(q [B,Hq,D], k_new [B,Hkv,D], v_new [B,Hkv,D]) bf16 bits of decode step ``step``.

        With ``query_mode="ar1"`` steps are cheapest when drawn in order.
        """
        c = self.cfg
        sk = step + 1
        if c.query_mode == "ar1":
            q = self.u + self._ar_state(step)
        else:
            q = self.u + _rng(c.seed, sk, _T_Q).standard_normal(
                (c.batch, c.hq, c.head_dim), dtype=np.float32)
        kn = _rng(c.seed, sk, _T_KNEW).standard_normal((c.batch, c.hkv, c.head_dim),
                                                       dtype=np.float32)
        vn = _rng(c.seed, sk, _T_VNEW).standard_normal((c.batch, c.hkv, c.head_dim),
                                                       dtype=np.float32)
        if c.new_key_outliers:
            m = _rng(c.seed, sk, _T_KNEW_MASK).random((c.batch, c.hkv)) < c.key_outlier_frac
            kn[m] += np.float32(c.key_outlier_mag) * self.u
        return to_bf16_bits(q), to_bf16_bits(kn), to_bf16_bits(vn)

    def seq_budgets(self) -> Optional[np.ndarray]:
        """Per-sequence budgets [B] (int32) of a ragged config, else None."""
        c = self.cfg
        if not c.seq_budget_min:
            return None
        g = _rng(c.seed, _PREFILL_KEY, _T_SEQ_BUDGET)
        return g.integers(c.seq_budget_min, c.budget + 1, size=c.batch).astype(np.int32)

    def iter_steps(self, steps: Optional[int] = None, start: int = 0) -> Iterable:
        n = self.cfg.steps if steps is None else steps
        for s in range(start, start + n):
            yield s, self.step_inputs(s)


def empty_cache_bits(rows_shape, budget: int, head_dim: int):
    """Zeroed K/V bit arrays and an all-empty position table (-1)."""
    k = np.zeros(tuple(rows_shape) + (budget, head_dim), np.uint16)
    return k, k.copy(), np.full(tuple(rows_shape) + (budget,), -1, np.int32)


def prefill_layout(k_bits: np.ndarray, v_bits: np.ndarray, budget: int):
    """Host-side layout of a prefilled cache: slots 0..n-1 hold the prompt.

    Returns (kcache, vcache, pos) with pos[j] = j for j < n and -1 after, the
    state the library's prefill call produces on the device.  Used to feed
    the oracle the same starting state without touching the GPU.
    """
    lead = k_bits.shape[:-2]
    n, D = k_bits.shape[-2:]
    kc, vc, pos = empty_cache_bits(lead, budget, D)
    kc[..., :n, :] = k_bits
    vc[..., :n, :] = v_bits
    pos[..., :n] = np.arange(n, dtype=np.int32)
    return kc, vc, pos
