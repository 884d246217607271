"""FP8 (E4M3) KV storage for the LongFlow decode step — TEST INFRASTRUCTURE ONLY.

Like ``oracle/longflow.py``, only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module; the library never
calls it and shares nothing with it.

Storing the cache in 8-bit floats is an idea of another page of the same
subject ("ARKV", section "Fase de Decodificación": medium-importance tokens
kept in low precision such as FP8 and dequantised on the fly before
attention); here it is applied to the whole LongFlow cache.  What it
computes, and the readings taken where nothing is stated:

* Format: OCP E4M3 "fn" (no infinities): 1 sign bit, 4 exponent bits with
  bias 7, 3 mantissa bits.  Exponent field 0 holds subnormals m/8 * 2^-6;
  S.1111.111 is NaN; the largest finite magnitude is 1.75 * 2^8 = 448.
* One scale per cache tensor (``k_scale``, ``v_scale``, positive fp32):
  a stored code c stands for E4M3(c) * scale.
* Writing a value x (bf16): the quotient x / scale is taken in fp32 (IEEE,
  correctly rounded), then rounded to the nearest E4M3 value, ties to the
  even code; a finite quotient beyond +-448 saturates to +-448.
* The new token takes part in this step's attention with its exact bf16
  k_new / v_new; only the copy written into the cache is quantised.
* Everything else is the decode step of ``oracle/longflow.py``, run on the
  dequantised cache.
"""
from __future__ import annotations

import numpy as np

from . import longflow

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_decode(codes) -> np.ndarray:
    """float64 value of every E4M3 code (NaN for S.1111.111)."""
    c = np.asarray(codes, np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = sign * (m / 8.0) * 2.0 ** -6
    v = np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


# the finite non-negative magnitudes, by code 0x00 .. 0x7E (increasing)
_MAGS = e4m3_decode(np.arange(0x7F))


def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 code of each value (ties to the even code), saturating
    finite values beyond +-448 to +-448; NaN gives the NaN code."""
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    hi = np.clip(np.searchsorted(_MAGS, a, side="left"), 0, len(_MAGS) - 1)
    lo = np.clip(hi - 1, 0, len(_MAGS) - 1)
    dlo = a - _MAGS[lo]
    dhi = _MAGS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(a >= _MAGS[-1], len(_MAGS) - 1, np.where(pick_hi, hi, lo))
    code = np.where(a <= 0.0, 0, code)
    code = code | np.where(np.signbit(x), 0x80, 0)
    return np.where(np.isnan(x), E4M3_NAN, code).astype(np.uint8)


def quantize(x, scale: float) -> np.ndarray:
    """Codes of values x stored with a tensor scale: fp32 quotient, then E4M3."""
    q = np.asarray(x, np.float32) / np.float32(scale)
    return e4m3_encode(q.astype(np.float64))


def dequantize(codes, scale: float) -> np.ndarray:
    return e4m3_decode(codes) * float(np.float32(scale))


def decode_step_fp8(kcodes, vcodes, pos, q, k_new, v_new, sink: int, window: int,
                    k_scale: float, v_scale: float, score: str = "mean_prob",
                    seq_budget=None) -> longflow.StepResult:
    """The decode step on an E4M3 cache: kcodes/vcodes [B,Hkv,N,D] uint8.
    Returns a StepResult whose kcache/vcache are the updated code arrays."""
    K = dequantize(kcodes, k_scale)
    V = dequantize(vcodes, v_scale)
    res = longflow.decode_step(K, V, pos, q, k_new, v_new, sink, window, score=score,
                               seq_budget=seq_budget)
    kq = np.array(kcodes, np.uint8, copy=True)
    vq = np.array(vcodes, np.uint8, copy=True)
    B, Hkv = kq.shape[:2]
    for b in range(B):
        for g in range(Hkv):
            slot = res.rows[b * Hkv + g].slot
            kq[b, g, slot] = quantize(k_new[b, g], k_scale)
            vq[b, g, slot] = quantize(v_new[b, g], v_scale)
    return longflow.StepResult(res.out, res.evicted, kq, vq, res.pos, res.rows)


def prefill_fp8(k, v, n: int, budget: int, k_scale: float, v_scale: float):
    """An E4M3 cache after prefill: slots 0..n-1 hold the quantised prompt,
    pos[j] = j; the rest is empty (pos -1, code 0)."""
    kc, vc, pos = longflow.prefill(k, v, n, budget)
    kq = quantize(kc, k_scale)
    vq = quantize(vc, v_scale)
    kq[..., n:, :] = 0
    vq[..., n:, :] = 0
    return kq, vq, pos
