"""CPU oracle of the LongFlow fused decode step — TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The library never calls it: the CUDA
path has no CPU fallback.  Nothing here is shared with the CUDA code.

Plain, slow, float64 NumPy.  Every input is a bf16 value held exactly in
float64, so the logits below are exact up to float64 rounding.

What one decode step computes, per row (batch entry b, KV head g), following

* "LongFlow: Efficient KV Cache Compression for Reasoning Models" (gist.science
  summary), §2A "Principios de Diseño": importance of every cached token is
  estimated from the current query alone (zero history) as a by-product of
  the attention itself (zero cost);
* same page, §2B "Derivación de la Métrica de Importancia": evict the token
  whose removal least changes the attention output, scored from the attention
  weight alpha of the current query;
* same page, §2C "Implementación de Alto Rendimiento": a statically
  pre-allocated KV cache and one fused pass doing attention, importance
  estimation and eviction;
* "Долгая память: Оптимизация кэша для сложных рассуждений" (blog page),
  section "Ограничения Памяти при Моделировании Длинных Последовательностей":
  one token is evicted after every attention computation.

Two scores are offered (argument ``score``):

* ``"mean_prob"`` (the default, fixed by the benchmark spec rather than the
  pages): the softmax probability of the current query averaged over the G
  query heads of the KV group;
* ``"alpha_l1v"``: the summary page's own form, §2B: the attention weight
  alpha of the token times the L1 norm of its value vector, sum_l |(v_j)_l|.
  The page states it for one attention head; for a KV group read by G query
  heads, alpha is read as the head-averaged probability, so this score is
  the ``"mean_prob"`` score times ||v_j||_1.  Both rank slots identically
  when every ||v_j||_1 is the same.

The first ``sink`` slots and the last ``window`` positions are protected;
ties go to the lowest slot index.

Readings of points the pages leave open:

* The new token takes part in this step's softmax (so with no eviction the
  output is plain decode attention over cache + new token); it is never a
  candidate for eviction.
* Eviction happens after the attention of the same step, so it never changes
  this step's output.
* t, the new token's position, is max(pos) + 1 over filled slots (0 for an
  empty cache); the window protects positions t - window .. t - 1.
* A slot with pos < 0 is empty.  If any slot is empty the new token goes to
  the lowest empty slot and nothing is evicted (evicted = -1).
* Query head h reads KV head h // G.
* Ragged batches: a sequence may have a budget n_b below the allocated
  slots N (``seq_budget``).  Its cache is then slots 0 .. n_b - 1 alone:
  the slots beyond are neither read (not even for t) nor written.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np


@dataclass
class RowStep:
    """Everything the oracle knows about one row's step."""

    out: np.ndarray          # [G, D] attention output
    evicted: int             # evicted slot, or -1 when an empty slot was filled
    slot: int                # slot that receives the new token
    t: int                   # position written for the new token
    p: np.ndarray            # [G, N] probabilities of cached slots (0 where empty)
    p_new: np.ndarray        # [G] probability of the new token
    score: Optional[np.ndarray]      # [N] eviction score of every slot (None: no eviction)
    candidates: Optional[np.ndarray]  # [N] bool, slots allowed to be evicted


SCORES = ("mean_prob", "alpha_l1v")


def decode_row(K, V, pos, q, k_new, v_new, sink: int, window: int,
               score: str = "mean_prob") -> RowStep:
    """One row of the decode step; inputs are not modified.

    K, V: [N, D] float64.  pos: [N] integer, -1 = empty.  q: [G, D].
    k_new, v_new: [D].  score: one of SCORES.
    """
    if score not in SCORES:
        raise ValueError(f"unknown score {score!r}")
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    q = np.asarray(q, np.float64)
    k_new = np.asarray(k_new, np.float64)
    v_new = np.asarray(v_new, np.float64)
    pos = np.asarray(pos, np.int64)
    N, D = K.shape
    G = q.shape[0]
    scale = 1.0 / math.sqrt(D)

    # position of the new token
    filled = pos >= 0
    t = int(pos[filled].max()) + 1 if filled.any() else 0

    # logits of the current query against every filled slot and the new key
    s = np.full((G, N), -np.inf)
    s[:, filled] = (q @ K[filled].T) * scale
    s_new = (q @ k_new) * scale

    # softmax over (filled slots) + (new token), per query head
    m = np.maximum(s.max(axis=1), s_new)
    e = np.zeros((G, N))
    e[:, filled] = np.exp(s[:, filled] - m[:, None])
    e_new = np.exp(s_new - m)
    l = e.sum(axis=1) + e_new
    p = e / l[:, None]
    p_new = e_new / l

    # attention output
    out = p[:, filled] @ V[filled] + p_new[:, None] * v_new[None, :]

    if not filled.all():
        slot = int(np.flatnonzero(~filled)[0])
        return RowStep(out, -1, slot, t, p, p_new, None, None)

    # zero-history score: this step's probability, averaged over the group
    alpha = p.mean(axis=0)
    if score == "alpha_l1v":
        # the page's form: alpha times the L1 norm of the slot's value vector
        sc = alpha * np.abs(V).sum(axis=1)
    else:
        sc = alpha
    j = np.arange(N)
    cand = (j >= sink) & (pos < t - window)
    if not cand.any():
        raise ValueError("no slot may be evicted (sink + window cover the cache)")
    slot = int(np.argmin(np.where(cand, sc, np.inf)))  # first minimum = lowest index
    return RowStep(out, slot, slot, t, p, p_new, sc, cand)


@dataclass
class StepResult:
    out: np.ndarray       # [B, Hq, D]
    evicted: np.ndarray   # [B, Hkv] int
    kcache: np.ndarray    # [B, Hkv, N, D] after the step
    vcache: np.ndarray
    pos: np.ndarray       # [B, Hkv, N] after the step
    rows: list            # RowStep per (b, g), row-major


def decode_step(kcache, vcache, pos, q, k_new, v_new, sink: int, window: int,
                score: str = "mean_prob", seq_budget=None) -> StepResult:
    """The batched decode step: kcache/vcache [B,Hkv,N,D], pos [B,Hkv,N],
    q [B,Hq,D], k_new/v_new [B,Hkv,D].  Returns new arrays; inputs untouched.
    score: one of SCORES (see decode_row).  seq_budget: None, or [B] budgets
    1 <= n_b <= N; batch entry b then uses slots 0 .. n_b - 1 only."""
    kcache = np.array(kcache, np.float64, copy=True)
    vcache = np.array(vcache, np.float64, copy=True)
    pos = np.array(pos, np.int64, copy=True)
    q = np.asarray(q, np.float64)
    B, Hkv, N, D = kcache.shape
    Hq = q.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    nb = _seq_budgets(seq_budget, B, N)
    out = np.zeros((B, Hq, D))
    evicted = np.zeros((B, Hkv), np.int64)
    rows = []
    for b in range(B):
        n = nb[b]
        for g in range(Hkv):
            r = decode_row(kcache[b, g, :n], vcache[b, g, :n], pos[b, g, :n],
                           q[b, g * G:(g + 1) * G], k_new[b, g], v_new[b, g],
                           sink, window, score)
            out[b, g * G:(g + 1) * G] = r.out
            evicted[b, g] = r.evicted
            kcache[b, g, r.slot] = k_new[b, g]
            vcache[b, g, r.slot] = v_new[b, g]
            pos[b, g, r.slot] = r.t
            rows.append(r)
    return StepResult(out, evicted, kcache, vcache, pos, rows)


def _seq_budgets(seq_budget, B: int, N: int) -> list:
    if seq_budget is None:
        return [N] * B
    nb = [int(x) for x in np.asarray(seq_budget).reshape(-1)]
    if len(nb) != B or any(n < 1 or n > N for n in nb):
        raise ValueError("seq_budget needs B entries in 1 .. N")
    return nb


def decode_attention(kcache, vcache, pos, q, k_new, v_new, seq_budget=None) -> np.ndarray:
    """Plain single-query decode attention over filled slots + the new token
    (the no-eviction control); nothing is scored or written.  seq_budget as
    in decode_step."""
    kcache = np.asarray(kcache, np.float64)
    vcache = np.asarray(vcache, np.float64)
    pos = np.asarray(pos)
    q = np.asarray(q, np.float64)
    B, Hkv, N, D = kcache.shape
    G = q.shape[1] // Hkv
    nb = _seq_budgets(seq_budget, B, N)
    out = np.zeros(q.shape)
    scale = 1.0 / math.sqrt(D)
    for b in range(B):
        n = nb[b]
        for g in range(Hkv):
            f = pos[b, g, :n] >= 0
            Kf = np.concatenate([kcache[b, g, :n][f], np.asarray(k_new[b, g], np.float64)[None]])
            Vf = np.concatenate([vcache[b, g, :n][f], np.asarray(v_new[b, g], np.float64)[None]])
            qs = q[b, g * G:(g + 1) * G]
            s = (qs @ Kf.T) * scale
            s -= s.max(axis=1, keepdims=True)
            w = np.exp(s)
            w /= w.sum(axis=1, keepdims=True)
            out[b, g * G:(g + 1) * G] = w @ Vf
    return out


def prefill(k, v, n: int, budget: int):
    """The cache after prefill: slots 0..n-1 hold the prompt K/V, pos[j] = j,
    the rest is empty (pos = -1, K/V zero).  A prompt longer than the budget
    is rejected: compressing the prefill is outside the method, which the
    summary page's §5 limits to autoregressive decode."""
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    if n > budget:
        raise ValueError("prefill longer than the budget")
    lead = k.shape[:-2]
    D = k.shape[-1]
    kc = np.zeros(lead + (budget, D))
    vc = np.zeros(lead + (budget, D))
    pos = np.full(lead + (budget,), -1, np.int64)
    kc[..., :n, :] = k[..., :n, :]
    vc[..., :n, :] = v[..., :n, :]
    pos[..., :n] = np.arange(n)
    return kc, vc, pos
