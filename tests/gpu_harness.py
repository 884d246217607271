"""Runs the CUDA path (through the C ABI) and the oracle on the same seeded
inputs and compares them under the acceptance rules:

* out: max-abs error <= 2e-3 against the fp64 oracle (bf16 inputs, fp32
  accumulation on the GPU);
* evicted slot: bit-exact, except where the oracle's two lowest candidate
  scores differ by less than 1e-6 relative; then any candidate whose oracle
  score is <= s_min * (1 + 1e-6) is accepted (and counted);
* positions and cache contents: bit-exact against the state the chosen slot
  implies.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

import oracle
from attention_lf_decode_b200 import binding, synth

OUT_ATOL = 2e-3
TIE_REL = 1e-6
# oracle score name -> the library's LF_SCORE_* code
SCORE_CODES = {"mean_prob": binding.LF_SCORE_MEAN_PROB, "alpha_l1v": binding.LF_SCORE_ALPHA_L1V}


@dataclass
class Stats:
    steps: int = 0
    rows: int = 0
    max_abs: float = 0.0
    exact_evictions: int = 0
    accepted_ties: int = 0
    appends: int = 0
    mismatches: list = field(default_factory=list)


class GpuCache:
    """Device-side cache of one config, driven through the C ABI."""

    def __init__(self, cfg: synth.DecodeConfig, prefill_k=None, prefill_v=None, n=None,
                 split: int = 0, zero_init: bool = True, score: str = "mean_prob"):
        import torch
        self.torch = torch
        self.cfg = cfg
        c = cfg
        dev = "cuda"
        alloc = torch.zeros if zero_init else torch.empty
        self.h = binding.lf_init(c.batch, c.hq, c.hkv, c.head_dim, c.budget)
        if split:
            binding.lf_set_split(self.h, split)
        self.score = score
        binding.lf_set_score(self.h, SCORE_CODES[score])
        self.kcache = alloc((c.batch, c.hkv, c.budget, c.head_dim), dtype=torch.bfloat16, device=dev)
        self.vcache = alloc((c.batch, c.hkv, c.budget, c.head_dim), dtype=torch.bfloat16, device=dev)
        self.pos = torch.full((c.batch, c.hkv, c.budget), -7, dtype=torch.int32, device=dev)
        self.out = torch.empty((c.batch, c.hq, c.head_dim), dtype=torch.float32, device=dev)
        self.evicted = torch.empty((c.batch, c.hkv), dtype=torch.int32, device=dev)
        n = c.prefill if n is None else n
        if n > 0:
            k = binding.bf16_from_bits(prefill_k)
            v = binding.bf16_from_bits(prefill_v)
        else:
            k = v = None
        binding.lf_prefill_cache(self.h, k, v, n, self.kcache, self.vcache, self.pos, c.budget)

    def set_state(self, kbits, vbits, pos):
        """Overwrite the whole device state (teacher forcing, custom states)."""
        self.kcache.copy_(binding.bf16_from_bits(kbits))
        self.vcache.copy_(binding.bf16_from_bits(vbits))
        self.pos.copy_(self.torch.from_numpy(np.ascontiguousarray(pos, np.int32)).cuda())

    def step(self, qb, knb, vnb, attention_only: bool = False):
        c = self.cfg
        q = binding.bf16_from_bits(qb)
        kn = binding.bf16_from_bits(knb)
        vn = binding.bf16_from_bits(vnb)
        if attention_only:
            binding.lf_decode_attention(self.h, q, kn, vn, self.kcache, self.vcache, self.pos,
                                        c.budget, self.out)
        else:
            binding.lf_decode_step(self.h, q, kn, vn, self.kcache, self.vcache, self.pos,
                                   c.budget, c.sink, c.window, self.out, self.evicted)
        return self

    def status(self):
        return binding.lf_get_status(self.h), binding.lf_status_bits(self.h)

    def host_rows(self, batch_idx: Optional[Sequence[int]] = None):
        """(out, evicted, kbits, vbits, pos) for the given batch entries."""
        t = self.torch
        t.cuda.synchronize()
        sel = slice(None) if batch_idx is None else t.tensor(list(batch_idx), device="cuda")
        if batch_idx is None:
            o, e, k, v, p = self.out, self.evicted, self.kcache, self.vcache, self.pos
        else:
            o, e = self.out.index_select(0, sel), self.evicted.index_select(0, sel)
            k, v, p = (x.index_select(0, sel) for x in (self.kcache, self.vcache, self.pos))
        return (o.cpu().numpy(), e.cpu().numpy(), binding.bits_from_bf16(k),
                binding.bits_from_bf16(v), p.cpu().numpy())


def oracle_state(kbits, vbits, pos):
    return synth.bf16_bits_to_f64(kbits), synth.bf16_bits_to_f64(vbits), pos.astype(np.int64)


def check_step(res: "oracle.StepResult", pre_pos, gpu, stats: Stats, kbits_pre, vbits_pre,
               knb, vnb, where: str = ""):
    """Compare one GPU step (host copies) with the oracle's step from the same
    pre-step state.  Returns the post-step state both agree on (bits, pos) so
    a teacher-forced run continues from it."""
    out, ev, kb, vb, pos = gpu
    stats.steps += 1
    err = float(np.max(np.abs(out.astype(np.float64) - res.out))) if out.size else 0.0
    stats.max_abs = max(stats.max_abs, err)
    assert err <= OUT_ATOL, f"{where}: out max-abs error {err}"
    B, Hkv = ev.shape
    exp_k = kbits_pre.copy()
    exp_v = vbits_pre.copy()
    exp_p = pre_pos.astype(np.int32).copy()
    for b in range(B):
        for g in range(Hkv):
            r = res.rows[b * Hkv + g]
            stats.rows += 1
            e_gpu = int(ev[b, g])
            if r.evicted == -1:
                stats.appends += 1
                assert e_gpu == -1, f"{where} row ({b},{g}): expected append, got {e_gpu}"
                slot = r.slot
            elif e_gpu == r.evicted:
                stats.exact_evictions += 1
                slot = e_gpu
            else:
                ok = (0 <= e_gpu < len(r.score)) and bool(r.candidates[e_gpu])
                smin = float(r.score[r.evicted])
                if ok:
                    ok = float(r.score[e_gpu]) <= smin * (1 + TIE_REL)
                if not ok:
                    cs = np.sort(r.score[r.candidates])[:3]
                    stats.mismatches.append((where, b, g, r.evicted, e_gpu))
                    raise AssertionError(
                        f"{where} row ({b},{g}): evicted {e_gpu}, oracle {r.evicted}; "
                        f"lowest oracle scores {cs}, gpu slot score "
                        f"{r.score[e_gpu] if 0 <= e_gpu < len(r.score) else None}")
                stats.accepted_ties += 1
                slot = e_gpu
            exp_k[b, g, slot] = knb[b, g]
            exp_v[b, g, slot] = vnb[b, g]
            exp_p[b, g, slot] = r.t
    assert np.array_equal(pos, exp_p), f"{where}: positions differ"
    assert np.array_equal(kb, exp_k), f"{where}: K cache differs"
    assert np.array_equal(vb, exp_v), f"{where}: V cache differs"
    return exp_k, exp_v, exp_p


def teacher_forced(cfg: synth.DecodeConfig, steps: int, batch_idx=None, split: int = 0,
                   gen: Optional[synth.SynthDecode] = None, score: str = "mean_prob") -> Stats:
    """Run `steps` decode steps on the GPU over the whole batch; after every
    step compare the rows of `batch_idx` with the oracle run from the same
    pre-step state.  Near-tie choices are accepted and the oracle follows the
    GPU's choice (the states stay identical)."""
    gen = gen or synth.SynthDecode(cfg)
    kpre, vpre = gen.prefill()
    g = GpuCache(cfg, kpre, vpre, split=split, score=score)
    bsel = list(range(cfg.batch)) if batch_idx is None else list(batch_idx)
    kb, vb = (synth.prefill_layout(kpre[bsel], vpre[bsel], cfg.budget)[:2])
    pos = synth.prefill_layout(kpre[bsel], vpre[bsel], cfg.budget)[2]
    del kpre, vpre
    stats = Stats()
    for s in range(steps):
        qb, knb, vnb = gen.step_inputs(s)
        g.step(qb, knb, vnb)
        K, V, P = oracle_state(kb, vb, pos)
        res = oracle.decode_step(K, V, P, synth.bf16_bits_to_f64(qb[bsel]),
                                 synth.bf16_bits_to_f64(knb[bsel]),
                                 synth.bf16_bits_to_f64(vnb[bsel]), cfg.sink, cfg.window,
                                 score=score)
        gpu = g.host_rows(None if batch_idx is None else bsel)
        kb, vb, pos = check_step(res, pos, gpu, stats, kb, vb, knb[bsel], vnb[bsel],
                                 where=f"{cfg.name} step {s}")
    code, bits = g.status()
    assert code == binding.LF_OK, f"device status bits {bits}"
    return stats
