"""The N > 1 path on CPU: two gloo ranks (world size 2).

* each rank draws its own data (different seeds, same recipe);
* the timing reduction is the max over ranks, and the whole-job rate counts
  every rank's steps;
* a batch split over ranks and decoded independently (oracle on CPU) gives
  exactly the single-process result: rows need no data-path collective.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from attention_lf_decode_b200 import scaling, synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # 1. per-rank data differs
        cfg = synth.CONFIGS["tiny"].with_(batch=4, budget=64, prefill=64, window=8)
        rc = scaling.rank_config(cfg, rank)
        k, _ = synth.SynthDecode(rc).prefill([0])
        ks = [torch.zeros_like(torch.from_numpy(k.astype(np.int32))) for _ in range(world)]
        dist.all_gather(ks, torch.from_numpy(k.astype(np.int32)))
        differs = not torch.equal(ks[0], ks[1])

        # 2. max over ranks
        mx = scaling.max_over_ranks(10.0 + rank)

        # 3. sharded decode equals the whole-batch decode
        gen = synth.SynthDecode(cfg)
        mine = list(scaling.shard_batch(cfg.batch, world, rank))
        kb, vb = gen.prefill(mine)
        kc, vc, pos = synth.prefill_layout(kb, vb, cfg.budget)
        K, V, P = synth.bf16_bits_to_f64(kc), synth.bf16_bits_to_f64(vc), pos.astype(np.int64)
        outs, evs = [], []
        for s in range(6):
            qb, knb, vnb = gen.step_inputs(s)
            res = oracle.decode_step(K, V, P, synth.bf16_bits_to_f64(qb[mine]),
                                     synth.bf16_bits_to_f64(knb[mine]),
                                     synth.bf16_bits_to_f64(vnb[mine]), cfg.sink, cfg.window)
            K, V, P = res.kcache, res.vcache, res.pos
            outs.append(res.out)
            evs.append(res.evicted)
        out_t = torch.from_numpy(np.stack(outs))
        ev_t = torch.from_numpy(np.stack(evs))
        go = [torch.zeros_like(out_t) for _ in range(world)]
        ge = [torch.zeros_like(ev_t) for _ in range(world)]
        dist.all_gather(go, out_t)  # gathering for the check only
        dist.all_gather(ge, ev_t)
        if rank == 0:
            q.put((differs, mx, torch.cat(go, dim=1).numpy(), torch.cat(ge, dim=1).numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        differs, mx, out, ev = q.get(timeout=240)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert differs
    assert mx == 11.0

    import oracle
    cfg = synth.CONFIGS["tiny"].with_(batch=4, budget=64, prefill=64, window=8)
    gen = synth.SynthDecode(cfg)
    kb, vb = gen.prefill()
    kc, vc, pos = synth.prefill_layout(kb, vb, cfg.budget)
    K, V, P = synth.bf16_bits_to_f64(kc), synth.bf16_bits_to_f64(vc), pos.astype(np.int64)
    for s in range(6):
        qb, knb, vnb = gen.step_inputs(s)
        res = oracle.decode_step(K, V, P, synth.bf16_bits_to_f64(qb), synth.bf16_bits_to_f64(knb),
                                 synth.bf16_bits_to_f64(vnb), cfg.sink, cfg.window)
        K, V, P = res.kcache, res.vcache, res.pos
        np.testing.assert_array_equal(out[s], res.out)
        np.testing.assert_array_equal(ev[s], res.evicted)


@pytest.mark.parametrize("batch,world", [(64, 1), (64, 8), (7, 3), (2, 4)])
def test_shard_batch_partitions(batch, world):
    parts = [list(scaling.shard_batch(batch, world, r)) for r in range(world)]
    assert sum(parts, []) == list(range(batch))
    sizes = [len(p) for p in parts]
    assert max(sizes) - min(sizes) <= 1


def test_whole_job_rate():
    assert scaling.whole_job_rate(4, 1000, 500.0) == 8000.0
