"""Host logic of the sequence-parallel split on CPU: two gloo ranks, each
with its SPPlan, compute the oracle's attention over their own tokens for the
whole chunk, exchange the partial results and merge their own query slice;
the slices must equal the oracle's whole-cache attention, and the plans must
cover every token and every query row exactly once.  (The GPU path, shard
caches plus the merge kernel, is checked on one GPU in
test_gpu_sequence_parallel.py.)"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, errq):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import kvsynth
        from nvfp4_kv_cache_append_b200.sp import SPPlan
        from oracle.merge import lse_merge
        from oracle.stream import OracleStream
        wl = kvsynth.WORKLOADS["tiny"]
        plan = SPPlan(rank, world, wl.T, wl.Lq)
        spans = [None] * world
        dist.all_gather_object(spans, (plan.tokens, plan.queries))
        toks = sorted(t for t, _ in spans)
        qs = sorted(q for _, q in spans)
        assert toks[0][0] == 0 and toks[-1][1] == wl.T
        assert qs[0][0] == 0 and qs[-1][1] == wl.Lq
        assert all(a[1] == b[0] for a, b in zip(toks, toks[1:]))
        assert all(a[1] == b[0] for a, b in zip(qs, qs[1:]))
        ora = OracleStream(wl, seed=3)
        rows = np.arange(wl.Lq)
        q0, q1 = plan.queries
        for step in range(1, 5):
            ora.step()
            for h in range(wl.H):
                o, l = ora.attention(0, h, rows, tokens=plan.tokens)
                parts = [None] * world
                dist.all_gather_object(parts, (o, l))
                mo, ml = lse_merge([p[0][q0:q1] for p in parts], [p[1][q0:q1] for p in parts])
                ref, ref_l = ora.attention(0, h, np.arange(q0, q1))
                np.testing.assert_allclose(mo, ref, rtol=1e-9, atol=1e-12)
                np.testing.assert_allclose(ml, ref_l, rtol=1e-12)
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:  # report to the parent
        errq.put(f"rank {rank}: {e!r}")
        raise


@pytest.mark.parametrize("world", [2, 4, 8])
def test_sp_plans_and_merge_over_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    errq = ctx.SimpleQueue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, errq)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    assert not alive, "a rank did not finish"
    assert not errs, errs
    assert all(p.exitcode == 0 for p in procs)


def test_plan_rejects_uneven_splits():
    from nvfp4_kv_cache_append_b200.sp import SPPlan
    with pytest.raises(ValueError):
        SPPlan(0, 7, 1560, 4680)
    with pytest.raises(ValueError):
        SPPlan(2, 2, 64, 64)
    p = SPPlan(3, 4, 1560, 4680)
    assert p.tokens == (1170, 1560) and p.queries == (3510, 4680)
