"""World-size-2 gloo ranks on CPU: the host logic of the one-process-per-GPU
bench (per-rank batches, barrier, max-over-ranks timing, whole-job value)."""
import os
import socket

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


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from latent_kv_cache_flash_b200 import multi, synth
    r, lr, w = multi.rank_info()
    wl = synth.llama3_8b(s_q=1, batch=2, seq_len=64)
    wl.seed = multi.rank_seed(0, r)
    inp = synth.make_inputs(wl, "cpu")
    multi.barrier()
    ms = 10.0 * (r + 1)                       # rank 1 is the slow one
    mx = multi.max_over_ranks(ms)
    results[r] = (r, lr, w, mx, float(inp.q.float().sum()), multi.job_tokens_per_s(2, 5, w, mx))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = results[0], results[1]
    assert (r0[0], r1[0]) == (0, 1) and r0[2] == r1[2] == 2
    assert r0[3] == r1[3] == 20.0               # both ranks see the max
    assert r0[4] != r1[4]                        # independent per-rank batches
    assert r0[5] == r1[5] == pytest.approx(2 * 2 * 5 / 20e-3)
