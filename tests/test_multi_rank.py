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


def _tp_worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from latent_kv_cache_flash_b200 import multi, synth
    from oracle import gqla_oracle as O
    d = synth.Dims(n_h=8, G=4, d_nope=16, d_rope=8, d_v=16, r=32, s_q=2, dtype="f32")
    inp = synth.make_inputs(synth.Workload("tp", d, batch=2, seq_len=40, seed=3), "cpu", seq_lens=[40, 9])
    sh = multi.tp_shard(inp, world, rank)
    sd = sh.dims
    outs = []
    for form in ("gqa", "absorb"):
        c = [sh.logical_latent(b)[:, :sd.r].double().numpy() for b in range(2)]
        kr = [sh.logical_latent(b)[:, sd.r:].double().numpy() for b in range(2)]
        o, l = O.decode_batch(sh.q.double().numpy(), c, kr, sh.W_uk.double().numpy(), sh.W_uv.double().numpy(),
                              sh.seq_lens_host, sd.softmax_scale, form=form)
        got = [torch.zeros((2, 2, 4, 16), dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, torch.from_numpy(np.ascontiguousarray(o)))
        outs.append(torch.cat(got, dim=2).numpy())
    if rank == 0:
        c = [inp.logical_latent(b)[:, :d.r].double().numpy() for b in range(2)]
        kr = [inp.logical_latent(b)[:, d.r:].double().numpy() for b in range(2)]
        full = O.decode_batch(inp.q.double().numpy(), c, kr, inp.W_uk.double().numpy(), inp.W_uv.double().numpy(),
                              inp.seq_lens_host, d.softmax_scale, form="gqa")[0]
        results["err"] = max(float(np.max(np.abs(o - full))) for o in outs)
        results["shape"] = (sd.n_h, sd.G, tuple(sh.q.shape), tuple(sh.W_uk.shape))
    dist.barrier()
    dist.destroy_process_group()


def test_group_tensor_parallel_two_gloo_ranks():
    """Each rank decodes its two groups' heads (the oracle, both forms); the
    gathered heads equal the unsharded decode: no exchange inside attention."""
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_tp_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert results["shape"] == (4, 2, (2, 2, 4, 24), (2, 32, 16))
    assert results["err"] < 1e-12


def test_tp_groups_and_cache_per_rank():
    from latent_kv_cache_flash_b200 import build, gqla, multi, synth
    assert [multi.tp_groups(16, 8, r) for r in (0, 7)] == [(0, 2), (14, 16)]
    with pytest.raises(ValueError):
        multi.tp_groups(8, 3, 0)
    build.build()
    d = synth.Dims(n_h=128, G=16, d_nope=128, d_rope=64, d_v=128, r=512)
    inp = synth.make_inputs(synth.Workload("tp", d, batch=1, seq_len=8, seed=0), "cpu")
    sh = multi.tp_shard(inp, 8, 3)
    full_g = gqla.gqla_cache_bytes_per_token(gqla.make_dims(d), gqla.GQLA_PATH_GQA)
    rank_g = gqla.gqla_cache_bytes_per_token(gqla.make_dims(sh.dims), gqla.GQLA_PATH_GQA)
    rank_a = gqla.gqla_cache_bytes_per_token(gqla.make_dims(sh.dims), gqla.GQLA_PATH_ABSORB)
    # GQA: each of 8 ranks holds 1/8 of the expanded cache (no redundancy);
    # absorb: every rank holds the whole latent row
    assert rank_g * 8 == full_g == 16 * 320 * 2
    assert rank_a == gqla.gqla_cache_bytes_per_token(gqla.make_dims(d), gqla.GQLA_PATH_ABSORB) == 576 * 2
    assert torch.equal(sh.q, inp.q[:, :, 3 * 16:4 * 16]) and torch.equal(sh.W_uk, inp.W_uk[6:8])
    assert sh.dims.softmax_scale == d.softmax_scale
