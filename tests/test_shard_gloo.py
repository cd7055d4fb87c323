"""The sharded data-parallel step's protocol, run by two real processes.

Two gloo ranks on the CPU (no GPU): each makes its own gradient, the ranks
exchange gradients, each steps only its own shard (opt2s_shard_range) with
the rank-order mean of the gradients, and the ranks exchange the updated
shards.  The assembled parameters and the state shards must equal a single
process stepping the whole buffer with the averaged gradient, bit for bit.
The arithmetic here is the CPU oracle's (this checks the partition and the
exchange that the fused kernel implements over peer memory; the kernel itself
is checked against the same oracle on a GPU with emulated ranks).
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

N, STEPS = 100_003, 3
HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, beta3=0.999, alpha=5.0, weight_decay=0.01)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _grads(rank, step, dtype):
    from elementwise_optimizer_b200 import synth
    g = synth.mixed_magnitude(synth.SEED_BASE + 50, (rank, step), N, zero_frac=0.05)
    return synth.to_storage(g, dtype)


def _init_params(dtype):
    from elementwise_optimizer_b200 import synth
    return synth.to_storage(synth.normal(synth.SEED_BASE + 51, (0,), N, 1.0), dtype)


def _rank_main(rank, world, port, dtype, algo, out_dir):
    import torch
    import torch.distributed as dist
    import oracle
    from elementwise_optimizer_b200 import binding as B
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        start, length = B.opt2s_shard_range(N, world, rank)
        params = _init_params(dtype)
        s1 = np.zeros(2 * length if algo == "ademamix" else length, np.float32)
        s2 = np.zeros(length, np.float32)
        for t in range(1, STEPS + 1):
            mine = _grads(rank, t, dtype)
            gathered = [torch.empty(N * mine.itemsize, dtype=torch.uint8) for _ in range(world)]
            dist.all_gather(gathered, torch.from_numpy(mine.view(np.uint8).copy()))
            grads = [g.numpy().view(mine.dtype) for g in gathered]
            avg = oracle.average_grads([g[start:start + length] for g in grads], dtype)
            shard = params[start:start + length].copy()
            oracle.step_f32_fgrad(shard, avg, s1, s2, dtype=dtype, algo=algo, step=t,
                                  skip_zeros=True, **HYPER)
            # all-gather of the updated shards (padded to the largest shard)
            width = max(B.opt2s_shard_range(N, world, r)[1] for r in range(world)) * mine.itemsize
            buf = np.zeros(width, np.uint8)
            buf[:length * mine.itemsize] = shard.view(np.uint8)
            out = [torch.empty(width, dtype=torch.uint8) for _ in range(world)]
            dist.all_gather(out, torch.from_numpy(buf))
            for r in range(world):
                a, n = B.opt2s_shard_range(N, world, r)
                params[a:a + n] = out[r].numpy()[:n * mine.itemsize].view(mine.dtype)
        np.save(os.path.join(out_dir, f"params_{rank}.npy"), params.view(np.uint8))
        np.save(os.path.join(out_dir, f"s1_{rank}.npy"), s1)
        np.save(os.path.join(out_dir, f"s2_{rank}.npy"), s2)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype,algo", [("f32", "adam"), ("bf16", "ademamix")])
def test_two_ranks_equal_one_process(tmp_path, dtype, algo):
    import oracle
    from elementwise_optimizer_b200 import binding as B
    B.lib()
    oracle.build()
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, dtype, algo, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    # one process, whole buffer
    params = _init_params(dtype)
    s1 = np.zeros(2 * N if algo == "ademamix" else N, np.float32)
    s2 = np.zeros(N, np.float32)
    for t in range(1, STEPS + 1):
        avg = oracle.average_grads([_grads(r, t, dtype) for r in range(world)], dtype)
        oracle.step_f32_fgrad(params, avg, s1, s2, dtype=dtype, algo=algo, step=t,
                              skip_zeros=True, **HYPER)
    for r in range(world):
        got = np.load(tmp_path / f"params_{r}.npy")
        assert np.array_equal(got, params.view(np.uint8))
        a, n = B.opt2s_shard_range(N, world, r)
        ref1 = np.concatenate([s1[a:a + n], s1[N + a:N + a + n]]) if algo == "ademamix" else s1[a:a + n]
        assert np.array_equal(np.load(tmp_path / f"s1_{r}.npy"), ref1)
        assert np.array_equal(np.load(tmp_path / f"s2_{r}.npy"), s2[a:a + n])


def _leaving_rank_main(rank, world, port, out_dir):
    """Rank 1 leaves after step 1 (between steps, nothing in flight); rank 0
    must learn of it from its next collective, which fails within the
    process group's short timeout instead of waiting forever."""
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    status = "no failure seen"
    try:
        for t in (1, 2, 3):
            if rank == 1 and t == 2:
                os._exit(3)                  # leaves between steps
            buf = [torch.empty(4) for _ in range(world)]
            dist.all_gather(buf, torch.full((4,), float(t)))
    except Exception as exc:                 # the detection this test is about
        status = f"detected: {type(exc).__name__}"
    with open(os.path.join(out_dir, f"status_{rank}.txt"), "w") as f:
        f.write(status)
    os._exit(0)


def test_a_rank_leaving_between_steps_is_detected(tmp_path):
    import time
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_leaving_rank_main, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    t0 = time.time()
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert procs[1].exitcode == 3
    assert procs[0].exitcode == 0
    assert (tmp_path / "status_0.txt").read_text().startswith("detected")
    assert time.time() - t0 < 100
