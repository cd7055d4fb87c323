"""The sharded step across processes, through real peer mappings.

Two processes, one rank each, on the GPUs this machine has (both on one GPU
when only one is visible; the kernels of the two processes never wait on one
another, they are ordered by host barriers).  Each rank owns a flat param
buffer (the same initial values on every rank) and its own gradients; the
buffers are mapped into the other process with CUDA IPC (PeerBuffers:
opt2s_ipc_export / opt2s_ipc_open), and each rank runs opt2s_shard_step on
its shard, between two gloo barriers.  After every step each rank's whole
param buffer must equal the oracle's single-process step of the rank-order
mean gradient, bit for bit, and its shard state the oracle's state slice.
"""
import os
import socket

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

N, STEPS = 1_000_003, 3
HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, beta3=0.999, alpha=5.0, weight_decay=0.01)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _grads(rank, step, dtype):
    from elementwise_optimizer_b200 import synth
    g = synth.mixed_magnitude(synth.SEED_BASE + 60, (rank, step), N, zero_frac=0.05)
    return synth.to_storage(g, dtype)


def _rank_main(rank, world, port, dtype, algo, out_dir):
    import datetime
    import torch.distributed as dist
    import oracle
    from elementwise_optimizer_b200 import binding as B
    from elementwise_optimizer_b200 import shard, synth
    from tests.gpu_support import storage_bits, to_device_storage
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dev = torch.device("cuda", rank % torch.cuda.device_count())
    torch.cuda.set_device(dev)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ok = False
    peers = None
    try:
        init = synth.from_storage(synth.to_storage(synth.normal(synth.SEED_BASE + 61, (0,), N, 1.0),
                                                   dtype), dtype)
        param = to_device_storage(init, dtype, dev)
        grad = torch.empty_like(param)
        peers = shard.PeerBuffers(param, grad)
        st = shard.ShardedStep(peers.params, peers.grads, rank, algo)
        h = B.make_hyper(algo, skip_zeros=True, **HYPER)
        # the oracle: one process stepping the whole buffer with the mean gradient
        hp = synth.to_storage(init, dtype)
        hs1 = np.zeros(2 * N if algo == "ademamix" else N, np.float32)
        hs2 = np.zeros(N, np.float32)
        start, length = st.start, st.length
        ok_all = True
        for t in range(1, STEPS + 1):
            grad.copy_(to_device_storage(synth.from_storage(_grads(rank, t, dtype), dtype), dtype, dev))
            torch.cuda.synchronize()
            dist.barrier()                      # every rank's gradient is complete
            st.step(h, t)
            torch.cuda.synchronize()
            dist.barrier()                      # every shard's params are written
            avg = oracle.average_grads([_grads(q, t, dtype) for q in range(world)], dtype)
            oracle.step_f32_fgrad(hp, avg, hs1, hs2, dtype=dtype, algo=algo, step=t,
                                  skip_zeros=True, **HYPER)
            s1 = hs1[start:start + length]
            if algo == "ademamix":
                s1 = np.concatenate([s1, hs1[N + start:N + start + length]])
            mine = (np.array_equal(storage_bits(param), hp.view(np.uint32 if dtype == "f32" else np.uint16))
                    and np.array_equal(st.state1.cpu().numpy(), s1)
                    and np.array_equal(st.state2.cpu().numpy(), hs2[start:start + length]))
            # every rank learns whether all agree before anyone steps again, so
            # no rank leaves (and frees its mapped buffers) while another steps
            flag = torch.tensor([1 if mine else 0], dtype=torch.int32)
            dist.all_reduce(flag, op=dist.ReduceOp.MIN)
            ok_all = ok_all and mine
            if int(flag.item()) == 0:
                break
        assert ok_all
        ok = True
    finally:
        torch.cuda.synchronize()
        try:
            dist.barrier()                      # no rank unmaps while a peer still steps
        finally:
            if peers is not None:
                peers.close()
            dist.destroy_process_group()
        with open(os.path.join(out_dir, f"rank{rank}"), "w") as f:
            f.write("ok" if ok else "fail")


@pytest.mark.parametrize("dtype,algo", [("f32", "adam"), ("bf16", "ademamix")])
def test_two_processes_step_their_shards_over_ipc(tmp_path, dtype, algo):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from elementwise_optimizer_b200 import _build
    _build.build()
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, dtype, algo, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
    results = [open(tmp_path / f"rank{r}").read() if (tmp_path / f"rank{r}").exists() else "missing"
               for r in range(world)]
    assert results == ["ok"] * world, results
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


def _bench_rank(rank, world, port, out_dir):
    import datetime
    import json
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dev = torch.device("cuda", rank % torch.cuda.device_count())
    torch.cuda.set_device(dev)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = bench.shard_measure(dev, world, rank, numel=4_000_037, steps=3, warmup=1)
        with open(os.path.join(out_dir, f"bench{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_bench_shard_leg_runs_across_processes(tmp_path):
    """The bench's sharded-step leg (run at N > 1): peer mappings, barriers and
    the max-over-ranks time, with two processes."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import json
    import torch.multiprocessing as mp
    from elementwise_optimizer_b200 import _build
    _build.build()
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_bench_rank, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(2):
        res = json.load(open(tmp_path / f"bench{r}.json"))
        assert "error" not in res, res
        assert res["ms_per_step"] > 0 and res["nvlink_bytes_per_rank"] == 8 * 4_000_037 // 2
