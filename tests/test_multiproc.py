"""The N>1 path on CPU: two gloo ranks each take their shard of the global
batch (bench.shard_tokens), score it independently (here with the oracle, the
device path being absent on CPU), and the shards gathered by the bench's
end-of-run collective (bench.gather_rows) equal the unsharded run; the job
time is the max over ranks."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import torch.distributed as dist

    import bench
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = synth.workload("tiny", batch=2, prompt=12)
    tok = bench.shard_tokens(w, rank, world)
    om = oracle.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)
    mine = torch.from_numpy(np.stack([om.replay_logprobs(t) for t in tok]))
    gathered = bench.gather_rows(mine, world)  # the bench's end-of-run collective
    slowest = bench.max_over_ranks(float(rank + 1), world)
    if rank == 0:
        np.save(os.path.join(out_dir, "gathered.npy"), gathered.numpy())
        np.save(os.path.join(out_dir, "slowest.npy"), np.array([slowest]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_shards_equal_unsharded(tmp_path):
    import synth
    import oracle
    import bench
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    gathered = np.load(tmp_path / "gathered.npy")
    w = synth.workload("tiny", batch=2, prompt=12)
    full = synth.tokens(w, batch=world * 2, length=12)
    om = oracle.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)
    want = np.stack([om.replay_logprobs(t) for t in full])
    assert np.array_equal(gathered, want)
    assert np.load(tmp_path / "slowest.npy")[0] == 2.0
    # shards partition the global batch
    assert np.array_equal(np.concatenate([bench.shard_tokens(w, r, world) for r in range(world)]), full)
