"""Multi-process host logic of N-GPU runs, on CPU with the gloo backend.

N GPUs run N replicas, each on its own slice of the batch (the mixer's
sequences are independent).  These tests run two ranks as processes and check
the pieces that involve more than one rank: the slices cover the global batch
and give the same results as one run over it, the timing reduction is the max
over ranks on every rank, the job rate counts every rank's tokens, and a rank
that never joins makes the others' barrier fail within the group's timeout.
"""
import json
import os
import socket

import numpy as np
import pytest

from mamba_selective_scan_jamba_b200 import replicas


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))


def _replica_rank(rank: int, world: int, port: int, out_dir: str) -> None:
    import torch.distributed as dist
    import oracle
    from mamba_selective_scan_jamba_b200 import synth
    _env(rank, world, port)
    replicas.init("gloo", 30.0)
    try:
        base = synth.Workload("replica_tiny", 2, 24, 64, 8, "bf16", seed=5, extra=True)
        wall = base.with_(batch=base.batch * world)
        lo, hi = replicas.shard(base.batch, rank)
        W = synth.make_weights(base)
        A = synth.make_activations(wall, lo, hi)
        y, fs, fc = oracle.mixer_fwd(oracle.dims_of(base), A["x"], A["z"], W,
                                     A["init_conv_state"], A["init_ssm_state"])
        ms = replicas.max_over_ranks(1.5 * (rank + 1))
        rate = replicas.job_rate(base.batch * base.seqlen, world, ms)
        replicas.barrier()
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), y=y, fs=fs, fc=fc)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"lo": lo, "hi": hi, "ms": ms, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def _absent_peer_rank(rank: int, world: int, port: int, out_dir: str) -> None:
    import torch.distributed as dist
    _env(rank, world, port)
    replicas.init("gloo", 3.0)
    replicas.barrier()                      # both ranks meet once
    if rank == 1:
        return                              # rank 1 leaves between steps
    err = ""
    try:
        replicas.barrier()                  # rank 0's next step waits for it
    except Exception as e:  # noqa: BLE001 - any error ends the wait, which is the point
        err = type(e).__name__ or "error"
    with open(os.path.join(out_dir, "rank0.json"), "w") as f:
        json.dump({"error": err}, f)
    try:
        dist.destroy_process_group()
    except Exception:  # noqa: BLE001
        pass


def test_shard_slices():
    assert replicas.shard(8, 0) == (0, 8)
    assert replicas.shard(8, 3) == (24, 32)
    assert replicas.job_rate(1000, 4, 2.0) == pytest.approx(2e6)
    with pytest.raises(ValueError):
        replicas.shard(-1, 0)
    with pytest.raises(ValueError):
        replicas.job_rate(1, 1, 0.0)


def test_max_over_ranks_without_group_is_identity():
    assert replicas.max_over_ranks(3.25) == 3.25


def test_two_replicas_match_one_run(tmp_path):
    import torch.multiprocessing as mp
    import oracle
    from mamba_selective_scan_jamba_b200 import synth
    world = 2
    mp.spawn(_replica_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    meta = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    # slices tile the global batch in rank order
    assert [(m["lo"], m["hi"]) for m in meta] == [(0, 2), (2, 4)]
    # the timing reduction gives every rank the slowest rank's time
    assert all(m["ms"] == 3.0 for m in meta)
    assert all(m["rate"] == pytest.approx(2 * 2 * 24 / 3.0e-3) for m in meta)
    # one run over the global batch gives the same results, sequence by sequence
    base = synth.Workload("replica_tiny", 2, 24, 64, 8, "bf16", seed=5, extra=True)
    wall = base.with_(batch=4)
    A = synth.make_activations(wall)
    y, fs, fc = oracle.mixer_fwd(oracle.dims_of(wall), A["x"], A["z"], synth.make_weights(wall),
                                 A["init_conv_state"], A["init_ssm_state"])
    np.testing.assert_array_equal(np.concatenate([p["y"] for p in parts]), y)
    np.testing.assert_array_equal(np.concatenate([p["fs"] for p in parts]), fs)
    np.testing.assert_array_equal(np.concatenate([p["fc"] for p in parts]), fc)


def test_absent_rank_ends_the_barrier_with_an_error(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.spawn(_absent_peer_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world,
             join=True)
    res = json.load(open(tmp_path / "rank0.json"))
    assert res["error"], "rank 0's barrier returned although rank 1 never joined"
