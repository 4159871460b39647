"""Host logic of the multi-rank run on CPU: the split of the (batch, head) problems over ranks, the global
keying of the draws (bh_offset), and the max-over-ranks timing, with two gloo ranks.

The problems of the method are independent ("HyperAttention: Long-context Attention in Near-Linear Time",
research-map summary, "Approach": each head is hashed, sorted and attended on its own), so the job needs no
data exchange: the outputs gathered from the ranks must equal one run over all problems, bit for bit.
The per-rank compute here is the oracle (CPU); the GPU counterpart is tests/test_gpu_shard.py.
"""
import os
import socket

import numpy as np
import pytest

from approximate_long_context_b200 import shard
from approximate_long_context_b200 import workload as wl

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("total,world", [(0, 1), (1, 1), (5, 2), (7, 3), (2, 4), (64, 8), (65, 8)])
def test_shard_ranges_cover_once(total, world):
    seen = []
    sizes = []
    for r in range(world):
        s = shard.shard_problems(total, world, r)
        assert s.offset == (seen[-1] + 1 if seen else 0) or s.count == 0
        seen.extend(range(s.offset, s.offset + s.count))
        sizes.append(s.count)
    assert seen == list(range(total))
    assert max(sizes) - min(sizes) <= 1


def test_weak_shard():
    for world in (1, 2, 4, 8):
        for r in range(world):
            s = shard.weak_shard(32, world, r)
            assert (s.offset, s.count) == (32 * r, 32)


def test_shard_rejects_bad_requests():
    for args in [(4, 0, 0), (4, 2, 2), (4, 2, -1), (-1, 1, 0)]:
        with pytest.raises(ValueError):
            shard.shard_problems(*args)


def test_max_over_ranks_single_process():
    assert shard.max_over_ranks(3.25) == 3.25


# ---------------------------------------------------------------------------- two gloo ranks

N, D, G = 256, 16, 5           # rows, head dim, problems of the whole job (uneven over 2 ranks)
KW = dict(block=64, m=32, r=6, causal=False, seed=77)
DATA_SEED = 0xABC


def _run_problem(Q, K, V, g, ora, sampling="uniform"):
    return ora.forward(wl.as_f32(Q), wl.as_f32(K), wl.as_f32(V), bh=g, sampling=sampling, **KW)["O"]


def _rank_main(rank, world, port, out_dir, sampling):
    import torch.distributed as dist
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        s = shard.shard_problems(G, world, rank)
        heads = range(s.offset, s.offset + s.count)
        Q, K, V = wl.make_inputs(N, D, G, data_seed=DATA_SEED, dtype="fp32", heads=heads)
        outs = [_run_problem(Q[i], K[i], V[i], g, oracle, sampling) for i, g in enumerate(heads)]
        local = np.stack(outs) if outs else np.zeros((0, N, D))
        gathered = [None] * world
        dist.all_gather_object(gathered, (s.offset, local))
        t = shard.max_over_ranks(1.5 + rank)
        if rank == 0:
            np.save(os.path.join(out_dir, "job.npy"), np.concatenate([a for _, a in sorted(gathered, key=lambda x: x[0])]))
            np.save(os.path.join(out_dir, "tmax.npy"), np.array([t]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


@pytest.mark.parametrize("sampling", ["uniform", "rownorm"])
def test_two_gloo_ranks_equal_one_run(tmp_path, ora, sampling):
    """Both samplings key their draws by the global problem index (the row-norm draws also by the problem's own
    value rows), so split runs equal one run."""
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), sampling), nprocs=world, join=True,
                       start_method="spawn")
    job = np.load(tmp_path / "job.npy")
    assert np.load(tmp_path / "tmax.npy")[0] == 2.5           # the slowest rank's time
    Q, K, V = wl.make_inputs(N, D, G, data_seed=DATA_SEED, dtype="fp32")
    whole = np.stack([_run_problem(Q[g], K[g], V[g], g, ora, sampling) for g in range(G)])
    assert job.shape == whole.shape
    assert np.array_equal(job, whole)


def test_problem_index_keys_the_draws(ora):
    """A rank that ignored its offset (keying its draws by local index) would give a different result:
    the check above can fail."""
    Q, K, V = wl.make_inputs(N, D, 1, data_seed=DATA_SEED, dtype="fp32", heads=[3])
    for sampling in ("uniform", "rownorm"):
        a = _run_problem(Q[0], K[0], V[0], 3, ora, sampling)
        b = _run_problem(Q[0], K[0], V[0], 0, ora, sampling)
        assert not np.array_equal(a, b)


def test_backward_shards_by_problem(ora):
    """The backward pass of a problem depends only on its own inputs and global index: per-rank slices of the
    job's gradients equal the whole job's (each rank runs the problems of its range with their global index)."""
    Q, K, V = wl.make_inputs(N, D, G, data_seed=DATA_SEED, dtype="fp32")
    dO = np.random.default_rng(4).standard_normal((G, N, D)).astype(np.float32)
    kw = dict(block=64, m=32, r=6, causal=False, seed=77)
    whole = [ora.backward(Q[g], K[g], V[g], dO[g], bh=g, **kw)["dK"] for g in range(G)]
    for world in (2, 3):
        for rank in range(world):
            s = shard.shard_problems(G, world, rank)
            for i, g in enumerate(range(s.offset, s.offset + s.count)):
                Qs, Ks, Vs = wl.make_inputs(N, D, G, data_seed=DATA_SEED, dtype="fp32", heads=[g])
                got = ora.backward(Qs[0], Ks[0], Vs[0], dO[g], bh=g, **kw)["dK"]
                assert np.array_equal(got, whole[g])
