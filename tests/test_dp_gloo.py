"""Data-parallel host logic on CPU with two gloo ranks: each rank computes the
gradient of its own batch columns (here with the fp64 oracle, on the CPU), the
shared-parameter gradients are all-reduced, and the result must equal the
gradient of the whole batch on one process."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from structured_trainable_laplace_b200 import dp, inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        h = inputs.phased_head(600, 40, 5, seed=3)
        cols = dp.shard_columns(5, rank, world)
        x, g = h["x"][:, cols], h["h"][:, cols]
        gr = oracle.rect_backward(h["a"], h["b"], x, g, h["phi"], h["psi"], transpose=True)
        t = {key: torch.from_numpy(v) for key, v in gr.items()}
        dp.allreduce_param_grads(t)
        w = inputs.sym_small_ties(1)
        B2 = 4
        xs = np.repeat(w["x"], B2, axis=1) * np.arange(1, B2 + 1, dtype=np.float32)
        gs = np.repeat(w["g"], B2, axis=1)
        c2 = dp.shard_columns(B2, rank, world)
        _, ga = oracle.sym_backward(w["a"], xs[:, c2], gs[:, c2])
        tg = {"ga": torch.from_numpy(ga)}
        dp.allreduce_param_grads(tg)
        q.put((rank, {key: v.numpy() for key, v in t.items()}, tg["ga"].numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_allreduce_matches_whole_batch():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    h = inputs.phased_head(600, 40, 5, seed=3)
    ref = oracle.rect_backward(h["a"], h["b"], h["x"], h["h"], h["phi"], h["psi"], transpose=True)
    w = inputs.sym_small_ties(1)
    xs = np.repeat(w["x"], 4, axis=1) * np.arange(1, 5, dtype=np.float32)
    _, ga_ref = oracle.sym_backward(w["a"], xs, np.repeat(w["g"], 4, axis=1))
    for rank, grads, ga in results:
        for key in ("ga", "gb", "gphi", "gpsi"):
            np.testing.assert_allclose(grads[key], ref[key], rtol=1e-12, atol=1e-12, err_msg=key)
        np.testing.assert_allclose(ga, ga_ref, rtol=1e-12, atol=1e-10)


@pytest.mark.parametrize("B,world", [(16, 1), (16, 2), (5, 2), (5, 3), (1, 4)])
def test_shard_columns_partition(B, world):
    cols = [dp.shard_columns(B, r, world) for r in range(world)]
    covered = np.concatenate([np.arange(B)[c] for c in cols])
    np.testing.assert_array_equal(covered, np.arange(B))


class _FakeDist:
    """Stands in for torch.distributed: a group of `world` ranks whose other ranks
    all hold `other` times this rank's values; counts the collectives issued."""

    def __init__(self, world, other):
        self.world, self.other, self.calls = world, other, []

    def is_initialized(self):
        return True

    def get_world_size(self, group=None):
        return self.world

    def all_reduce(self, t, group=None):
        self.calls.append(t.numel())
        t.mul_(1 + self.other * (self.world - 1))


def test_param_grads_reduced_in_one_collective():
    """Every shared-parameter gradient present goes through one flat all-reduce and
    comes back in place with its own shape; vector gradients are left alone."""
    rng = np.random.default_rng(0)
    grads = {"gx": torch.from_numpy(rng.standard_normal((7, 3))), "ga": torch.from_numpy(rng.standard_normal(7)),
             "gb": torch.from_numpy(rng.standard_normal(5)), "gphi": torch.from_numpy(rng.standard_normal(7)),
             "gpsi": torch.from_numpy(rng.standard_normal(5))}
    before = {k: v.clone() for k, v in grads.items()}
    fake = _FakeDist(world=3, other=2.0)
    out = dp.allreduce_param_grads(grads, dist=fake)
    assert out is grads
    assert fake.calls == [7 + 5 + 7 + 5]
    for key in ("ga", "gb", "gphi", "gpsi"):
        np.testing.assert_array_equal(grads[key].numpy(), 5.0 * before[key].numpy())
    np.testing.assert_array_equal(grads["gx"].numpy(), before["gx"].numpy())
    one = {"ga": torch.ones(4)}
    fake1 = _FakeDist(world=2, other=1.0)
    dp.allreduce_param_grads(one, dist=fake1)
    assert fake1.calls == [4] and torch.equal(one["ga"], torch.full((4,), 2.0))
