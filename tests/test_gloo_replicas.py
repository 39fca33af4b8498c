"""The multi-GPU host logic, run as two gloo ranks on the CPU.

Each rank takes its slice of the rows or blocks (sharding.py) and runs a head
on it; the slices gathered on every rank must equal the unsharded result. The
head here is a CPU stand-in backed by the oracle, since this machine has no
GPU; the CUDA head has the same two methods.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from rank_markov_draft_vanillamarkov_b200 import sharding
from rank_markov_draft_vanillamarkov_b200 import workloads as W


class OracleHead:
    def __init__(self, w1, w2):
        self.w1 = w1.to(torch.float64).numpy()
        self.w2 = w2.to(torch.float64).numpy()

    def apply_block_logits(self, base_logits, *, token_ids):
        return torch.from_numpy(oracle.apply_block_logits(base_logits.to(torch.float64).numpy(), self.w1, self.w2,
                                                          token_ids.numpy(), "bf16"))

    def apply_block_logits_backward(self, grad_out, *, token_ids):
        g1, g2 = oracle.apply_block_logits_backward(grad_out.to(torch.float64).numpy(), self.w1, self.w2,
                                                    token_ids.numpy())
        return torch.from_numpy(g1), torch.from_numpy(g2)

    def sample_block_tokens(self, base_logits, *, first_prev_token_ids, temperature=0.0, seed=0):
        t, c = oracle.sample_block_tokens(base_logits.to(torch.float64).numpy(), self.w1, self.w2,
                                          first_prev_token_ids.numpy(), "bf16", temperature, seed)
        return torch.from_numpy(t), torch.from_numpy(c)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.small_variants()[0]
        d = W.make_inputs(wl)
        head = OracleHead(d["w1"], d["w2"])
        part = sharding.apply_block_logits_shard(head, d["base"], d["prev_ids"], rank, world)
        parts = [None] * world
        dist.all_gather_object(parts, part)
        full_apply = torch.cat(parts, 0)

        swl = W.GREEDY.with_(batch=7, vocab=1000, rank=64, weight_std=0.3, data_seed=2)
        s = W.make_inputs(swl)
        sh = OracleHead(s["w1"], s["w2"])
        tk, _ = sharding.sample_block_tokens_shard(sh, s["base"], s["first_prev"], rank, world, 0.0)
        toks = [None] * world
        dist.all_gather_object(toks, tk)

        tt, tc = sharding.sample_block_tokens_shard(sh, s["base"], s["first_prev"], rank, world, 0.8, seed=11)
        temps = [None] * world
        dist.all_gather_object(temps, (tt, tc))

        t = torch.tensor([float(rank + 1) * 1.5], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            q.put((full_apply.numpy(), torch.cat(toks, 0).numpy(),
                   [(a.numpy(), b.numpy()) for a, b in temps], float(t.item())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_shards_match_unsharded():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    full_apply, toks, temps, tmax = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    wl = W.small_variants()[0]
    d = W.make_inputs(wl)
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    want = oracle.apply_block_logits(f(d["base"]), f(d["w1"]), f(d["w2"]), d["prev_ids"].numpy(), "bf16")
    np.testing.assert_array_equal(full_apply, want)

    swl = W.GREEDY.with_(batch=7, vocab=1000, rank=64, weight_std=0.3, data_seed=2)
    s = W.make_inputs(swl)
    wt, _ = oracle.sample_block_tokens(f(s["base"]), f(s["w1"]), f(s["w2"]), s["first_prev"].numpy(), "bf16", 0.0)
    np.testing.assert_array_equal(toks, wt)

    # temperature: each shard is a valid Gumbel-max draw under its own seed,
    # and the two shards' block 0 do not share noise
    lo1, _ = sharding.shard_range(7, 1, 2)
    assert sharding.shard_seed(11, 0) != sharding.shard_seed(11, lo1)
    for r, (tt, tc) in enumerate(temps):
        lo, hi = sharding.shard_range(7, r, 2)
        seed = sharding.shard_seed(11, lo)
        for b in range(hi - lo):
            for k in range(swl.proposal_len):
                sc = oracle.temperature_scores(tc[b, k], 0.8, seed, b, k)
                assert tt[b, k] == int(np.argmax(sc))
    assert tmax == 3.0


def test_shard_range_tiles_exactly():
    for n in (0, 1, 7, 320, 2561):
        for world in (1, 2, 3, 8):
            spans = [sharding.shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sharding.shard_range(4, 2, 2)


def _backward_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.small_variants()[0]  # 2 x 20 blocks x 5, V = 1000, Zipf ids (shared across the two slices)
        d = W.make_inputs(wl)
        grad = torch.randn(d["base"].shape, generator=torch.Generator().manual_seed(4), dtype=torch.float64)
        head = OracleHead(d["w1"], d["w2"])
        g1, g2 = sharding.apply_block_logits_backward_shard(head, grad, d["prev_ids"], rank, world)
        q.put((rank, g1.numpy(), g2.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_backward_all_reduce_matches_full_batch():
    """Each rank differentiates its half of the batch; after the all-reduce
    both ranks hold the full-batch gradients of W1 and W2."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_backward_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = W.small_variants()[0]
    d = W.make_inputs(wl)
    grad = torch.randn(d["base"].shape, generator=torch.Generator().manual_seed(4), dtype=torch.float64)
    want1, want2 = oracle.apply_block_logits_backward(grad.numpy(), d["w1"].double().numpy(),
                                                      d["w2"].double().numpy(), d["prev_ids"].numpy())
    for _, g1, g2 in got:
        np.testing.assert_allclose(g1, want1, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g2, want2, rtol=1e-12, atol=1e-12)
