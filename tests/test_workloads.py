"""The seeded input generators produce the shapes and distributions the
workloads name, deterministically."""
import numpy as np
import torch

from rank_markov_draft_vanillamarkov_b200 import workloads as W


def test_apply_320_shapes_and_determinism():
    a = W.make_inputs(W.APPLY_320)
    b = W.make_inputs(W.APPLY_320)
    assert a["base"].shape == (4, 16, 5, 129280) and a["base"].dtype == torch.bfloat16
    assert a["w1"].shape == (129280, 128) and a["w2"].shape == (129280, 128)
    assert a["prev_ids"].shape == (4, 16, 5) and a["prev_ids"].dtype == torch.int64
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert abs(float(a["w1"].float().std()) - 0.02) < 1e-3
    assert abs(float(a["base"].float().std()) - 2.0) < 2e-2


def test_zipf_ids_favour_small_ranks():
    g = torch.Generator().manual_seed(0)
    ids = W.zipf_ids(g, 200_000, 129280, 1.1).numpy()
    assert ids.min() >= 0 and ids.max() < 129280
    c = np.bincount(ids, minlength=10)
    assert c[0] > c[1] > c[3] > c[9]
    # p(0)/p(1) = 2^1.1
    assert abs(c[0] / c[1] - 2 ** 1.1) < 0.15


def test_padding_blocks_use_pad_id():
    d = W.make_inputs(W.APPLY_2560.with_(vocab=1024, rank=64))
    pad = d["pad_mask"]
    assert abs(pad.float().mean().item() - 0.2) < 0.01
    assert (d["prev_ids"][pad] == W.PAD_TOKEN_ID).all()


def test_greedy_spike_present():
    wl = W.greedy(8).with_(vocab=4096)
    d = W.make_inputs(wl)
    x = d["base"].float()
    assert d["base"].shape == (8, 5, 4096)
    assert (x.max(-1).values > 6.0).float().mean() > 0.9


def test_byte_counts():
    assert W.APPLY_320.bytes_moved() == 2 * 320 * 129280 * 2 + 129280 * 128 * 2 + 320 * 128 * 2 + 320 * 8
    assert W.APPLY_320.flops() == 2 * 320 * 129280 * 128


def test_transition_workload():
    wl = W.TRANSITION_320
    assert wl.bytes_moved() == 320 * 129280 * 2 + 129280 * 128 * 2 + 2 * 320 * 128 * 2 + 320 * 8
    d = W.make_inputs(wl)
    assert tuple(d["prev_ids"].shape) == (4, 16, 5) and "base" not in d
    assert torch.equal(d["prev_ids"], W.make_inputs(wl)["prev_ids"])
