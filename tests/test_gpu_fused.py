"""Parity of the fused producer (base logits from the LM head in the same
kernel as the transition bias) against the fp64 oracle (B200).

fp32 output: |got - exact| <= 1e-4 for every element. bf16 output: the
one-rounding rule of ``oracle.checks`` with the fp32 accumulation bound of
the d + r products.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.checks import check_logits
from rank_markov_draft_vanillamarkov_b200 import VanillaMarkov, device_status, last_algo
from rank_markov_draft_vanillamarkov_b200 import _native as N
from rank_markov_draft_vanillamarkov_b200 import workloads as W
from rank_markov_draft_vanillamarkov_b200.build import build

from _helpers import f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    N.load()
    yield


def _run(d, out_dtype=torch.float32, hidden=None, ids=None):
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    h = (d["hidden"] if hidden is None else hidden).cuda()
    x = (d["prev_ids"] if ids is None else ids).cuda()
    got = head.fused_lm_head_logits(h, d["lm_head"].cuda(), token_ids=x, out_dtype=out_dtype)
    used = last_algo()
    torch.cuda.synchronize()
    return got, used, device_status()


def _check(d, got, dtype, hidden=None, ids=None, vchunk=16384):
    """Every element, in vocabulary chunks so that the fp64 LM head stays small."""
    h = f64(d["hidden"] if hidden is None else hidden)
    h = h.reshape(-1, h.shape[-1])
    x = (d["prev_ids"] if ids is None else ids).reshape(-1).numpy()
    w1 = f64(d["w1"])
    v = d["lm_head"].shape[0]
    g = f64(got).reshape(-1, v)
    peak = 0.0
    for v0 in range(0, v, vchunk):
        v1 = min(v, v0 + vchunk)
        lm, w2 = f64(d["lm_head"][v0:v1]), f64(d["w2"][v0:v1])
        exact = oracle.fused_lm_head_exact(h, lm, w1, w2, x)
        acc = oracle.fused_accumulation_bound(h, lm, w1, w2, x) if dtype == "bf16" else None
        rep = check_logits(g[:, v0:v1], exact, dtype, acc)
        assert rep.ok, f"ids {v0}..{v1 - 1}: {rep.bad} of {rep.n} bad, first {rep.first_bad}, max_abs {rep.max_abs}"
        peak = max(peak, float(np.abs(exact).max()))
    return peak


def _small(rows_blocks, hidden, vocab, rank, out="fp32", seed=0, wstd=0.3):
    return W.FUSED_320.with_(name=f"fused_small_{rows_blocks}_{hidden}_{vocab}_{rank}", batch=1,
                             num_blocks=rows_blocks, vocab=vocab, rank=rank, hidden=hidden, logits_dtype=out,
                             weight_std=wstd, lm_std=0.05, data_seed=seed)


@pytest.mark.parametrize("blocks,hidden,vocab,rank,out", [
    (40, 512, 2056, 64, "fp32"),     # 200 rows: a ragged 72-row tile; ragged last 256-id tile
    (27, 1024, 4096, 128, "bf16"),   # 135 rows
    (66, 200, 1000, 256, "fp32"),    # hidden not a multiple of 64 (zero-filled K tail), 1000 ids
    (26, 64, 264, 16, "bf16"),       # rank 16: one partial K block of W1 / W2; 264 ids
])
def test_fused_small(blocks, hidden, vocab, rank, out):
    wl = _small(blocks, hidden, vocab, rank, out, seed=blocks)
    d = W.make_inputs(wl)
    got, used, st = _run(d, torch.float32 if out == "fp32" else torch.bfloat16)
    assert used == 2 and st == 0
    assert got.shape == (1, blocks, 5, vocab)
    _check(d, got, out)


def test_fused_bias_probe_zero_hidden():
    """hidden = 0: the output is the bias alone, so a kernel that dropped the
    W1 / W2 blocks cannot hide under the LM-head sum."""
    wl = _small(64, 1024, 129280, 128, "fp32", seed=5, wstd=0.02)
    d = W.make_inputs(wl)
    zero = torch.zeros_like(d["hidden"])
    got, used, st = _run(d, hidden=zero)
    assert used == 2 and st == 0
    assert _check(d, got, "fp32", hidden=zero) > 1e-2


def test_fused_strong_bias_full_vocab_bf16():
    wl = _small(64, 1024, 129280, 128, "bf16", seed=6, wstd=0.3)
    d = W.make_inputs(wl)
    got, used, st = _run(d, torch.bfloat16)
    assert used == 2 and st == 0
    _check(d, got, "bf16")


def test_fused_full_size():
    """320 rows x hidden 5120 x 129280 ids x rank 128, fp32 out, every element."""
    d = W.make_inputs(W.FUSED_320)
    got, used, st = _run(d)
    assert used == 2 and st == 0
    assert got.dtype == torch.float32 and got.shape == (4, 16, 5, 129280)
    _check(d, got, "fp32")


def test_fused_out_of_range_ids_report_status():
    wl = _small(30, 256, 2056, 64, "fp32", seed=7)
    d = W.make_inputs(wl)
    ids = d["prev_ids"].clone()
    ids.view(-1)[4] = wl.vocab
    ids.view(-1)[9] = -1
    got, used, st = _run(d, ids=ids)
    assert st & N.DSPARK_STATUS_TOKEN_RANGE
    keep = np.setdiff1d(np.arange(wl.rows), [4, 9])
    sub = {k: d[k] for k in ("w1", "w2", "lm_head")}
    sub["hidden"] = d["hidden"].reshape(-1, wl.hidden)[keep]
    sub["prev_ids"] = ids.reshape(-1)[keep]
    _check(sub, got.reshape(-1, wl.vocab)[torch.from_numpy(keep).cuda()], "fp32")
    # the invalid rows carry the LM-head logits alone (a zero bias)
    bad = torch.tensor([4, 9])
    h = f64(d["hidden"].reshape(-1, wl.hidden)[bad])
    u = h @ f64(d["lm_head"]).T
    assert np.abs(f64(got.reshape(-1, wl.vocab)[bad.cuda()]) - u).max() <= 1e-4


def test_fused_unsupported_shapes_are_refused():
    wl = _small(2, 100, 1000, 64, "fp32", seed=8)  # hidden 100 is not a multiple of 8
    d = W.make_inputs(wl)
    with pytest.raises(RuntimeError):
        _run(d)
    wl = _small(2, 64, 1000, 64, "fp32", seed=8)
    d = W.make_inputs(wl)
    head = VanillaMarkov(d["w1"].float().cuda(), d["w2"].float().cuda())
    with pytest.raises((RuntimeError, ValueError)):
        head.fused_lm_head_logits(d["hidden"].float().cuda(), d["lm_head"].float().cuda(),
                                  token_ids=d["prev_ids"].cuda())


def test_fused_empty_rows():
    wl = _small(1, 64, 1000, 64, "fp32", seed=9)
    d = W.make_inputs(wl)
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    out = head.fused_lm_head_logits(torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda"), d["lm_head"].cuda(),
                                    token_ids=torch.zeros(0, dtype=torch.long, device="cuda"))
    assert out.shape == (0, 1000)
