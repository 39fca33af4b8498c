"""Parity of the CUDA transition bias (the head's forward: bias alone plus
embeddings, dspark_markov_transition_logits) against the fp64 oracle (B200).

The bias is checked element by element under the tolerance rule of
``oracle.checks`` (bf16: within one ulp of the correctly rounded value and
within 2e-2 + ulp/2 of the exact sum; fp32: 1e-4), with the base taken as
zero; the embeddings are exact copies of W1's rows.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import markov as om
from oracle.checks import check_logits
from rank_markov_draft_vanillamarkov_b200 import VanillaMarkov, device_status, last_algo, set_algo
from rank_markov_draft_vanillamarkov_b200 import _native as N
from rank_markov_draft_vanillamarkov_b200 import workloads as W
from rank_markov_draft_vanillamarkov_b200.build import build

from _helpers import f64

pytestmark = pytest.mark.gpu

TC, GEN = N.DSPARK_ALGO_TENSOR_CORE, N.DSPARK_ALGO_GENERIC


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    N.load()
    yield
    set_algo(N.DSPARK_ALGO_AUTO)


def _run(w1, w2, ids, algo, with_embeddings=True):
    set_algo(algo)
    head = VanillaMarkov(w1.cuda(), w2.cuda())
    tr, emb = head.transition_logits(ids.cuda(), with_embeddings=with_embeddings)
    torch.cuda.synchronize()
    return tr, emb, last_algo(), device_status()


def _check(w1, w2, ids, tr, emb, dtype="bf16"):
    i = ids.reshape(-1).numpy()
    vocab = w2.shape[0]
    zero = np.zeros((i.size, vocab))
    exact = om.exact_block_logits(zero, f64(w1), f64(w2), i)
    acc = oracle.accumulation_bound(zero, f64(w1), f64(w2), i)
    rep = check_logits(f64(tr).reshape(exact.shape), exact, dtype, acc)
    assert rep.ok, (rep.bad, rep.n, rep.first_bad, rep.max_abs)
    if emb is not None:
        assert torch.equal(emb.cpu().reshape(i.size, -1), w1[torch.from_numpy(i)])


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
@pytest.mark.parametrize("rows,vocab,rank", [(200, 1000, 64), (330, 2056, 256), (135, 4096, 128)])
def test_transition_small(rows, vocab, rank, algo):
    """Ragged row and vocabulary tiles; 330 rows at rank 256 take the
    tensor-core kernel's per-unit (non-resident) gather."""
    wl = W.APPLY_320.with_(vocab=vocab, rank=rank, weight_std=0.3, data_seed=rows)
    g = torch.Generator().manual_seed(rows)
    w1, w2 = W.make_weights(wl, g)
    ids = W.zipf_ids(g, rows, vocab)
    tr, emb, used, st = _run(w1, w2, ids, algo)
    assert used == (2 if algo == TC else 1) and st == 0
    assert tr.shape == (rows, vocab) and tr.dtype == torch.bfloat16 and emb.shape == (rows, rank)
    _check(w1, w2, ids, tr, emb)


def test_transition_320_full_size_block_shape():
    """320 ids shaped (4, 16, 5) at V = 129280, rank 128 (the teacher-forced
    apply's shapes), every element, no embeddings requested."""
    d = W.make_inputs(W.APPLY_320)
    tr, emb, used, st = _run(d["w1"], d["w2"], d["prev_ids"], N.DSPARK_ALGO_AUTO, with_embeddings=False)
    assert used == 2 and st == 0 and emb is None
    assert tr.shape == (4, 16, 5, 129280)
    _check(d["w1"], d["w2"], d["prev_ids"], tr, None)


def test_transition_fp32_weights_generic():
    wl = W.TINY_FP32
    g = torch.Generator().manual_seed(0)
    w1, w2 = W.make_weights(wl, g)
    ids = W.uniform_ids(g, 10, wl.vocab)
    tr, emb, used, st = _run(w1, w2, ids, N.DSPARK_ALGO_AUTO)
    assert used == 1 and st == 0 and tr.dtype == torch.float32
    _check(w1, w2, ids, tr, emb, dtype="fp32")


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_transition_out_of_range_ids(algo):
    """An id outside [0, V) gives zero rows and the TOKEN_RANGE status; the
    other rows are still correct."""
    wl = W.APPLY_320.with_(vocab=2056, rank=128, weight_std=0.3)
    g = torch.Generator().manual_seed(9)
    w1, w2 = W.make_weights(wl, g)
    ids = W.uniform_ids(g, 150, 2056)
    ids[3], ids[140] = 2056, -1
    tr, emb, used, st = _run(w1, w2, ids, algo)
    assert st & N.DSPARK_STATUS_TOKEN_RANGE
    assert (tr[3] == 0).all() and (tr[140] == 0).all() and (emb[3] == 0).all() and (emb[140] == 0).all()
    keep = torch.from_numpy(np.setdiff1d(np.arange(150), [3, 140]))
    _check(w1, w2, ids[keep], tr.cpu()[keep], emb.cpu()[keep])
    assert device_status() == 0
