"""Parity of the CUDA backward of the teacher-forced apply against the fp64
oracle (B200).

The gradients are fp32 sums of products that are exact in fp32 (bf16 x bf16,
or fp32 x fp32 for the fp32 case only up to one rounding each), so the only
error is the fp32 accumulation. A sum of K terms in any order is within about
u * sqrt(K) * sum|terms| of the exact value for random-sign terms (u = 2^-24);
the tests allow 16 u sqrt(K) * sum|terms| per element, with K the number of
terms of that element.
"""
import numpy as np
import pytest
import torch

import oracle
from rank_markov_draft_vanillamarkov_b200 import VanillaMarkov, device_status, last_algo, last_variant, set_algo
from rank_markov_draft_vanillamarkov_b200 import _native as N
from rank_markov_draft_vanillamarkov_b200 import workloads as W
from rank_markov_draft_vanillamarkov_b200.build import build

from _helpers import f64

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


TC, GEN = N.DSPARK_ALGO_TENSOR_CORE, N.DSPARK_ALGO_GENERIC


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    N.load()
    yield
    set_algo(N.DSPARK_ALGO_AUTO)


def _inputs(rows, vocab, rank, seed, ldt=torch.bfloat16, wdt=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    w1 = (torch.randn(vocab, rank, generator=g) * 0.3).to(wdt)
    w2 = (torch.randn(vocab, rank, generator=g) * 0.3).to(wdt)
    dout = torch.randn(rows, vocab, generator=g).to(ldt)
    ids = W.zipf_ids(g, rows, vocab)
    return w1, w2, dout, ids


def _check(w1, w2, dout, ids, gw1, gw2):
    d, a1, a2, i = f64(dout), f64(w1), f64(w2), ids.numpy()
    want1, want2 = oracle.apply_block_logits_backward(d, a1, a2, i)
    # sum of |terms| of every element, and its number of terms
    abs2 = np.abs(d).T @ np.abs(a1[i])
    abs1 = np.zeros_like(a1)
    np.add.at(abs1, i, np.abs(d) @ np.abs(a2))
    counts = np.bincount(i, minlength=a1.shape[0])[:, None]
    k1 = np.maximum(counts * d.shape[1], 1)
    tol1 = 16 * U * np.sqrt(k1) * abs1 + 1e-30
    tol2 = 16 * U * np.sqrt(d.shape[0]) * abs2 + 1e-30
    e1 = np.abs(gw1.cpu().double().numpy() - want1)
    e2 = np.abs(gw2.cpu().double().numpy() - want2)
    assert (e1 <= tol1).all(), (e1.max(), np.unravel_index(np.argmax(e1 - tol1), e1.shape))
    assert (e2 <= tol2).all(), (e2.max(), np.unravel_index(np.argmax(e2 - tol2), e2.shape))


def _run(w1, w2, dout, ids, algo, **kw):
    set_algo(algo)
    head = VanillaMarkov(w1.cuda(), w2.cuda())
    gw1, gw2 = head.apply_block_logits_backward(dout.cuda(), token_ids=ids.cuda(), **kw)
    used = last_algo()
    torch.cuda.synchronize()
    return gw1, gw2, used


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
@pytest.mark.parametrize("rows,vocab,rank", [
    (200, 1000, 64),     # ragged 128-id tile and 64-row stage
    (330, 2056, 256),    # four 64-column blocks, 6 row stages
    (150, 2048, 192),    # three column blocks
    (700, 20480, 128),   # 160 id tiles: CTAs take two dW2 units
    (19000, 64, 128),    # 149 row tiles: CTAs take two dW1 units; one dW2 unit over 297 stages
])
def test_backward_small(rows, vocab, rank, algo):
    w1, w2, dout, ids = _inputs(rows, vocab, rank, seed=rows)
    gw1, gw2, used = _run(w1, w2, dout, ids, algo)
    assert used == (2 if algo == TC else 1)
    assert device_status() == 0
    _check(w1, w2, dout, ids, gw1, gw2)


@pytest.mark.parametrize("rows,rank,accumulate,resident", [
    (130, 256, False, True),    # rank 256: four W1 boxes per row beside the resident block, the widest MMA
    (192, 256, True, True),     # the largest row count that keeps rank 256 resident; TMA reduce-add epilogue
    (193, 256, False, False),   # one more stage no longer fits: per-stage gathers
    (330, 128, True, True),
])
def test_backward_resident_w1_choice(rows, rank, accumulate, resident):
    """The tensor-core dW2 keeps every row's W1 row resident exactly when the
    block fits beside three gradient stages; both forms match the oracle."""
    w1, w2, dout, ids = _inputs(rows, 2056, rank, seed=rows + rank)
    kw = {}
    if accumulate:
        kw = dict(grad_w1=torch.full((2056, rank), 0.5, device="cuda"),
                  grad_w2=torch.full((2056, rank), -0.25, device="cuda"), accumulate=True)
    gw1, gw2, used = _run(w1, w2, dout, ids, TC, **kw)
    assert used == 2 and device_status() == 0
    assert bool(last_variant() & N.DSPARK_VARIANT_BWD_RESIDENT_W1) == resident
    if accumulate:
        gw1, gw2 = kw["grad_w1"] - 0.5, kw["grad_w2"] + 0.25
    _check(w1, w2, dout, ids, gw1, gw2)


def test_backward_generic_only_shapes():
    """rank 96 and V = 4099 (not a multiple of 8) take the CUDA-core kernels
    under AUTO; forcing the tensor cores is refused."""
    w1, w2, dout, ids = _inputs(37, 4099, 96, seed=37)
    gw1, gw2, used = _run(w1, w2, dout, ids, N.DSPARK_ALGO_AUTO)
    assert used == 1 and device_status() == 0
    _check(w1, w2, dout, ids, gw1, gw2)
    set_algo(TC)
    head = VanillaMarkov(w1.cuda(), w2.cuda())
    with pytest.raises(RuntimeError):
        head.apply_block_logits_backward(dout.cuda(), token_ids=ids.cuda())


def test_backward_full_size_block_shape():
    """320 rows shaped (4, 16, 5) at V = 129280, rank 128, Zipf(1.1) ids
    (so many rows share an id and their dW1 contributions add up)."""
    d = W.make_inputs(W.APPLY_320)
    g = torch.Generator().manual_seed(1)
    dout = torch.randn(4, 16, 5, 129280, generator=g).to(torch.bfloat16)
    gw1, gw2, used = _run(d["w1"], d["w2"], dout, d["prev_ids"], N.DSPARK_ALGO_AUTO)
    assert used == 2 and device_status() == 0
    _check(d["w1"], d["w2"], dout.view(-1, 129280), d["prev_ids"].view(-1), gw1, gw2)


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_backward_bf16_accumulate(algo):
    """accumulate = True adds onto the given buffers (dW2 by TMA reduce-add on
    the tensor-core path)."""
    w1, w2, dout, ids = _inputs(260, 1032, 128, seed=11)
    b1 = torch.full((1032, 128), 0.5, device="cuda")
    b2 = torch.full((1032, 128), -0.25, device="cuda")
    _, _, used = _run(w1, w2, dout, ids, algo, grad_w1=b1, grad_w2=b2, accumulate=True)
    assert used == (2 if algo == TC else 1) and device_status() == 0
    _check(w1, w2, dout, ids, b1 - 0.5, b2 + 0.25)


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_backward_one_gradient(algo):
    """Only dW2 (want_w1 = False), then only dW1 (want_w2 = False): each
    kernel alone."""
    w1, w2, dout, ids = _inputs(90, 512, 64, seed=4)
    set_algo(algo)
    head = VanillaMarkov(w1.cuda(), w2.cuda())
    only1, g2 = head.apply_block_logits_backward(dout.cuda(), token_ids=ids.cuda(), want_w1=False)
    g1, only2 = head.apply_block_logits_backward(dout.cuda(), token_ids=ids.cuda(), want_w2=False)
    torch.cuda.synchronize()
    assert only1 is None and only2 is None and device_status() == 0
    _check(w1, w2, dout, ids, g1, g2)


def test_backward_fp32_and_accumulate():
    """fp32 operands (CUDA-core kernels), and accumulate = True adds onto
    given buffers."""
    w1, w2, dout, ids = _inputs(50, 1024, 16, seed=3, ldt=torch.float32, wdt=torch.float32)
    set_algo(N.DSPARK_ALGO_AUTO)
    head = VanillaMarkov(w1.cuda(), w2.cuda())
    b1 = torch.full((1024, 16), 0.5, device="cuda")
    b2 = torch.full((1024, 16), -0.25, device="cuda")
    head.apply_block_logits_backward(dout.cuda(), token_ids=ids.cuda(), grad_w1=b1, grad_w2=b2, accumulate=True)
    torch.cuda.synchronize()
    _check(w1, w2, dout, ids, b1 - 0.5, b2 + 0.25)


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_backward_out_of_range_ids(algo):
    """A row with an id outside [0, V) contributes nothing and sets the
    TOKEN_RANGE status."""
    w1, w2, dout, ids = _inputs(64, 1000, 64, seed=5)
    ids[10] = 1000
    ids[20] = -3
    gw1, gw2, used = _run(w1, w2, dout, ids, algo)
    assert used == (2 if algo == TC else 1)
    assert device_status() & N.DSPARK_STATUS_TOKEN_RANGE
    keep = torch.from_numpy(np.setdiff1d(np.arange(64), [10, 20]))
    _check(w1, w2, dout[keep], ids[keep], gw1, gw2)
