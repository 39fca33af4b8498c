"""Parity of the CUDA left-to-right sampler against the fp64 oracle (B200).

Tokens are checked with the oracle teacher-forced on the sampled tokens
(``oracle.checks.check_sampled_block``): exact where the oracle's top-1/top-2
margin exceeds 1e-2 and no allowed rounding closes it, otherwise any id within
that window of the best; exact everywhere for fp32.
"""
import numpy as np
import pytest
import torch
from scipy import stats
from scipy.special import softmax

import oracle
from oracle.checks import check_logits, check_sampled_block
from rank_markov_draft_vanillamarkov_b200 import (VanillaMarkov, device_status, last_algo, last_variant, set_algo,
                                                 set_debug)
from rank_markov_draft_vanillamarkov_b200 import _native as N
from rank_markov_draft_vanillamarkov_b200 import workloads as W
from rank_markov_draft_vanillamarkov_b200.build import build

from _helpers import f64

pytestmark = pytest.mark.gpu

TC, GEN, AUTO = N.DSPARK_ALGO_TENSOR_CORE, N.DSPARK_ALGO_GENERIC, N.DSPARK_ALGO_AUTO


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    N.load()
    yield
    set_algo(AUTO)
    set_debug(0, 0)


_VARIANT = {}


def _sample(d, algo, temperature, seed=0, base=None, first=None):
    set_algo(algo)
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    base = (d["base"] if base is None else base).cuda()
    first = (d["first_prev"] if first is None else first).cuda()
    toks, corr = head.sample_block_tokens(base, first_prev_token_ids=first, temperature=temperature, seed=seed)
    _VARIANT["last"] = last_variant()
    torch.cuda.synchronize()
    return toks, corr, last_algo(), device_status()


@pytest.fixture(params=["tile", "rows"])
def layout(request):
    """The tensor-core sampler forced into its tile layout or its row layout
    (each only where it fits)."""
    set_debug(N.DSPARK_DEBUG_SAMPLE_ROWS if request.param == "rows" else N.DSPARK_DEBUG_SAMPLE_TILE, 0)
    yield request.param
    set_debug(0, 0)


@pytest.mark.parametrize("batch,vocab,rank,m,temperature", [
    (1, 1000, 64, 1, 0.0),     # one step: the chain's first and last step at once
    (64, 2056, 128, 2, 0.8),   # the largest batch (64 padded rows), the last range ends inside a span
    (17, 4104, 256, 3, 0.0),   # rank 256, V not a multiple of 64
    (40, 136, 64, 4, 1.1),     # three CTAs, the last with 8 ids
    (32, 9600, 192, 5, 0.6),   # rank 192 with chunks of several widths
])
def test_row_layout_edge_shapes(batch, vocab, rank, m, temperature):
    """The row-layout sampler at the edges of its plan (steps, batch, rank,
    ranges that end inside a 64-id span, tiny grids), forced, every (b, k)
    against the oracle with weights that move tokens."""
    wl = _small(batch, vocab, rank, m=m, wstd=0.3, seed=50 + batch).with_(temperature=temperature)
    d = W.make_inputs(wl)
    set_debug(N.DSPARK_DEBUG_SAMPLE_ROWS, 0)
    try:
        toks, corr, used, st = _sample(d, TC, temperature, seed=9)
    finally:
        set_debug(0, 0)
    assert used == 2 and st == 0 and _rows_kernel_ran()
    _check(d, toks, corr, temperature, 9)


@pytest.mark.parametrize("temperature", [0.0, 0.7])
def test_default_layout_by_mode(temperature):
    """Unforced, temperature sampling takes the row layout and greedy decoding
    the tile layout (the measured faster of the two on the full-vocabulary
    shapes); batch 70, above the row layout's 64, takes the tile layout
    either way. Both against the oracle."""
    set_debug(0, 0)
    for batch, want_rows in [(8, temperature > 0), (70, False)]:
        wl = _small(batch, 2056, 128, m=3, wstd=0.3)
        d = W.make_inputs(wl)
        toks, corr, used, st = _sample(d, AUTO, temperature, seed=3)
        assert used == 2 and st == 0 and _rows_kernel_ran() == want_rows
        _check(d, toks, corr, temperature, 3)


def _rows_kernel_ran() -> bool:
    """The tensor-core sampler ran in its row layout (batch on the MMA's M
    side), not the tile layout (vocabulary ids on M)."""
    return bool(_VARIANT["last"] & N.DSPARK_VARIANT_SAMPLE_ROWS)


def _check(d, toks, corr, temperature, seed, dtype="bf16", rows=None):
    rep = check_sampled_block(toks.cpu().numpy(), f64(corr), f64(d["base"]), f64(d["w1"]), f64(d["w2"]),
                              d["first_prev"].numpy(), dtype, temperature, seed, rows=rows)
    assert rep.logits.ok, (rep.logits.bad, rep.logits.first_bad, rep.logits.max_abs)
    assert rep.bad == 0, (rep.bad, rep.exact_required, rep.near_ties)
    return rep


def _small(batch, vocab=1000, rank=64, m=5, wstd=0.3, seed=21, spike=6.0):
    return W.GREEDY.with_(name=f"greedy_small_b{batch}_v{vocab}_k{rank}", batch=batch, vocab=vocab, rank=rank,
                          proposal_len=m, weight_std=wstd, spike=spike, data_seed=seed)


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
@pytest.mark.parametrize("batch,vocab,rank", [(1, 1000, 64), (5, 2056, 128), (33, 1000, 192), (70, 4096, 256),
                                              (128, 2056, 64), (150, 4096, 128), (256, 1000, 64)])
def test_greedy_small(batch, vocab, rank, algo, layout):
    """The row layout takes batches up to 64 (32 or 64 padded rows); 70,
    128, 150 and 256 always take the tile layout."""
    wl = _small(batch, vocab, rank)
    d = W.make_inputs(wl)
    toks, corr, used, st = _sample(d, algo, 0.0)
    assert used == (2 if algo == TC else 1) and st == 0
    if algo == TC:
        assert _rows_kernel_ran() == (layout == "rows" and batch <= 64)
    # invariant: each token is the first argmax of its own corrected row
    assert torch.equal(toks, corr.float().argmax(-1))
    _check(d, toks, corr, 0.0, 0)


@pytest.mark.parametrize("batch", W.GREEDY_BATCHES)
def test_greedy_full_size(batch, layout):
    """M = 5, V = 129280, rank 128, peaked logits, every (b, k)."""
    wl = W.greedy(batch)
    d = W.make_inputs(wl)
    toks, corr, used, st = _sample(d, AUTO, 0.0)
    assert used == 2 and st == 0 and _rows_kernel_ran() == (layout == "rows")
    assert torch.equal(toks, corr.float().argmax(-1))
    _check(d, toks, corr, 0.0, 0)


@pytest.mark.parametrize("temperature", [0.0, 0.8])
@pytest.mark.parametrize("rank", [192, 256])
def test_row_kernel_streams_w2_at_large_ranks(rank, temperature):
    """Full vocabulary at ranks 192 and 256: a CTA's W2 chunks do not all fit
    in shared memory, so most stream from L2 through the two-slot ring every
    step. Weights that move tokens; every (b, k) against the oracle."""
    wl = W.greedy(24).with_(rank=rank, weight_std=0.3, spike=0.0, proposal_len=3, data_seed=30 + rank)
    d = W.make_inputs(wl)
    set_debug(N.DSPARK_DEBUG_SAMPLE_ROWS, 0)
    try:
        toks, corr, used, st = _sample(d, AUTO, temperature, seed=11)
    finally:
        set_debug(0, 0)
    assert used == 2 and st == 0 and _rows_kernel_ran()
    _check(d, toks, corr, temperature, 11)


def test_tile_kernel_full_vocabulary():
    """Batch 140 (above the row layout's 64) at full vocabulary and rank 64:
    the tile-layout kernel, every (b, k) against the oracle."""
    wl = W.greedy(140).with_(rank=64, weight_std=0.3, spike=0.0, proposal_len=2, data_seed=41)
    d = W.make_inputs(wl)
    toks, corr, used, st = _sample(d, AUTO, 0.0)
    assert used == 2 and st == 0 and not _rows_kernel_ran()
    _check(d, toks, corr, 0.0, 0)


def test_greedy_strong_bias_changes_tokens():
    """Weights ~N(0, 0.3) make the bias decide tokens; the chain must follow
    its own choices (a teacher-forced or bias-free chain would differ)."""
    wl = W.greedy(32).with_(weight_std=0.3, spike=0.0, data_seed=3)
    d = W.make_inputs(wl)
    toks, corr, used, st = _sample(d, AUTO, 0.0)
    assert used == 2 and st == 0
    _check(d, toks, corr, 0.0, 0)
    unbiased = d["base"].float().argmax(-1)
    assert (toks.cpu() != unbiased).float().mean() > 0.2


def test_temperature_full_size(layout):
    """B = 32, M = 8, V = 151936, rank 64, T = 0.7, Philox seed 1234."""
    wl = W.TEMPERATURE
    d = W.make_inputs(wl)
    toks, corr, used, st = _sample(d, AUTO, wl.temperature, seed=wl.philox_seed)
    assert used == 2 and st == 0 and _rows_kernel_ran() == (layout == "rows")
    rep = _check(d, toks, corr, wl.temperature, wl.philox_seed)
    assert rep.exact_required > 0.9 * wl.batch * wl.proposal_len


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_temperature_small(algo):
    wl = _small(40, 2056, 128, m=6, wstd=0.3).with_(temperature=1.3)
    d = W.make_inputs(wl)
    toks, corr, used, st = _sample(d, algo, 1.3, seed=99)
    assert st == 0
    _check(d, toks, corr, 1.3, 99)


def test_tiny_fp32_greedy_exact():
    wl = W.TINY_FP32
    g = torch.Generator().manual_seed(0)
    w1, w2 = W.make_weights(wl, g)
    base = (torch.randn(2, 5, wl.vocab, generator=g) * wl.logit_std).float()
    d = {"w1": w1, "w2": w2, "base": base, "first_prev": W.uniform_ids(g, 2, wl.vocab)}
    toks, corr, used, st = _sample(d, AUTO, 0.0)
    assert used == 1 and st == 0
    _check(d, toks, corr, 0.0, 0, dtype="fp32")
    t_or, _ = oracle.sample_block_tokens(f64(base), f64(w1), f64(w2), d["first_prev"].numpy(), "fp32", 0.0)
    np.testing.assert_array_equal(toks.cpu().numpy(), t_or)


@pytest.mark.parametrize("temperature", [0.0, 0.9])
def test_sample_matches_apply_on_its_own_tokens(temperature):
    """The sampler's corrected logits equal the teacher-forced apply computed
    with prev = [first_prev, tok_0, ..., tok_{M-2}] (both tensor-core paths)."""
    wl = W.greedy(16).with_(weight_std=0.3, data_seed=8)
    d = W.make_inputs(wl)
    toks, corr, used, _ = _sample(d, TC, temperature, seed=5)
    prev = torch.cat([d["first_prev"].cuda()[:, None], toks[:, :-1]], dim=1)
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    ref = head.apply_block_logits(d["base"].cuda(), token_ids=prev)
    diff = np.abs(f64(ref) - f64(corr)).reshape(-1, wl.vocab)
    ulp = oracle.ulp_bfloat16(f64(ref)).reshape(diff.shape)
    acc = oracle.accumulation_bound(f64(d["base"]).reshape(-1, wl.vocab), f64(d["w1"]), f64(d["w2"]),
                                    prev.cpu().numpy().reshape(-1))
    assert (diff <= ulp + 2 * acc).all()


def test_gpu_sampling_follows_softmax():
    """V = 64, M = 1, 128 identical rows per call, 128 seeds: counts must fit
    softmax(c / T) by chi-square."""
    v, rows, temp = 64, 128, 0.8
    rng = np.random.default_rng(4)
    logits = torch.from_numpy(rng.standard_normal(v) * 1.2).to(torch.bfloat16)
    base = logits.view(1, 1, v).expand(rows, 1, v).contiguous()
    d = {"w1": torch.zeros(v, 64, dtype=torch.bfloat16), "w2": torch.zeros(v, 64, dtype=torch.bfloat16),
         "base": base, "first_prev": torch.zeros(rows, dtype=torch.long)}
    counts = np.zeros(v)
    for seed in range(128):
        toks, _, used, st = _sample(d, TC, temp, seed=seed)
        assert used == 2 and st == 0
        counts += np.bincount(toks.cpu().numpy()[:, 0], minlength=v)
    p = softmax(f64(logits) / temp)
    keep = p * counts.sum() >= 5
    obs = np.append(counts[keep], counts[~keep].sum())
    exp = np.append(p[keep], p[~keep].sum()) * counts.sum()
    assert stats.chisquare(obs, exp).pvalue > 1e-3


def test_philox_draws_match_the_oracle_bit_for_bit():
    """Zero weights and all-equal logits: the token is the argmax of the
    Gumbel noise alone, so the GPU's Philox must reproduce the oracle's draw."""
    v, rows = 512, 64
    base = torch.zeros(rows, 3, v, dtype=torch.bfloat16)
    d = {"w1": torch.zeros(v, 64, dtype=torch.bfloat16), "w2": torch.zeros(v, 64, dtype=torch.bfloat16),
         "base": base, "first_prev": torch.zeros(rows, dtype=torch.long)}
    seed = (3 << 32) | 12345
    toks, _, _, st = _sample(d, TC, 1.0, seed=seed)
    want = np.array([[int(np.argmax(oracle.gumbel_noise(seed, b, k, v))) for k in range(3)] for b in range(rows)])
    np.testing.assert_array_equal(toks.cpu().numpy(), want)
    toks_g, _, _, _ = _sample(d, GEN, 1.0, seed=seed)
    np.testing.assert_array_equal(toks_g.cpu().numpy(), want)


def test_same_seed_same_draws_other_seed_differs():
    wl = _small(16, 2056, 64, wstd=0.05, spike=0.0)
    d = W.make_inputs(wl)
    a, ca, _, _ = _sample(d, TC, 1.0, seed=7)
    b, cb, _, _ = _sample(d, TC, 1.0, seed=7)
    c, _, _, _ = _sample(d, TC, 1.0, seed=8)
    assert torch.equal(a, b) and torch.equal(ca, cb)
    assert not torch.equal(a, c)


def test_zero_length_block():
    d = W.make_inputs(_small(4))
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    e = torch.zeros(4, 0, 1000, dtype=torch.bfloat16, device="cuda")
    toks, corr = head.sample_block_tokens(e, first_prev_token_ids=torch.zeros(4, dtype=torch.long, device="cuda"))
    assert corr is e and toks.shape == (4, 0) and toks.dtype == torch.long


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_out_of_range_first_prev_reports_status(algo):
    d = W.make_inputs(_small(8))
    first = d["first_prev"].clone()
    first[2] = 10 ** 9
    _, _, _, st = _sample(d, algo, 0.0, first=first)
    assert st & N.DSPARK_STATUS_TOKEN_RANGE


@pytest.mark.parametrize("which", ["tile", "rows"])
def test_barrier_timeout_is_reported_not_hung(which):
    """One CTA withholds its grid-barrier arrival (a host-set test flag):
    the other CTAs' bounded waits run out after 20 ms, the TIMEOUT bit is
    set, the kernel returns, and the next call is correct again. Both
    sampler layouts."""
    wl = W.greedy(8)
    d = W.make_inputs(wl)
    force = N.DSPARK_DEBUG_SAMPLE_ROWS if which == "rows" else N.DSPARK_DEBUG_SAMPLE_TILE
    set_debug(N.DSPARK_DEBUG_SKIP_BARRIER_ARRIVAL | force, 20_000_000)
    try:
        _, _, used, st = _sample(d, TC, 0.0)
        assert _rows_kernel_ran() == (which == "rows")
    finally:
        set_debug(0, 0)
    assert used == 2
    assert st & N.DSPARK_STATUS_TIMEOUT
    set_debug(force, 0)
    try:
        toks, corr, used, st = _sample(d, TC, 0.0)
    finally:
        set_debug(0, 0)
    assert st == 0
    _check(d, toks, corr, 0.0, 0)


def _edge_rows(vocab: int, m: int):
    """Base logits (B, M, V) of selection edge cases, with the first NaN, the
    lowest tied id, etc. spread over lanes, warps, tiles and CTAs."""
    rows = []
    # ties at the maximum: far apart (other CTAs) and adjacent (one warp)
    r = torch.full((vocab,), -1.0)
    for v in (vocab - 1, 70001 % vocab, 41, 40, 3 + 128 * 5):
        r[v] = 5.0
    rows.append(r)
    # NaN counts as the largest value whatever its sign bit; the first NaN
    # wins, above +inf (the lowest one here has its sign bit set)
    r = torch.zeros(vocab)
    r[7] = float("inf")
    for v in (100003 % vocab, vocab - 1):
        r[v] = float("nan")
    r[500 % vocab] = -torch.tensor(float("nan"))
    rows.append(r)
    # -0 and +0 are equal: the lower id wins whichever sign it has
    r = torch.full((vocab,), -1.0)
    r[1234 % vocab] = -0.0
    r[1000 % vocab] = 0.0
    rows.append(r)
    r = torch.full((vocab,), -1.0)
    r[2000 % vocab] = 0.0
    r[1500 % vocab] = -0.0
    rows.append(r)
    # every value -inf: all equal, id 0 wins
    rows.append(torch.full((vocab,), float("-inf")))
    # the maximum in the ragged last tile
    r = torch.full((vocab,), -3.0)
    r[vocab - 1] = 2.0
    rows.append(r)
    # a unique maximum in a middle CTA, negative values elsewhere
    r = -torch.rand(vocab, generator=torch.Generator().manual_seed(5)) - 0.5
    r[vocab // 2 + 17] = -0.25
    rows.append(r)
    base = torch.stack(rows).unsqueeze(1).repeat(1, m, 1)
    return base.to(torch.bfloat16)


@pytest.mark.parametrize("algo", [TC + 100, TC, GEN], ids=["tc_rows", "tc_tile", "generic"])
@pytest.mark.parametrize("vocab", [129280, 1000])
def test_greedy_ties_nan_signed_zero_and_inf(algo, vocab):
    """Greedy selection on exact ties, NaN, -0/+0 and all -inf: with W2 = 0
    every corrected logit is its base logit, so each token is numpy's argmax
    (first NaN, else the lowest id among equal maxima) of its base row. The
    tensor-core sampler in both layouts."""
    rows_layout = algo == TC + 100
    algo = TC if rows_layout else algo
    set_debug(N.DSPARK_DEBUG_SAMPLE_ROWS if rows_layout else 0, 0)
    m, rank = 3, 64
    base = _edge_rows(vocab, m)
    g = torch.Generator().manual_seed(2)
    w1 = (torch.randn(vocab, rank, generator=g) * 0.1).to(torch.bfloat16)
    w2 = torch.zeros(vocab, rank, dtype=torch.bfloat16)
    first = torch.arange(base.shape[0], dtype=torch.long) * 13
    d = {"w1": w1, "w2": w2, "base": base, "first_prev": first}
    try:
        toks, corr, used, st = _sample(d, algo, 0.0)
    finally:
        set_debug(0, 0)
    assert used == (2 if algo == TC else 1) and st == 0
    if algo == TC:
        assert _rows_kernel_ran() == rows_layout
    want = oracle.select_greedy(f64(base))
    np.testing.assert_array_equal(toks.cpu().numpy(), want)
    # the corrected logits are the base logits (-0 + 0 = +0, NaN stays NaN)
    c, b = f64(corr), f64(base)
    assert np.array_equal(np.isnan(c), np.isnan(b))
    ok = ~np.isnan(b)
    assert np.array_equal(c[ok], b[ok] + 0.0)


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_temperature_nan_is_selected_first(algo):
    """With temperature, a NaN logit gives a NaN score, which counts as the
    largest: the first NaN id of each row is drawn whatever the noise."""
    vocab, m, rank = 129280, 2, 64
    g = torch.Generator().manual_seed(4)
    base = (torch.randn(3, m, vocab, generator=g) * 2.0)
    for b, ids in enumerate([(90000, 65), (5,), (129279, 64000)]):
        for v in ids:
            base[b, :, v] = float("nan")
    base[0, :, 65] = -torch.tensor(float("nan"))  # sign bit set: still the largest
    base = base.to(torch.bfloat16)
    assert (base[0, 0, 65].view(torch.int16) < 0).item()
    w1 = (torch.randn(vocab, rank, generator=g) * 0.1).to(torch.bfloat16)
    w2 = torch.zeros(vocab, rank, dtype=torch.bfloat16)
    d = {"w1": w1, "w2": w2, "base": base, "first_prev": torch.tensor([1, 2, 3])}
    toks, corr, used, st = _sample(d, algo, 0.8, seed=7)
    assert used == (2 if algo == TC else 1) and st == 0
    np.testing.assert_array_equal(toks.cpu().numpy(), [[65, 65], [5, 5], [64000, 64000]])


def test_gumbel_noise_every_word_within_bound():
    """Every possible uniform (all 2^23 values of w >> 9) through the device's
    Gumbel function, against g = -log(-log u) in fp64: the absolute error
    stays below 1e-5, and the low 9 bits of the word are ignored."""
    import ctypes
    lib = N.load()
    m = torch.arange(1 << 23, dtype=torch.int64)
    low = torch.randint(0, 512, (1 << 23,), generator=torch.Generator().manual_seed(3))
    words = ((m << 9) | low).to(torch.int64)
    words32 = (words - ((words >> 31) << 32)).to(torch.int32).cuda()  # same bits as uint32
    out = torch.empty(1 << 23, dtype=torch.float32, device="cuda")
    code = lib.dspark_markov_debug_gumbel(words32.data_ptr(), out.data_ptr(), 1 << 23,
                                          torch.cuda.current_stream().cuda_stream)
    assert code == 0
    torch.cuda.synchronize()
    u = (2.0 * m.double().numpy() + 1.0) * 2.0 ** -24
    exact = -np.log(-np.log(u))
    err = np.abs(out.cpu().double().numpy() - exact)
    assert err.max() < 1e-5, (err.max(), int(err.argmax()))
    # u closest to 1 (the largest draws) and closest to 0
    assert abs(out[-1].item() - exact[-1]) < 1e-5 and abs(out[0].item() - exact[0]) < 1e-5


@pytest.mark.parametrize("temperature", [0.0, 0.9])
@pytest.mark.parametrize("batch", [1, 3, 4])
def test_small_batches_full_vocabulary(batch, temperature, layout):
    """Batches of one to four on the tensor-core sampler at full vocabulary,
    rank 128 (so a CTA keeps W2 tiles in both shared and tensor memory),
    with weights that move tokens: every (b, k) against the oracle."""
    wl = W.greedy(batch).with_(weight_std=0.3, spike=0.0, data_seed=20 + batch)
    d = W.make_inputs(wl)
    toks, corr, used, st = _sample(d, TC, temperature, seed=5)
    assert used == 2 and st == 0
    _check(d, toks, corr, temperature, 5)
