"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test ties one part of the oracle to something it does not compute
itself: hand-worked values (tests/golden), a library routine that covers a
special case, a closed form, or a distributional law checked by chi-square.
"""
import json
import os

import numpy as np
import pytest
import torch
from scipy import stats
from scipy.special import softmax

import oracle
from oracle import markov as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f(s):
    return float(s) if s in ("inf", "-inf", "nan") else float.fromhex(s)


# --------------------------------------------------------------------------
# bfloat16 rounding
# --------------------------------------------------------------------------

def test_bf16_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "bf16_rounding.json")))["cases"]
    x = np.array([_f(c["x"]) for c in cases])
    want = np.array([_f(c["want"]) for c in cases])
    got = oracle.round_to_bfloat16(x)
    for xi, gi, wi, c in zip(x, got, want, cases):
        if np.isnan(wi):
            assert np.isnan(gi), c["why"]
        else:
            assert gi == wi and np.signbit(gi) == np.signbit(wi), (c["x"], gi.hex(), c["why"])


def test_bf16_matches_torch_on_binary32_inputs():
    """For inputs that are binary32 values there is one rounding either way,
    so the oracle must agree with torch's float32 -> bfloat16 conversion
    (round to nearest even) bit for bit."""
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2 ** 32, size=400_000, dtype=np.uint64).astype(np.uint32)
    x32 = bits.view(np.float32)
    x32 = x32[np.isfinite(x32)]
    extra = np.array([1.0, 1.00390625, 1.01171875, 3.3895314e38, -3.3895314e38, 1e-40, -1e-41, 0.0],
                     dtype=np.float32)
    x32 = np.concatenate([x32, extra, (rng.standard_normal(100_000) * 4).astype(np.float32)])
    want = torch.from_numpy(x32.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_to_bfloat16(x32.astype(np.float64))
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all(), (x32[~same][:5], got[~same][:5], want[~same][:5])


def test_bf16_ulp():
    assert oracle.ulp_bfloat16(np.array([1.0]))[0] == 2 ** -7
    assert oracle.ulp_bfloat16(np.array([9.5]))[0] == 2 ** -4
    assert oracle.ulp_bfloat16(np.array([0.0]))[0] == 2 ** -7  # defined at 1 for zero
    assert oracle.ulp_bfloat16(np.array([1e-40]))[0] == 2 ** -133


# --------------------------------------------------------------------------
# The bias and the add
# --------------------------------------------------------------------------

def _worked():
    return json.load(open(os.path.join(GOLDEN, "worked_example.json")))


def test_worked_example_bias_table():
    d = _worked()
    w1, w2 = np.array(d["w1"], float), np.array(d["w2"], float)
    got = oracle.compute_step_bias(w1, w2, np.arange(3))
    np.testing.assert_array_equal(got, np.array(d["bias_table"]["rows"], float))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_worked_example_apply(dtype):
    d = _worked()
    w1, w2 = np.array(d["w1"], float), np.array(d["w2"], float)
    a = d["apply"]
    got = oracle.apply_block_logits(np.array(a["base"], float), w1, w2, np.array(a["prev_ids"]), dtype)
    np.testing.assert_array_equal(got, np.array(a["want"], float))


def test_worked_example_greedy_chain():
    d = _worked()
    w1, w2 = np.array(d["w1"], float), np.array(d["w2"], float)
    s = d["sample_greedy"]
    toks, corr = oracle.sample_block_tokens(np.array(s["base"], float), w1, w2, np.array(s["first_prev"]),
                                            "bf16", temperature=0.0)
    np.testing.assert_array_equal(toks, np.array(s["want_tokens"]))
    np.testing.assert_array_equal(corr, np.array(s["want_corrected"], float))
    # temperature None and below the 1e-5 threshold are greedy too
    for t in (None, 0.0, 9.9e-6, -1.0):
        t2, _ = oracle.sample_block_tokens(np.array(s["base"], float), w1, w2, np.array(s["first_prev"]),
                                           "bf16", temperature=t)
        np.testing.assert_array_equal(t2, np.array(s["want_tokens"]))


def _bigram_case(v=16, seed=0):
    """W1 = identity (r = V): B(x, v) = W2[v, x], a plain bigram table.
    Integer weights keep every sum exact."""
    rng = np.random.default_rng(seed)
    w1 = np.eye(v)
    w2 = rng.integers(-8, 9, size=(v, v)).astype(float)  # not symmetric
    table = w2.T.copy()  # table[x, v] = logit bias of token v after token x
    return w1, w2, table


def test_bigram_special_case_is_a_table_lookup():
    w1, w2, table = _bigram_case()
    assert not np.array_equal(w2, w2.T)
    ids = np.array([3, 0, 15, 3, 7])
    got = oracle.compute_step_bias(w1, w2, ids)
    for i, x in enumerate(ids):
        np.testing.assert_array_equal(got[i], table[x])


def test_transition_logits_worked_example_and_bigram():
    """The head's forward (bias alone + embeddings): the hand-worked bias
    table rows and W1's rows for the worked example, and, with W1 = identity,
    the bigram table rows and one-hot embeddings, for ids of shape (2, 3)."""
    d = _worked()
    w1, w2 = np.array(d["w1"], float), np.array(d["w2"], float)
    ids = np.array([[2, 0, 1], [1, 1, 0]])
    tr, emb = oracle.transition_logits(w1, w2, ids, "fp32")
    assert tr.shape == (2, 3, w2.shape[0]) and emb.shape == (2, 3, w1.shape[1])
    table = np.array(d["bias_table"]["rows"], float)
    np.testing.assert_array_equal(tr, table[ids])
    np.testing.assert_array_equal(emb, w1[ids])
    bw1, bw2, btable = _bigram_case()
    bids = np.array([[3, 0, 15], [7, 7, 1]])
    tr, emb = oracle.transition_logits(bw1, bw2, bids, "bf16")
    np.testing.assert_array_equal(tr, btable[bids])
    np.testing.assert_array_equal(emb, np.eye(16)[bids])


def test_backward_matches_torch_autograd():
    """The backward against torch.autograd (a library implementation) on the
    fp64 forward U + Embedding(W1)(x) @ W2^T, with repeated ids."""
    rng = np.random.default_rng(7)
    v, r = 37, 6
    w1, w2 = rng.standard_normal((v, r)), rng.standard_normal((v, r))
    ids = np.array([[3, 3, 0, 36], [5, 3, 9, 0]])
    dout = rng.standard_normal((2, 4, v))
    dw1, dw2 = oracle.apply_block_logits_backward(dout, w1, w2, ids)
    t1 = torch.tensor(w1, requires_grad=True)
    t2 = torch.tensor(w2, requires_grad=True)
    base = torch.tensor(rng.standard_normal((2, 4, v)))
    out = base + torch.nn.functional.embedding(torch.tensor(ids), t1) @ t2.T
    out.backward(torch.tensor(dout))
    np.testing.assert_allclose(dw1, t1.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dw2, t2.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_backward_bigram_closed_form():
    """W1 = identity: dW2[v, x] is the sum of dOut[i, v] over rows with
    previous token x, and dW1[x] the sum of dOut[i] @ W2 over those rows;
    exact with integer values."""
    w1, w2, _ = _bigram_case()
    ids = np.array([3, 0, 15, 3, 7, 3])
    dout = np.random.default_rng(2).integers(-4, 5, size=(6, 16)).astype(float)
    dw1, dw2 = oracle.apply_block_logits_backward(dout, w1, w2, ids)
    for x in range(16):
        rows = ids == x
        np.testing.assert_array_equal(dw2[:, x], dout[rows].sum(0))
        np.testing.assert_array_equal(dw1[x], (dout[rows] @ w2).sum(0))


def test_zero_w2_passes_logits_through_bit_for_bit():
    rng = np.random.default_rng(1)
    base = oracle.round_to_bfloat16(rng.standard_normal((3, 4, 5, 64)) * 3)
    w1 = rng.standard_normal((64, 16))
    got = oracle.apply_block_logits(base, w1, np.zeros((64, 16)), rng.integers(0, 64, (3, 4, 5)), "bf16")
    np.testing.assert_array_equal(got, base)
    toks, corr = oracle.sample_block_tokens(base[:, 0], w1, np.zeros((64, 16)), rng.integers(0, 64, 3), "bf16")
    np.testing.assert_array_equal(corr, base[:, 0])
    np.testing.assert_array_equal(toks, np.argmax(base[:, 0], axis=-1))


def test_bias_row_by_row_against_explicit_sums():
    """B(x, v) = sum_j W1[x, j] W2[v, j], summed in exact rational arithmetic
    on small dyadic values (so any fp64 sum is exact)."""
    from fractions import Fraction
    rng = np.random.default_rng(2)
    w1 = rng.integers(-64, 65, size=(12, 5)) / 32.0
    w2 = rng.integers(-64, 65, size=(12, 5)) / 16.0
    ids = rng.integers(0, 12, size=7)
    got = oracle.compute_step_bias(w1, w2, ids)
    for i, x in enumerate(ids):
        for v in range(12):
            s = sum(Fraction(w1[x, j]) * Fraction(w2[v, j]) for j in range(5))
            assert Fraction(got[i, v]) == s


def test_hidden_states_are_ignored():
    rng = np.random.default_rng(3)
    base = rng.standard_normal((2, 3, 4, 32))
    w1, w2 = rng.standard_normal((32, 8)), rng.standard_normal((32, 8))
    ids = rng.integers(0, 32, (2, 3, 4))
    a = oracle.apply_block_logits(base, w1, w2, ids, "bf16")
    b = oracle.apply_block_logits(base, w1, w2, ids, "bf16", hidden_states=rng.standard_normal((2, 3, 4, 7)))
    np.testing.assert_array_equal(a, b)
    t1, c1 = oracle.sample_block_tokens(base[:, 0], w1, w2, ids[:, 0, 0], "bf16", 0.7, seed=5)
    t2, c2 = oracle.sample_block_tokens(base[:, 0], w1, w2, ids[:, 0, 0], "bf16", 0.7, seed=5,
                                        hidden_states=rng.standard_normal((2, 4, 9)))
    np.testing.assert_array_equal(t1, t2)
    np.testing.assert_array_equal(c1, c2)


def test_empty_inputs_return_the_input_object():
    w1 = np.ones((8, 2))
    w2 = np.ones((8, 2))
    e1 = np.zeros((2, 0, 8))
    assert oracle.apply_block_logits(e1, w1, w2, np.zeros((2, 0), int), "bf16") is e1
    e2 = np.zeros((0, 3, 8))
    assert oracle.apply_block_logits(e2, w1, w2, np.zeros((0, 3), int), "bf16") is e2
    toks, corr = oracle.sample_block_tokens(e1, w1, w2, np.array([1, 2]), "bf16")
    assert corr is e1 and toks.shape == (2, 0) and toks.dtype == np.int64


def test_out_of_range_ids_are_rejected():
    with pytest.raises(IndexError):
        oracle.compute_step_bias(np.ones((4, 2)), np.ones((4, 2)), np.array([4]))
    with pytest.raises(IndexError):
        oracle.compute_step_bias(np.ones((4, 2)), np.ones((4, 2)), np.array([-1]))


def test_greedy_ties_take_the_lowest_index_and_nan_wins():
    assert oracle.select_greedy(np.array([[1.0, 3.0, 3.0, 2.0]]))[0] == 1
    assert oracle.select_greedy(np.array([[1.0, np.nan, 3.0, np.nan]]))[0] == 1
    assert oracle.select_greedy(np.array([[-np.inf, -np.inf]]))[0] == 0


# --------------------------------------------------------------------------
# The greedy chain
# --------------------------------------------------------------------------

def test_greedy_chain_brute_force_bigram():
    """V = 16, M = 4, every first token: walk the bigram chain by hand
    (explicit loops over the table, no matrix product) and compare."""
    v, m = 16, 4
    w1, w2, table = _bigram_case(v, seed=4)
    rng = np.random.default_rng(5)
    base = rng.integers(-16, 17, size=(v, m, v)).astype(float) / 4  # one block per first token
    toks, corr = oracle.sample_block_tokens(base, w1, w2, np.arange(v), "bf16", temperature=0.0)
    for x0 in range(v):
        prev = x0
        for k in range(m):
            row = [base[x0, k, j] + table[prev][j] for j in range(v)]
            best = max(range(v), key=lambda j: (row[j], -j))
            assert toks[x0, k] == best
            assert list(corr[x0, k]) == row
            prev = best


def test_tokens_are_argmax_of_returned_logits():
    rng = np.random.default_rng(6)
    base = oracle.round_to_bfloat16(rng.standard_normal((4, 5, 300)) * 2)
    w1, w2 = rng.standard_normal((300, 16)) * 0.3, rng.standard_normal((300, 16)) * 0.3
    toks, corr = oracle.sample_block_tokens(base, w1, w2, rng.integers(0, 300, 4), "bf16")
    np.testing.assert_array_equal(toks, np.argmax(corr, axis=-1))


def test_sample_equals_apply_on_its_own_tokens():
    """The two modes differ only in where x_{k-1} comes from: the corrected
    logits of a sampled block equal the teacher-forced ones computed with
    prev = [first_prev, tok_0, ..., tok_{M-2}]."""
    rng = np.random.default_rng(7)
    base = oracle.round_to_bfloat16(rng.standard_normal((6, 5, 200)) * 2)
    w1, w2 = rng.standard_normal((200, 32)) * 0.3, rng.standard_normal((200, 32)) * 0.3
    first = rng.integers(0, 200, 6)
    for temp in (0.0, 0.8):
        toks, corr = oracle.sample_block_tokens(base, w1, w2, first, "bf16", temp, seed=9)
        prev = np.concatenate([first[:, None], toks[:, :-1]], axis=1)
        np.testing.assert_array_equal(oracle.apply_block_logits(base, w1, w2, prev, "bf16"), corr)


# --------------------------------------------------------------------------
# Philox4x32-10 and the temperature sampler
# --------------------------------------------------------------------------

_TRITON_PHILOX = r"""
import os, sys, json
os.environ["TRITON_INTERPRET"] = "1"
import torch, triton, triton.language as tl
@triton.jit
def k(out, c0p, c1p, c2p, c3p, k0p, k1p, N: tl.constexpr):
    i = tl.arange(0, N)
    a, b, c, d = tl.philox_impl(tl.load(c0p + i), tl.load(c1p + i), tl.load(c2p + i), tl.load(c3p + i),
                                tl.load(k0p + i), tl.load(k1p + i), 10)
    tl.store(out + i, a); tl.store(out + N + i, b); tl.store(out + 2 * N + i, c); tl.store(out + 3 * N + i, d)
cols = json.loads(sys.stdin.read())
n = len(cols[0])
t = [torch.tensor(c, dtype=torch.int64).to(torch.uint32) for c in cols]
out = torch.zeros(4 * n, dtype=torch.uint32)
k[(1,)](out, *t, n)
print(json.dumps(out.to(torch.int64).view(4, n).tolist()))
"""


def test_philox_matches_an_independent_library_implementation():
    """Triton's own Philox4x32 (its CPU interpreter, a library routine the
    oracle does not share) must give the same words for the same counters and
    keys, including all-zero and all-ones corners."""
    import subprocess
    import sys
    rng = np.random.default_rng(8)
    n = 64
    cols = [rng.integers(0, 2 ** 32, n, dtype=np.uint64) for _ in range(6)]
    for c in cols:
        c[0], c[1] = 0, 2 ** 32 - 1
    cols = [c.astype(np.int64).tolist() for c in cols]
    env = dict(os.environ, TRITON_INTERPRET="1")
    res = subprocess.run([sys.executable, "-c", _TRITON_PHILOX], input=json.dumps(cols), capture_output=True,
                         text=True, env=env, timeout=600)
    if res.returncode != 0:
        pytest.skip("triton interpreter unavailable: " + res.stderr[-300:])
    want = np.array(json.loads(res.stdout.strip().splitlines()[-1]), dtype=np.uint64)
    c = [np.array(x, dtype=np.uint64).astype(np.uint32) for x in cols]
    for i in range(n):
        got = oracle.philox4x32((c[0][i], c[1][i], c[2][i], c[3][i]), (int(c[4][i]), int(c[5][i])))
        assert [int(w) for w in got] == [int(w) for w in want[:, i]], i


def test_philox_words_look_uniform():
    w = np.concatenate([oracle.noise_words(1234, b, k, 4096) for b in range(4) for k in range(4)])
    counts = np.bincount((w >> np.uint32(24)).astype(np.int64), minlength=256)
    assert stats.chisquare(counts).pvalue > 1e-3
    u = oracle.uniform_from_word(w)
    assert u.min() > 0 and u.max() < 1
    # neighbouring ids (same Philox call and across calls) are uncorrelated
    assert abs(np.corrcoef(u[:-1], u[1:])[0, 1]) < 0.02


def test_uniform_mapping_endpoints():
    u = oracle.uniform_from_word(np.array([0, 0xFFFFFFFF, 0x1FF, 0x200], dtype=np.uint32))
    assert u[0] == 2.0 ** -24 and u[1] == 1 - 2.0 ** -24
    assert u[2] == 2.0 ** -24 and u[3] == 3 * 2.0 ** -24


def test_noise_layout_four_ids_per_call():
    seed = (7 << 32) | 99
    w = oracle.noise_words(seed, b=5, k=3, vocab=10)
    for v in range(10):
        words = oracle.philox4x32((np.uint32(v >> 2), np.uint32(3), np.uint32(5), np.uint32(0)), (99, 7))
        assert int(w[v]) == int(words[v & 3])


@pytest.mark.parametrize("temp", [0.5, 0.7, 1.0, 2.0])
def test_temperature_sampling_follows_softmax(temp):
    """V = 8, M = 1: many rows of the same logits, each with its own noise
    (row index b is part of the Philox counter). Counts must fit
    softmax(c / T) (scipy) by chi-square."""
    v, rows = 8, 1 << 14
    rng = np.random.default_rng(10)
    logits = oracle.round_to_bfloat16(rng.standard_normal(v) * 1.5)
    w1, w2 = np.zeros((v, 2)), np.zeros((v, 2))
    base = np.broadcast_to(logits, (rows, 1, v))
    toks, _ = oracle.sample_block_tokens(base, w1, w2, np.zeros(rows, int), "bf16", temp, seed=1234)
    counts = np.bincount(toks[:, 0], minlength=v)
    p = softmax(logits / temp)
    assert stats.chisquare(counts, p * rows).pvalue > 1e-3


def test_chain_joint_distribution_bigram():
    """V = 4, M = 3, bigram table (W1 = I): the frequencies of all 64 sampled
    sequences must fit the product of the per-step conditionals
    softmax((U_k + T[x_{k-1}]) / T), written out with scipy's softmax."""
    v, m, rows, temp = 4, 3, 1 << 14, 0.9
    w1 = np.eye(v)
    w2 = np.array([[1.0, -1, 0, 0.5], [0, 2, -1, 0], [-1, 0, 1.5, -0.5], [0.5, 0, -1, 1]])
    table = w2.T
    u = np.array([[0.2, 0.0, -0.3, 0.1], [0.0, 0.5, 0.0, -0.5], [-0.2, 0.1, 0.3, 0.0]])
    base = np.broadcast_to(u, (rows, m, v))
    x0 = 2
    toks, _ = oracle.sample_block_tokens(base, w1, w2, np.full(rows, x0), "fp32", temp, seed=77)
    idx = toks[:, 0] * 16 + toks[:, 1] * 4 + toks[:, 2]
    counts = np.bincount(idx, minlength=64)
    p = np.zeros(64)
    for a in range(v):
        for b in range(v):
            for c in range(v):
                pa = softmax((u[0] + table[x0]) / temp)[a]
                pb = softmax((u[1] + table[a]) / temp)[b]
                pc = softmax((u[2] + table[b]) / temp)[c]
                p[a * 16 + b * 4 + c] = pa * pb * pc
    assert abs(p.sum() - 1) < 1e-12
    keep = p * rows >= 5  # chi-square needs expected counts >= 5
    obs = np.append(counts[keep], counts[~keep].sum())
    exp = np.append(p[keep] * rows, p[~keep].sum() * rows)
    assert stats.chisquare(obs, exp).pvalue > 1e-3


# --------------------------------------------------------------------------
# The comparison rules (oracle/checks.py) that every GPU parity test uses.
# Each rule is pinned from both sides: values a correct implementation may
# return are accepted, and each plausible kind of wrong value is rejected.
# --------------------------------------------------------------------------
from oracle import checks as oc  # noqa: E402


def _bf16(x):
    return oracle.round_to_bfloat16(np.asarray(x, float))


def test_check_logits_accepts_one_rounding_of_any_sum_within_the_bound():
    """A correct kernel returns RNE(e) for some fp32 sum e within acc of the
    exact sum; every such value is accepted, at every magnitude."""
    rng = np.random.default_rng(20)
    exact = rng.standard_normal(40_000) * np.repeat([0.01, 0.3, 3.0, 12.0, 40.0, 0.5], [8000, 8000, 8000, 8000,
                                                                                         4000, 4000])
    acc = np.abs(exact) * 2.0 ** -18 + 1e-9
    for e in (exact + acc * rng.uniform(-1, 1, exact.shape), exact + acc, exact - acc, exact):
        rep = oc.check_logits(_bf16(e), exact, "bf16", acc)
        assert rep.ok, rep


def test_check_logits_rejects_two_ulps_off():
    """Clause 1 alone: near |x| = 0.3 two bf16 ulps are 4e-3, well inside the
    2e-2 max-abs bound, and must still be rejected."""
    exact = np.linspace(0.26, 0.49, 64)
    acc = np.full_like(exact, 1e-7)
    got = _bf16(exact) + 2 * oracle.ulp_bfloat16(exact)
    assert np.all(np.abs(got - exact) < oc.LOGIT_ABS_TOL_BF16)
    assert oc.check_logits(got, exact, "bf16", acc).bad == exact.size


def test_check_logits_rejects_truncation_away_from_a_halfway_point():
    """Truncating instead of rounding is one ulp off where the exact sum is
    clearly above the halfway point (0.8 of the way to the next value)."""
    lo = 1.0 + np.arange(1, 100) * 2.0 ** -7
    exact = lo + 0.8 * 2.0 ** -7
    acc = np.full_like(exact, 1e-6)
    assert np.all(_bf16(exact) == lo + 2.0 ** -7)
    assert oc.check_logits(lo, exact, "bf16", acc).bad == exact.size


def test_check_logits_allows_the_other_neighbour_only_near_a_halfway_point():
    """Within acc of a halfway point both neighbours are one rounding of an
    allowed sum; farther away only the nearer one is."""
    lo = 1.0 + np.arange(1, 100) * 2.0 ** -7
    hi = lo + 2.0 ** -7
    half = lo + 2.0 ** -8
    acc = np.full_like(half, 1e-6)
    near = half + 0.5e-6
    assert oc.check_logits(lo, near, "bf16", acc).ok and oc.check_logits(hi, near, "bf16", acc).ok
    far = half + 3e-6
    assert oc.check_logits(hi, far, "bf16", acc).ok
    assert oc.check_logits(lo, far, "bf16", acc).bad == far.size


def test_check_logits_rejects_a_value_far_from_the_exact_sum_inside_the_rounding_window():
    """Clause 2 alone. Where U and the bias cancel, acc is large and clause 1
    admits a wide window, yet the value must stay within 2e-2 (+ ulp/2) of
    the exact sum; so must a value one ulp from the rounded sum at
    |x| in [4, 8), where that ulp is 1/32."""
    exact = np.array([1e-3, -2e-3, 4e-3])
    acc = np.full(3, 0.06)
    got = _bf16(exact + 0.035)
    lo, hi = oc.bf16_allowed_interval(exact, acc)
    assert np.all((got >= lo) & (got <= hi))
    assert oc.check_logits(got, exact, "bf16", acc).bad == 3
    exact = np.array([5.0 + 0.4 * 2.0 ** -5])
    got = np.array([5.0 - 2.0 ** -5])
    acc = np.array([0.05])
    lo, hi = oc.bf16_allowed_interval(exact, acc)
    assert lo[0] <= got[0] <= hi[0]
    assert abs(got[0] - exact[0]) > 3e-2
    assert oc.check_logits(got, exact, "bf16", acc).bad == 1


def test_check_logits_fp32_bound():
    rng = np.random.default_rng(21)
    exact = rng.standard_normal(1000) * 3
    assert oc.check_logits(exact + 5e-5, exact, "fp32").ok
    assert oc.check_logits(exact + 2e-4, exact, "fp32").bad == exact.size
    assert oc.check_logits(exact - 2e-4, exact, "fp32").bad == exact.size


def test_check_logits_nan_and_infinities():
    exact = np.array([1.0, np.inf, -np.inf, np.nan, 2.0])
    acc = np.zeros(5)
    assert oc.check_logits(exact.copy(), exact, "bf16", acc).ok
    for i, wrong in ((0, np.nan), (1, 3.0), (2, np.inf), (3, 1.0)):
        got = exact.copy()
        got[i] = wrong
        rep = oc.check_logits(got, exact, "bf16", acc)
        assert rep.bad == 1 and rep.first_bad == (i,), (i, rep)


def _strong_block(seed, b=6, m=4, v=300, r=32, std=0.3, dtype="bf16"):
    rng = np.random.default_rng(seed)
    rnd = (lambda x: _bf16(x)) if dtype == "bf16" else oracle.round_to_float32
    base = rnd(rng.standard_normal((b, m, v)) * 2)
    w1, w2 = rnd(rng.standard_normal((v, r)) * std), rnd(rng.standard_normal((v, r)) * std)
    return base, w1, w2, rng.integers(0, v, b)


def test_dropped_bias_is_rejected_at_strong_weights():
    """With weights ~N(0, 0.3) the bias has std ~1.7; returning the base
    logits (bias skipped) fails the logits rule almost everywhere, in both
    the teacher-forced and the sampled form."""
    base, w1, w2, first = _strong_block(23)
    ids = np.random.default_rng(24).integers(0, 300, base.shape[:2])
    exact = oracle.markov.exact_block_logits(base, w1, w2, ids)
    acc = oc.accumulation_bound(base, w1, w2, ids)
    assert oc.check_logits(_bf16(exact), exact, "bf16", acc).ok
    assert oc.check_logits(base, exact, "bf16", acc).bad > 0.9 * base.size
    toks = np.argmax(base, axis=-1)
    rep = oc.check_sampled_block(toks, base, base, w1, w2, first, "bf16", 0.0, 0)
    assert not rep.ok and rep.logits.bad > 0.9 * base.size


@pytest.mark.parametrize("dtype,temp", [("bf16", 0.0), ("bf16", 0.8), ("fp32", 0.0), ("fp32", 1.3)])
def test_oracle_output_passes_the_check(dtype, temp):
    base, w1, w2, first = _strong_block(25, dtype=dtype)
    toks, corr = oracle.sample_block_tokens(base, w1, w2, first, dtype, temp, seed=5)
    rep = oc.check_sampled_block(toks, corr, base, w1, w2, first, dtype, temp, 5)
    assert rep.ok and rep.exact_required > 0, rep


def _top2_gap(s):
    o = np.sort(s)[::-1]
    return o[0] - o[1]


@pytest.mark.parametrize("temp", [0.0, 0.8])
def test_wrong_token_above_the_margin_is_rejected(temp):
    """At the last step (nothing later depends on it) of a row whose
    top-1/top-2 score gap exceeds 5e-2, the runner-up is rejected; the
    logits stay correct, so exactly one token is counted bad."""
    base, w1, w2, first = _strong_block(26)
    toks, corr = oracle.sample_block_tokens(base, w1, w2, first, "bf16", temp, seed=3)
    k = base.shape[1] - 1
    for b in range(base.shape[0]):
        c = corr[b, k]
        s = c if temp == 0.0 else oracle.temperature_scores(c, temp, 3, b, k)
        if _top2_gap(s) > 5e-2:
            break
    else:
        pytest.fail("no row with a clear margin")
    wrong = toks.copy()
    wrong[b, k] = int(np.argsort(s)[::-1][1])
    rep = oc.check_sampled_block(wrong, corr, base, w1, w2, first, "bf16", temp, 3)
    assert rep.logits.ok and rep.bad == 1


def test_near_tie_accepts_the_runner_up_and_rejects_the_third():
    """W2 = 0 makes the corrected logits the base logits. Margin 2^-7 (below
    1e-2): the runner-up is accepted, an id 0.5 below is not. Margin 2^-6
    (above 1e-2): the runner-up is rejected too."""
    v = 64
    w1, w2 = np.zeros((v, 4)), np.zeros((v, 4))
    for gap, runner_ok in ((2.0 ** -7, True), (2.0 ** -6, False)):
        base = np.zeros((1, 1, v))
        base[0, 0, 40] = 1.5
        base[0, 0, 7] = 1.5 - gap
        base[0, 0, 20] = 1.0
        for tok, ok in ((40, True), (7, runner_ok), (20, False)):
            rep = oc.check_sampled_block(np.array([[tok]]), base, base, w1, w2, np.array([0]), "bf16", 0.0, 0)
            assert (rep.bad == 0) == ok, (gap, tok, rep)


def test_one_ulp_flip_at_large_logits_is_accepted_only_near_a_halfway_point():
    """At |x| >= 8 a bf16 ulp (1/16) exceeds 1e-2. Id 0's exact sum lies just
    below the halfway point between 10 and 10 + 1/16, so the oracle rounds it
    to 10 and picks id 1 (10 + 1/16). Within the accumulation bound of that
    point a correct kernel may round id 0 up instead, tie, and pick id 0 (the
    lower index): accepted. Farther from the point it may not: rejected."""
    w1 = np.ones((2, 1))
    base = np.array([[[10.0, 10.0625]]])
    for delta, ok in ((1e-6, True), (1e-5, False)):
        w2 = np.array([[2.0 ** -5 - delta], [0.0]])
        acc = oc.accumulation_bound(base[:, 0], w1, w2, [0])[0, 0]
        assert (delta < acc) == ok
        oracle_c = np.array([[[10.0, 10.0625]]])
        flipped_c = np.array([[[10.0625, 10.0625]]])
        rep = oc.check_sampled_block(np.array([[0]]), oracle_c, base, w1, w2, np.array([0]), "bf16", 0.0, 0)
        assert rep.logits.ok and (rep.bad == 0) == ok, (delta, rep)
        rep = oc.check_sampled_block(np.array([[0]]), flipped_c, base, w1, w2, np.array([0]), "bf16", 0.0, 0)
        assert rep.ok == ok, (delta, rep)


def test_chain_is_checked_against_its_own_previous_tokens():
    """With a strong bias the chain's own tokens decide later steps. The
    oracle's chain passes; a chain that fed back nothing (first_prev at every
    step) or a token two steps old fails."""
    base, w1, w2, first = _strong_block(27, m=5)
    toks, corr = oracle.sample_block_tokens(base, w1, w2, first, "bf16", 0.0)
    assert oc.check_sampled_block(toks, corr, base, w1, w2, first, "bf16", 0.0, 0).ok
    m = base.shape[1]
    for stale in ("none", "two back"):
        prev = first.copy()
        wt, wc = np.zeros_like(toks), np.zeros_like(corr)
        for k in range(m):
            if stale == "none":
                p = first
            else:
                p = first if k < 2 else wt[:, k - 2]
            wc[:, k] = oracle.apply_step_logits(base[:, k], w1, w2, p, "bf16")
            wt[:, k] = np.argmax(wc[:, k], axis=-1)
        assert not np.array_equal(wt, toks), stale  # the test has power
        rep = oc.check_sampled_block(wt, wc, base, w1, w2, first, "bf16", 0.0, 0)
        assert not rep.ok, stale


def _fp32_sum(terms):
    s = np.zeros(terms[0].shape, np.float32)
    for t in terms:
        s = (s + t).astype(np.float32)
    return s


def test_accumulation_bound_covers_fp32_sums_in_several_orders():
    """Recursive fp32 sums of U and the r exact products, in the orders a
    kernel may use (U first or last, forward, reversed, numpy's pairwise sum,
    16-term blocks as a tensor-core K step, a fixed shuffle), with and without
    cancellation, all stay within the bound."""
    rng = np.random.default_rng(28)
    v, r, rows = 256, 128, 8
    w1, w2 = _bf16(rng.standard_normal((v, r)) * 0.3), _bf16(rng.standard_normal((v, r)) * 0.3)
    ids = rng.integers(0, v, rows)
    bias = w1[ids] @ w2.T
    for base in (_bf16(rng.standard_normal((rows, v)) * 2), -_bf16(bias)):
        exact = base + bias
        bound = oc.accumulation_bound(base, w1, w2, ids)
        prods = [(w1[ids, j][:, None].astype(np.float32) * w2[None, :, j].astype(np.float32)) for j in range(r)]
        u32 = base.astype(np.float32)
        perm = rng.permutation(r)
        sums = {
            "u first": _fp32_sum([u32] + prods),
            "u last": _fp32_sum(prods + [u32]),
            "reversed": _fp32_sum([u32] + prods[::-1]),
            "pairwise": (np.sum(np.stack(prods), axis=0, dtype=np.float32) + u32).astype(np.float32),
            "blocks of 16": _fp32_sum([u32] + [np.sum(np.stack(prods[i:i + 16]), axis=0, dtype=np.float32)
                                               for i in range(0, r, 16)]),
            "shuffled": _fp32_sum([prods[j] for j in perm] + [u32]),
        }
        for name, s in sums.items():
            err = np.abs(s.astype(np.float64) - exact)
            assert np.all(err <= bound), (name, float((err / bound).max()))


def test_accumulation_bound_is_attained_within_a_factor_of_three():
    """U = 1 and r products of 2^-24 (W1 = W2 = 2^-12): each fp32 addition of
    2^-24 to 1 is a halfway case that rounds to even, back to 1, so the
    recursive sum loses every product. The error r 2^-24 is reached, and the
    bound, about 2 (r + 1) 2^-24, is no more than three times it."""
    r = 64
    w1 = np.full((1, r), 2.0 ** -12)
    w2 = np.full((1, r), 2.0 ** -12)
    u = np.array([[1.0]])
    s = _fp32_sum([u.astype(np.float32)] + [np.full((1, 1), 2.0 ** -24, np.float32)] * r)
    assert s[0, 0] == 1.0
    err = abs(float(s[0, 0]) - (1.0 + r * 2.0 ** -24))
    bound = float(oc.accumulation_bound(u, w1, w2, [0])[0, 0])
    assert err <= bound <= 3 * err, (err, bound)


# --------------------------------------------------------------------------
# The fused producer: base logits U = hidden @ lm_head^T made in the same
# pass as the bias, rounded once.
# --------------------------------------------------------------------------

def test_fused_producer_explicit_sums():
    """Small integers, every sum written out as Python loops (no matrix
    product): out[i, v] = sum_j h[i, j] lm[v, j] + sum_j W1[x_i, j] W2[v, j].
    A square lm_head (d = V) that is not symmetric catches a transposed
    weight."""
    rng = np.random.default_rng(40)
    for rows, d, v, r in ((4, 6, 6, 3), (3, 5, 4, 2)):
        h = rng.integers(-4, 5, size=(rows, d)).astype(float)
        lm = rng.integers(-4, 5, size=(v, d)).astype(float)
        w1 = rng.integers(-3, 4, size=(v, r)).astype(float)
        w2 = rng.integers(-3, 4, size=(v, r)).astype(float)
        ids = rng.integers(0, v, size=rows)
        want = [[sum(h[i][j] * lm[t][j] for j in range(d)) + sum(w1[ids[i]][j] * w2[t][j] for j in range(r))
                 for t in range(v)] for i in range(rows)]
        got = oracle.fused_lm_head_logits(h, lm, w1, w2, ids, "fp32")
        np.testing.assert_array_equal(got, np.array(want))
        if d == v:
            assert not np.array_equal(lm, lm.T)


def test_fused_producer_reduces_to_the_pinned_head():
    """lm_head = 0 gives the transition bias alone (the head's forward); a
    one-hot hidden row e_j gives base logits lm_head[:, j], so the result is
    apply_block_logits on those base logits."""
    rng = np.random.default_rng(41)
    rows, d, v, r = 7, 12, 50, 8
    h = _bf16(rng.standard_normal((rows, d)))
    lm = _bf16(rng.standard_normal((v, d)) * 0.5)
    w1, w2 = _bf16(rng.standard_normal((v, r)) * 0.3), _bf16(rng.standard_normal((v, r)) * 0.3)
    ids = rng.integers(0, v, rows)
    tr, _ = oracle.transition_logits(w1, w2, ids, "bf16")
    np.testing.assert_array_equal(oracle.fused_lm_head_logits(h, np.zeros_like(lm), w1, w2, ids, "bf16"), tr)
    onehot = np.zeros((rows, d))
    cols = rng.integers(0, d, rows)
    onehot[np.arange(rows), cols] = 1.0
    base = lm[:, cols].T  # row i: lm_head[:, cols[i]]
    want = oracle.apply_block_logits(base[:, None, :], w1, w2, ids[:, None], "bf16")[:, 0]
    np.testing.assert_array_equal(oracle.fused_lm_head_logits(onehot, lm, w1, w2, ids, "bf16"), want)


def test_fused_producer_rounds_once():
    """U = 1 + 2^-30 and a bias of 2^-8: the exact sum lies just above the
    halfway point between 1 and 1 + 2^-7, so one rounding to bf16 goes up.
    Rounding U to fp32 first (to 1) lands exactly on the halfway point,
    which ties to even (down)."""
    h = np.array([[1.0, 2.0 ** -15]])
    lm = np.array([[1.0, 2.0 ** -15]])
    w1, w2 = np.array([[1.0]]), np.array([[2.0 ** -8]])
    got = oracle.fused_lm_head_logits(h, lm, w1, w2, [0], "bf16")
    assert got[0, 0] == 1.0 + 2.0 ** -7


def test_fused_producer_matches_a_library_matmul():
    """W2 = 0: the result is the fp64 matrix product of a library (torch)
    rounded once, for leading dims (2, 3)."""
    rng = np.random.default_rng(42)
    h = _bf16(rng.standard_normal((2, 3, 64)))
    lm = _bf16(rng.standard_normal((100, 64)) * 0.1)
    w1, w2 = _bf16(rng.standard_normal((100, 4))), np.zeros((100, 4))
    ids = rng.integers(0, 100, (2, 3))
    want = torch.from_numpy(h).double() @ torch.from_numpy(lm).double().T
    got = oracle.fused_lm_head_logits(h, lm, w1, w2, ids, "fp32")
    np.testing.assert_array_equal(got, oracle.round_to_float32(want.numpy()))


def test_fused_accumulation_bound_covers_fp32_sums():
    """fp32 recursive sums of the d + r products (forward, reversed, 16-term
    blocks) stay within the fused bound."""
    rng = np.random.default_rng(43)
    rows, d, v, r = 4, 256, 64, 64
    h = _bf16(rng.standard_normal((rows, d)))
    lm = _bf16(rng.standard_normal((v, d)) * 0.05)
    w1, w2 = _bf16(rng.standard_normal((v, r)) * 0.3), _bf16(rng.standard_normal((v, r)) * 0.3)
    ids = rng.integers(0, v, rows)
    exact = oracle.fused_lm_head_exact(h, lm, w1, w2, ids)
    bound = oc.fused_accumulation_bound(h, lm, w1, w2, ids)
    prods = [h[:, j][:, None].astype(np.float32) * lm[None, :, j].astype(np.float32) for j in range(d)]
    prods += [w1[ids, j][:, None].astype(np.float32) * w2[None, :, j].astype(np.float32) for j in range(r)]
    for name, terms in (("forward", prods), ("reversed", prods[::-1]),
                        ("blocks of 16", [np.sum(np.stack(prods[i:i + 16]), axis=0, dtype=np.float32)
                                          for i in range(0, d + r, 16)])):
        err = np.abs(_fp32_sum(terms).astype(np.float64) - exact)
        assert np.all(err <= bound), name
