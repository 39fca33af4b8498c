"""Comparison rules between a result under test and the oracle.

Test infrastructure only.

Corrected logits, bf16 storage. The value under test is the one rounding
(round-to-nearest-even) of an fp32-accumulated sum, and the fp32 sum lies
within ``acc`` of the exact (fp64) sum, where ``acc`` is the forward error
bound of ``accumulation_bound``. Rounding is monotone, so a correct value
lies in

    [RNE(exact - acc), RNE(exact + acc)]                          (clause 1)

which is the single value RNE(exact) unless the exact sum lies within ``acc``
of a rounding boundary, where the neighbouring bf16 value is also allowed.
It must also satisfy the stated max-abs tolerance, widened by the half-ulp
that rounding itself must be allowed (at |x| >= 8 a bf16 half-ulp already
exceeds 2e-2):

    |got - exact| <= 2e-2 + ulp(exact) / 2                         (clause 2)

fp32 storage: |got - exact| <= 1e-4.

Tokens. Each step is recomputed with the chain's OWN previous token (the
oracle is teacher-forced on the tokens under test), so that a legitimate
flip at a near-tie does not make every later step differ. Every id v gets a
score s_v (the rounded corrected logit c_v for greedy, c_v / T + g_v under
temperature) and a deviation d_v: how far a correct implementation's score
may lie from the oracle's, i.e. the largest move of c_v allowed by clause 1
(divided by T under temperature, plus the error bound of the Gumbel variate
and of the fp32 evaluation of the score). With t1 the oracle's choice, a
token t is accepted when

    t == t1   or   s_t1 - s_t <= max(1e-2, d_t1 + d_t).

So the token must equal the oracle's wherever the top-1/top-2 margin
exceeds 1e-2 and no allowed rounding can close it; near such ties it may be
any id whose score lies within that window of the best. With fp32 logits
every token must equal the oracle's.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .markov import GREEDY_TEMPERATURE, apply_step_logits, compute_step_bias
from .philox import gumbel_noise
from .rounding import round_to, ulp_bfloat16

LOGIT_ABS_TOL_BF16 = 2e-2
LOGIT_ABS_TOL_FP32 = 1e-4
TOKEN_MARGIN = 1e-2
# Bound on the error of a Gumbel variate g = -ln(-ln u) computed in fp32 (the
# CUDA path's is below 5e-6 over all 2^23 possible u, checked on the GPU).
GUMBEL_ABS_ERR = 1e-5
# Relative error bound of evaluating c * (1/T) + g in fp32: the reciprocal,
# the product and the sum each round once (3 * 2^-24), doubled.
SCORE_EVAL_REL = 2.0 ** -21


@dataclass
class LogitReport:
    n: int
    max_abs: float
    max_ulps_vs_rne: float
    bad: int
    first_bad: tuple = field(default=())

    @property
    def ok(self) -> bool:
        return self.bad == 0


def accumulation_bound(base, w1, w2, token_ids) -> np.ndarray:
    """Forward error bound of summing U and the r products W1[x, j] W2[v, j]
    in fp32, in any order: (r + 1) * 2^-23 * (|U| + sum_j |W1[x, j] W2[v, j]|).
    This is twice the classical bound gamma_{r+1} ~ (r + 1) * 2^-24 of a
    recursive sum of r + 1 terms, so that neither the tensor cores' internal
    accumulation order nor a truncating (rather than nearest) adder in them
    can exceed it. The products of two bf16 values are exact in fp32."""
    base = np.abs(np.asarray(base, dtype=np.float64))
    v = base.shape[-1]
    ids = np.asarray(token_ids, dtype=np.int64).reshape(-1)
    a = np.abs(np.asarray(w1, dtype=np.float64)[ids])
    mag = a @ np.abs(np.asarray(w2, dtype=np.float64)).T
    r = a.shape[-1]
    return ((r + 1) * 2.0 ** -23 * (base.reshape(-1, v) + mag)).reshape(base.shape)


def fused_accumulation_bound(hidden, lm_head, w1, w2, token_ids) -> np.ndarray:
    """The same bound for the fused producer's sums, whose d + r products
    are hidden[i, j] lm_head[v, j] and W1[x_i, j] W2[v, j]:
    (d + r + 1) * 2^-23 * (sum_j |h lm| + sum_j |W1 W2|)."""
    h = np.abs(np.asarray(hidden, dtype=np.float64))
    d = h.shape[-1]
    lead = h.shape[:-1]
    mag_u = h.reshape(-1, d) @ np.abs(np.asarray(lm_head, dtype=np.float64)).T
    ids = np.asarray(token_ids, dtype=np.int64).reshape(-1)
    a = np.abs(np.asarray(w1, dtype=np.float64)[ids])
    mag_b = a @ np.abs(np.asarray(w2, dtype=np.float64)).T
    r = a.shape[-1]
    return ((d + r + 1) * 2.0 ** -23 * (mag_u + mag_b)).reshape(lead + (mag_u.shape[-1],))


def bf16_allowed_interval(exact, acc):
    """Clause 1: the bf16 values a correct one-rounding implementation may
    return for exact sums ``exact`` computed with error at most ``acc``."""
    exact = np.asarray(exact, dtype=np.float64)
    acc = np.asarray(acc, dtype=np.float64)
    return round_to("bf16", exact - acc), round_to("bf16", exact + acc)


def bf16_logit_bad(got, exact, acc) -> np.ndarray:
    """Per element: True where ``got`` breaks clause 1 or clause 2."""
    lo, hi = bf16_allowed_interval(exact, acc)
    near_rounding = (got >= lo) & (got <= hi)
    near_exact = np.abs(got - exact) <= LOGIT_ABS_TOL_BF16 + 0.5 * ulp_bfloat16(exact)
    return ~(near_rounding & near_exact)


def fp32_logit_bad(got, exact) -> np.ndarray:
    return ~(np.abs(got - exact) <= LOGIT_ABS_TOL_FP32)


def check_logits(got, exact, dtype: str, acc=None) -> LogitReport:
    """Element-wise check of logits under test against the exact (fp64) sums.
    ``acc`` is the accumulation bound (0 when not given, which then asks for
    exactly the rounded value in bf16)."""
    got = np.asarray(got, dtype=np.float64)
    exact = np.asarray(exact, dtype=np.float64)
    with np.errstate(invalid="ignore"):  # inf - inf where both are infinite
        return _check_logits(got, exact, dtype, acc)


def _check_logits(got, exact, dtype, acc) -> LogitReport:
    diff = np.abs(got - exact)
    if dtype == "bf16":
        slack = np.zeros_like(exact) if acc is None else np.broadcast_to(np.asarray(acc, np.float64), exact.shape)
        bad = bf16_logit_bad(got, exact, slack)
        ulps = np.abs(got - round_to("bf16", exact)) / ulp_bfloat16(exact)
        max_ulps = float(np.nanmax(ulps)) if ulps.size else 0.0
    elif dtype == "fp32":
        bad = fp32_logit_bad(got, exact)
        max_ulps = 0.0
    else:
        raise ValueError(f"unsupported logits dtype {dtype!r}")
    # Equal values (infinities included) and NaN where the exact sum is NaN
    # are correct; NaN anywhere else is not.
    both_nan = np.isnan(got) & np.isnan(exact)
    bad = (bad & ~(got == exact) & ~both_nan) | (np.isnan(got) != np.isnan(exact))
    nbad = int(bad.sum())
    first = tuple(int(i) for i in np.argwhere(bad)[0]) if nbad else ()
    max_abs = float(np.nanmax(diff)) if diff.size and not np.isnan(diff).all() else 0.0
    return LogitReport(int(got.size), max_abs, max_ulps, nbad, first)


@dataclass
class TokenReport:
    steps: int
    exact_required: int
    exact_matched: int
    near_ties: int
    bad: int
    logits: LogitReport

    @property
    def ok(self) -> bool:
        return self.bad == 0 and self.logits.ok


def rounding_deviation(exact, acc, dtype: str) -> np.ndarray:
    """Per id: the largest distance between the oracle's rounded corrected
    logit and any value clause 1 allows (0 unless the exact sum lies within
    the accumulation bound of a bf16 rounding boundary)."""
    c = round_to(dtype, exact)
    if dtype != "bf16":
        return np.zeros_like(c)
    lo, hi = bf16_allowed_interval(exact, acc)
    return np.maximum(hi - c, c - lo)


def acceptable_tokens(scores, dev, exact_only: bool) -> np.ndarray:
    """Boolean mask over ids: the tokens a correct implementation may choose,
    given the oracle's scores and each id's deviation (see the module
    docstring). ``exact_only`` keeps only the oracle's own choice."""
    scores = np.asarray(scores, dtype=np.float64)
    t1 = int(np.argmax(scores))  # first maximum; NaN counts as the largest
    mask = np.zeros(scores.shape, dtype=bool)
    mask[t1] = True
    if exact_only:
        return mask
    window = np.maximum(TOKEN_MARGIN, dev[t1] + dev)
    with np.errstate(invalid="ignore"):
        mask |= (scores[t1] - scores) <= window
    return mask


def teacher_forced_prev(first_prev, tokens, rows, k: int) -> np.ndarray:
    """The previous token of step k in the chain under test: first_prev at
    k = 0, else the chain's own token at k - 1."""
    return first_prev[rows] if k == 0 else tokens[rows, k - 1]


def check_sampled_block(tokens, corrected, base, w1, w2, first_prev, dtype: str,
                        temperature, seed: int, rows=None) -> TokenReport:
    """Check (tokens [B, M], corrected [B, M, V]) under test against the oracle,
    teacher-forced on the tokens under test. ``rows`` restricts the check to
    some batch rows (for full-size runs)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    corrected = np.asarray(corrected, dtype=np.float64)
    base = np.asarray(base, dtype=np.float64)
    first_prev = np.asarray(first_prev, dtype=np.int64)
    batch, m, _ = base.shape
    rows = np.arange(batch) if rows is None else np.asarray(rows)
    greedy = temperature is None or temperature < GREEDY_TEMPERATURE
    exact_req = exact_ok = ties = bad = 0
    got_all, exact_all, acc_all = [], [], []
    for k in range(m):
        prev = teacher_forced_prev(first_prev, tokens, rows, k)
        exact = base[rows, k, :] + compute_step_bias(w1, w2, prev)
        acc = accumulation_bound(base[rows, k, :], w1, w2, prev)
        got_all.append(corrected[rows, k, :])
        exact_all.append(exact)
        acc_all.append(acc)
        c = round_to(dtype, exact)
        dev = rounding_deviation(exact, acc, dtype)
        for i, b in enumerate(rows):
            if greedy:
                s, d = c[i], dev[i]
            else:
                g = gumbel_noise(seed, int(b), k, c.shape[-1])
                s = c[i] / float(temperature) + g
                d = dev[i] / float(temperature) + GUMBEL_ABS_ERR + \
                    SCORE_EVAL_REL * (np.abs(c[i]) / float(temperature) + np.abs(g))
            ok = acceptable_tokens(s, d, exact_only=(dtype == "fp32"))
            t = int(tokens[b, k])
            inside = 0 <= t < ok.size and bool(ok[t])
            if ok.sum() == 1:
                exact_req += 1
                exact_ok += int(inside)
            else:
                ties += 1
            bad += int(not inside)
    lr = check_logits(np.stack(got_all), np.stack(exact_all), dtype, np.stack(acc_all))
    return TokenReport(m, exact_req, exact_ok, ties, bad, lr)


def check_tokens(tokens, corrected, base, w1, w2, first_prev, dtype, temperature, seed, rows=None):
    return check_sampled_block(tokens, corrected, base, w1, w2, first_prev, dtype, temperature, seed, rows)


def oracle_step(base_k, w1, w2, prev, dtype):
    """One teacher-forced position (B, V), rounded."""
    return apply_step_logits(base_k, w1, w2, prev, dtype)
