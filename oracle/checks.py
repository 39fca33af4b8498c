"""Comparison rules between a result under test and the oracle.

Test infrastructure only.

Corrected logits (bf16 storage): the value under test ``got`` must satisfy
both
    |got - RNE(exact)| <= 1 bfloat16 ulp at exact + acc, and
    |got - exact|      <= 2e-2 + ulp/2,
where ``exact`` is the fp64 sum and ``acc`` the forward error bound of an
fp32 accumulation of the r products and U (see ``accumulation_bound``; 0 when
not given). The first bound allows the one-ulp difference that an fp32 sum
can make next to a rounding boundary, widened where U and the bias cancel and
the result is far smaller than its terms; the second is the 2e-2 max-abs
bound widened by the half-ulp that rounding itself must be allowed (at
|x| >= 8 a bfloat16 half-ulp already exceeds 2e-2). fp32 storage:
|got - exact| <= 1e-4.

Tokens: a step is recomputed with the chain's OWN previous token (the oracle
is teacher-forced on the tokens under test), so that a legitimate flip at a
near-tie does not make every later step differ. Where the oracle's top-1 /
top-2 margin exceeds 1e-2 the token must equal the oracle's; otherwise it
must be one of the two. With fp32 logits every token must match.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .markov import GREEDY_TEMPERATURE, apply_step_logits, compute_step_bias, temperature_scores
from .rounding import round_to, ulp_bfloat16

LOGIT_ABS_TOL_BF16 = 2e-2
LOGIT_ABS_TOL_FP32 = 1e-4
TOKEN_MARGIN = 1e-2


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
    in fp32, in any order: (r + 1) * 2^-23 * (|U| + sum_j |W1[x, j] W2[v, j]|)
    (twice the classical gamma_n bound, so that the tensor cores' internal
    accumulation order and width need not be known)."""
    base = np.abs(np.asarray(base, dtype=np.float64))
    v = base.shape[-1]
    ids = np.asarray(token_ids, dtype=np.int64).reshape(-1)
    a = np.abs(np.asarray(w1, dtype=np.float64)[ids])
    mag = a @ np.abs(np.asarray(w2, dtype=np.float64)).T
    r = a.shape[-1]
    return ((r + 1) * 2.0 ** -23 * (base.reshape(-1, v) + mag)).reshape(base.shape)


def check_logits(got, exact, dtype: str, acc=None) -> LogitReport:
    got = np.asarray(got, dtype=np.float64)
    exact = np.asarray(exact, dtype=np.float64)
    diff = np.abs(got - exact)
    if dtype == "bf16":
        ulp = ulp_bfloat16(exact)
        rne = round_to("bf16", exact)
        slack = 0.0 if acc is None else np.asarray(acc, dtype=np.float64)
        ulps = np.abs(got - rne) / ulp
        bad = (np.abs(got - rne) > ulp + slack) | (diff > LOGIT_ABS_TOL_BF16 + 0.5 * ulp)
        max_ulps = float(ulps.max()) if ulps.size else 0.0
    else:
        bad = diff > LOGIT_ABS_TOL_FP32
        max_ulps = 0.0
    bad |= np.isnan(got) != np.isnan(exact)
    nbad = int(bad.sum())
    first = tuple(int(i) for i in np.argwhere(bad)[0]) if nbad else ()
    return LogitReport(int(got.size), float(np.nanmax(diff)) if diff.size else 0.0, max_ulps, nbad, first)


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


def _top2(scores: np.ndarray):
    """(first index of the maximum, index of the runner-up, their margin)."""
    scores = np.asarray(scores, dtype=np.float64)
    t1 = int(np.argmax(scores))
    if scores.size == 1:
        return t1, t1, np.inf
    rest = scores.copy()
    rest[t1] = -np.inf
    t2 = int(np.argmax(rest))
    return t1, t2, float(scores[t1] - scores[t2])


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
        prev = first_prev[rows] if k == 0 else tokens[rows, k - 1]
        exact = base[rows, k, :] + compute_step_bias(w1, w2, prev)
        got_all.append(corrected[rows, k, :])
        exact_all.append(exact)
        acc_all.append(accumulation_bound(base[rows, k, :], w1, w2, prev))
        c = round_to(dtype, exact)
        for i, b in enumerate(rows):
            s = c[i] if greedy else temperature_scores(c[i], temperature, seed, int(b), k)
            t1, t2, margin = _top2(s)
            t = int(tokens[b, k])
            if dtype == "fp32" or margin > TOKEN_MARGIN:
                exact_req += 1
                if t == t1:
                    exact_ok += 1
                else:
                    bad += 1
            else:
                ties += 1
                if t not in (t1, t2):
                    bad += 1
    lr = check_logits(np.stack(got_all), np.stack(exact_all), dtype, np.stack(acc_all))
    return TokenReport(m, exact_req, exact_ok, ties, bad, lr)


def check_tokens(tokens, corrected, base, w1, w2, first_prev, dtype, temperature, seed, rows=None):
    return check_sampled_block(tokens, corrected, base, w1, w2, first_prev, dtype, temperature, seed, rows)


def oracle_step(base_k, w1, w2, prev, dtype):
    """One teacher-forced position (B, V), rounded."""
    return apply_step_logits(base_k, w1, w2, prev, dtype)
