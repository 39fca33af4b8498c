"""Plant plausible mistakes in the oracle (on the CPU, via monkeypatch) and
check that the pins in test_oracle_pins.py catch each one."""
import numpy as np
import pytest

import oracle
from oracle import markov as om
from oracle import rounding as orr

import test_oracle_pins as pins


def _fails(fn, *a, **kw):
    with pytest.raises(AssertionError):
        fn(*a, **kw)


def test_transposed_w2_is_caught(monkeypatch):
    monkeypatch.setattr(om, "project_bias", lambda latent, w2: np.asarray(latent, float) @ np.asarray(w2, float))
    _fails(pins.test_bigram_special_case_is_a_table_lookup)


def test_dropped_bias_is_caught(monkeypatch):
    monkeypatch.setattr(om, "compute_step_bias",
                        lambda w1, w2, ids, hidden_states=None: np.zeros((np.size(ids), np.shape(w2)[0])))
    _fails(pins.test_worked_example_apply, "bf16")


def test_double_rounding_is_caught(monkeypatch):
    real = orr.round_to_bfloat16
    monkeypatch.setattr(orr, "round_to_bfloat16", lambda x: real(np.asarray(x, float).astype(np.float32)))
    monkeypatch.setattr(oracle, "round_to_bfloat16", orr.round_to_bfloat16)
    _fails(pins.test_bf16_hand_cases)


def test_truncating_rounding_is_caught(monkeypatch):
    def trunc(x):
        x = np.asarray(x, np.float32)
        return (x.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)
    monkeypatch.setattr(oracle, "round_to_bfloat16", trunc)
    _fails(pins.test_bf16_matches_torch_on_binary32_inputs)


def test_unbiased_chain_feedback_is_caught(monkeypatch):
    """Feeding the argmax of the base logits (not of the corrected logits)
    to the next step."""
    def unbiased_choice(base_logits, w1, w2, first_prev, out_dtype, temperature=0.0, seed=0, hidden_states=None):
        base = np.asarray(base_logits, float)
        prev = np.asarray(first_prev)
        toks, corr = [], []
        for k in range(base.shape[1]):
            corr.append(om.apply_step_logits(base[:, k], w1, w2, prev, out_dtype))
            prev = np.argmax(base[:, k], axis=-1)
            toks.append(prev)
        return np.stack(toks, 1), np.stack(corr, 1)
    monkeypatch.setattr(oracle, "sample_block_tokens", unbiased_choice)
    _fails(pins.test_worked_example_greedy_chain)


def test_off_by_one_prev_is_caught(monkeypatch):
    """Using the first previous token for every step (no feedback)."""
    def no_feedback(base_logits, w1, w2, first_prev, out_dtype, temperature=0.0, seed=0, hidden_states=None):
        base = np.asarray(base_logits, float)
        b, m, _ = base.shape
        prev = np.asarray(first_prev)
        corr = np.stack([om.apply_step_logits(base[:, k], w1, w2, prev, out_dtype) for k in range(m)], 1)
        toks = np.stack([om.sample_tokens(corr[:, k], temperature, seed, k) for k in range(m)], 1)
        return toks, corr
    monkeypatch.setattr(oracle, "sample_block_tokens", no_feedback)
    _fails(pins.test_greedy_chain_brute_force_bigram)


def test_missing_temperature_is_caught(monkeypatch):
    real = om.gumbel_noise
    monkeypatch.setattr(om, "temperature_scores",
                        lambda row, t, seed, b, k: np.asarray(row, float) + real(seed, b, k, np.shape(row)[-1]))
    _fails(pins.test_temperature_sampling_follows_softmax, 0.5)


def test_shared_noise_across_rows_is_caught(monkeypatch):
    """Dropping the row index b from the Philox counter makes every row draw
    the same token."""
    real = om.gumbel_noise
    monkeypatch.setattr(om, "gumbel_noise", lambda seed, b, k, v: real(seed, 0, k, v))
    _fails(pins.test_temperature_sampling_follows_softmax, 1.0)


def test_highest_index_tie_break_is_caught(monkeypatch):
    monkeypatch.setattr(om, "select_greedy",
                        lambda x: (np.shape(x)[-1] - 1 - np.argmax(np.asarray(x)[..., ::-1], axis=-1)))
    _fails(pins.test_worked_example_greedy_chain)


def test_transition_embeddings_from_the_wrong_table_are_caught(monkeypatch):
    """The head's forward returning rows of W2 (the Linear weight) as the
    conditioning embeddings instead of rows of W1."""
    real = om.transition_logits

    def wrong(w1, w2, ids, out_dtype):
        tr, _ = real(w1, w2, ids, out_dtype)
        i = np.asarray(ids, np.int64)
        return tr, np.asarray(w2, float)[i.reshape(-1)][:, :np.shape(w1)[1]].reshape(i.shape + (np.shape(w1)[1],))
    monkeypatch.setattr(oracle, "transition_logits", wrong)
    _fails(pins.test_transition_logits_worked_example_and_bigram)


def test_transition_with_transposed_lookup_is_caught(monkeypatch):
    """The bias read from the bigram table's column (W2[x] . W1^T) instead of
    its row."""
    def wrong(w1, w2, ids, out_dtype):
        i = np.asarray(ids, np.int64)
        flat = i.reshape(-1)
        bias = np.asarray(w2, float)[flat] @ np.asarray(w1, float).T if np.shape(w1)[1] == np.shape(w2)[1] else None
        emb = np.asarray(w1, float)[flat]
        return (oracle.round_to(out_dtype, bias).reshape(i.shape + (np.shape(w2)[0],)),
                emb.reshape(i.shape + (np.shape(w1)[1],)))
    monkeypatch.setattr(oracle, "transition_logits", wrong)
    _fails(pins.test_transition_logits_worked_example_and_bigram)


def test_backward_overwriting_repeated_ids_is_caught(monkeypatch):
    """dW1 written (not added) at ids that occur in several rows."""
    def wrong(grad_out, w1, w2, token_ids):
        vocab = np.shape(w2)[0]
        dout = np.asarray(grad_out, float).reshape(-1, vocab)
        ids = np.asarray(token_ids, np.int64).reshape(-1)
        emb = np.asarray(w1, float)[ids]
        dw1 = np.zeros(np.shape(w1))
        dw1[ids] = dout @ np.asarray(w2, float)
        return dw1, dout.T @ emb
    monkeypatch.setattr(oracle, "apply_block_logits_backward", wrong)
    _fails(pins.test_backward_matches_torch_autograd)


# ---------------------------------------------------------------------------
# The comparison rules (oracle/checks.py): each planted mistake makes a
# checker pin fail.
# ---------------------------------------------------------------------------
from oracle import checks as oc  # noqa: E402


def test_logit_rule_needing_only_one_clause_is_caught(monkeypatch):
    """`or` in place of `and`: a value breaking only one clause passes."""
    def either(got, exact, acc):
        lo, hi = oc.bf16_allowed_interval(exact, acc)
        near_rounding = (got >= lo) & (got <= hi)
        near_exact = np.abs(got - exact) <= oc.LOGIT_ABS_TOL_BF16 + 0.5 * oracle.ulp_bfloat16(exact)
        return ~(near_rounding | near_exact)
    monkeypatch.setattr(oc, "bf16_logit_bad", either)
    _fails(pins.test_check_logits_rejects_two_ulps_off)
    _fails(pins.test_check_logits_rejects_a_value_far_from_the_exact_sum_inside_the_rounding_window)


def test_logit_rule_of_one_ulp_around_the_rounded_sum_is_caught(monkeypatch):
    """The looser rule |got - RNE(exact)| <= 1 ulp lets truncation through."""
    def one_ulp(got, exact, acc):
        rne = oracle.round_to_bfloat16(exact)
        ulp = oracle.ulp_bfloat16(exact)
        return (np.abs(got - rne) > ulp + acc) | (np.abs(got - exact) > oc.LOGIT_ABS_TOL_BF16 + 0.5 * ulp)
    monkeypatch.setattr(oc, "bf16_logit_bad", one_ulp)
    _fails(pins.test_check_logits_rejects_truncation_away_from_a_halfway_point)


def test_loosened_fp32_rule_is_caught(monkeypatch):
    monkeypatch.setattr(oc, "fp32_logit_bad", lambda got, exact: ~(np.abs(got - exact) <= 1e-3))
    _fails(pins.test_check_logits_fp32_bound)


def test_flipped_token_margin_is_caught(monkeypatch):
    """Exact match demanded at near-ties and top-window membership above the
    margin (the comparison turned around)."""
    def flipped(scores, dev, exact_only):
        scores = np.asarray(scores, dtype=np.float64)
        t1 = int(np.argmax(scores))
        mask = np.zeros(scores.shape, dtype=bool)
        mask[t1] = True
        window = np.maximum(oc.TOKEN_MARGIN, dev[t1] + dev)
        mask |= (scores[t1] - scores) > window
        return mask
    monkeypatch.setattr(oc, "acceptable_tokens", flipped)
    _fails(pins.test_near_tie_accepts_the_runner_up_and_rejects_the_third)
    _fails(pins.test_wrong_token_above_the_margin_is_rejected, 0.0)


def test_token_window_without_the_rounding_deviation_is_caught(monkeypatch):
    """A fixed 1e-2 window rejects the legitimate one-ulp flip at |x| >= 8."""
    monkeypatch.setattr(oc, "rounding_deviation", lambda exact, acc, dtype: np.zeros(np.shape(exact)))
    _fails(pins.test_one_ulp_flip_at_large_logits_is_accepted_only_near_a_halfway_point)


@pytest.mark.parametrize("scale", [2.0 ** -20, 2.0 ** 20])
def test_accumulation_bound_off_by_a_power_of_two_is_caught(monkeypatch, scale):
    real = oc.accumulation_bound
    monkeypatch.setattr(oc, "accumulation_bound", lambda *a: real(*a) * scale)
    _fails(pins.test_accumulation_bound_is_attained_within_a_factor_of_three)


def test_accumulation_bound_without_the_base_term_is_caught(monkeypatch):
    """Dropping |U| from the bound: sums where U dominates break it."""
    real = oc.accumulation_bound
    monkeypatch.setattr(oc, "accumulation_bound",
                        lambda base, w1, w2, ids: real(np.zeros_like(np.asarray(base, float)), w1, w2, ids))
    _fails(pins.test_accumulation_bound_is_attained_within_a_factor_of_three)


@pytest.mark.parametrize("wrong", ["first", "same step"])
def test_checker_teacher_forced_on_the_wrong_token_is_caught(monkeypatch, wrong):
    if wrong == "first":
        monkeypatch.setattr(oc, "teacher_forced_prev", lambda first, toks, rows, k: first[rows])
    else:
        monkeypatch.setattr(oc, "teacher_forced_prev",
                            lambda first, toks, rows, k: first[rows] if k == 0 else toks[rows, k])
    _fails(pins.test_chain_is_checked_against_its_own_previous_tokens)


def test_fused_producer_without_the_bias_is_caught(monkeypatch):
    monkeypatch.setattr(om, "fused_lm_head_exact",
                        lambda h, lm, w1, w2, ids: np.asarray(h, float) @ np.asarray(lm, float).T)
    _fails(pins.test_fused_producer_reduces_to_the_pinned_head)


def test_fused_producer_with_a_transposed_lm_head_is_caught(monkeypatch):
    real = om.fused_lm_head_exact
    monkeypatch.setattr(om, "fused_lm_head_exact",
                        lambda h, lm, w1, w2, ids: real(h, np.asarray(lm, float).T, w1, w2, ids))
    _fails(pins.test_fused_producer_explicit_sums)


def test_fused_producer_rounding_u_first_is_caught(monkeypatch):
    """Base logits rounded to fp32 before the bias is added (two roundings)."""
    def twice(h, lm, w1, w2, ids):
        u = oracle.round_to_float32(np.asarray(h, float) @ np.asarray(lm, float).T)
        return u + om.compute_step_bias(w1, w2, np.asarray(ids).reshape(-1))
    monkeypatch.setattr(om, "fused_lm_head_exact", twice)
    _fails(pins.test_fused_producer_rounds_once)
