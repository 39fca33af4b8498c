"""The VanillaMarkov head, written out plainly in fp64 on the CPU.

Test infrastructure only: this is the oracle the CUDA path is checked
against. Nothing in the product imports it.

Source: ``markov_head.py`` (the vendored DSpark-style low-rank Markov
sequential head), module docstring "WHAT THIS IS" and class
``VanillaMarkov``; and the API docs of
``nemo_automodel.components.speculative.dspark.markov_head``
(``VanillaMarkov``). The head keeps two weights, both stored ``[V, r]``:
``W1`` is an embedding table (row x is the latent of token x) and ``W2`` is
the weight of a bias-free ``Linear(r, V)`` (row v maps the latent to the
logit of token v). The transition bias of a previous token x is
``B(x, v) = sum_j W1[x, j] * W2[v, j]`` and a corrected logit is
``U_k[v] + B(x_{k-1}, v)``.

Readings where the pages leave a step open (each is listed with its reason in
the design notes):

* one rounding: the corrected logit is the exact sum rounded once
  (round-to-nearest-even) to the logits dtype; the pages round the bias to
  the weight dtype and then round again after the add;
* greedy selection takes the first (lowest) index among equal maxima of the
  ROUNDED corrected logits; NaN counts as larger than every number;
* temperature selection is Gumbel-max over Philox4x32-10 noise (see
  ``philox.py``), which draws from softmax(c / T) like the pages'
  softmax + multinomial, but not draw for draw;
* the returned corrected logits are the values before division by T.

All weights and logits are taken as the exact values of their storage dtype
converted to fp64; every sum below is an fp64 sum.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .philox import gumbel_noise
from .rounding import round_to

GREEDY_TEMPERATURE = 1e-5  # temperature below this (or None) means argmax


def get_prev_embeddings(w1: np.ndarray, token_ids) -> np.ndarray:
    """``VanillaMarkov.get_prev_embeddings``: the embedding rows W1[x].
    Ids outside [0, V) are an error, as they are for an embedding lookup."""
    ids = np.asarray(token_ids, dtype=np.int64)
    vocab = w1.shape[0]
    if ids.size and (ids.min() < 0 or ids.max() >= vocab):
        raise IndexError("token id outside [0, vocab)")
    return np.asarray(w1, dtype=np.float64)[ids]


def project_bias(latent: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """``VanillaMarkov.project_bias``: the bias-free Linear(r, V) whose weight
    is stored [V, r], i.e. latent @ W2^T."""
    return np.asarray(latent, dtype=np.float64) @ np.asarray(w2, dtype=np.float64).T


def compute_step_bias(w1, w2, token_ids, hidden_states=None) -> np.ndarray:
    """``VanillaMarkov.compute_step_bias``: the vanilla head is a pure function
    of the previous token; ``hidden_states`` is accepted and ignored."""
    del hidden_states
    return project_bias(get_prev_embeddings(w1, token_ids), w2)


def apply_step_logits(logits, w1, w2, token_ids, out_dtype: str, hidden_states=None) -> np.ndarray:
    """``VanillaMarkov.apply_step_logits`` for one position: (B, V) logits plus
    the bias of each row's previous token, rounded once to ``out_dtype``."""
    bias = compute_step_bias(w1, w2, token_ids, hidden_states)
    return round_to(out_dtype, np.asarray(logits, dtype=np.float64) + bias)


def apply_block_logits(base_logits, w1, w2, token_ids, out_dtype: str, hidden_states=None):
    """``VanillaMarkov.apply_block_logits``: teacher-forced bias for every
    position at once. Shape-agnostic over leading dims: ``base_logits`` is
    (..., M, V) and ``token_ids`` (..., M). When the input is empty, or its
    position axis has length 0, the input object itself is returned."""
    base = base_logits
    if np.size(base) == 0 or np.shape(base)[-2] == 0:
        return base_logits
    return round_to(out_dtype, exact_block_logits(base, w1, w2, token_ids, hidden_states))


def exact_block_logits(base_logits, w1, w2, token_ids, hidden_states=None) -> np.ndarray:
    """The unrounded corrected logits U + B(prev) of every position, in fp64."""
    base = np.asarray(base_logits, dtype=np.float64)
    vocab = base.shape[-1]
    ids = np.asarray(token_ids, dtype=np.int64).reshape(-1)
    bias = compute_step_bias(w1, w2, ids, hidden_states)
    return (base.reshape(-1, vocab) + bias).reshape(base.shape)


def transition_logits(w1, w2, token_ids, out_dtype: str):
    """``_DeepseekV41DSparkMarkovHead.forward`` (page
    nemo_automodel.components.models.deepseek_v41.dspark): for token ids of
    any shape (...), the transition bias alone, shape (..., V), rounded once to
    ``out_dtype`` (the module's dtype), and the conditioning embeddings W1[x],
    shape (..., r), which are exact copies of W1's rows."""
    ids = np.asarray(token_ids, dtype=np.int64)
    emb = get_prev_embeddings(w1, ids.reshape(-1))
    bias = project_bias(emb, w2)
    vocab, rank = np.shape(w2)[0], np.shape(w1)[1]
    return (round_to(out_dtype, bias).reshape(ids.shape + (vocab,)), emb.reshape(ids.shape + (rank,)))


def apply_block_logits_backward(grad_out, w1, w2, token_ids):
    """Gradients of the teacher-forced ``apply_block_logits`` (its train-time
    use: "At TRAIN time x_{k-1} is the teacher-forced ground-truth
    predecessor (apply_block_logits)"), in fp64. With out = U + W1[x] W2^T:

        dU = dOut (returned unchanged),
        dW2[v, j] = sum_i dOut[i, v] W1[x_i, j],
        dW1[x, j] = sum over rows i with x_i = x of sum_v dOut[i, v] W2[v, j]

    (the embedding lookup's backward adds each row's gradient at its id).
    ``grad_out`` is (..., M, V) and ``token_ids`` (..., M); returns
    (dW1 [V, r], dW2 [V, r])."""
    vocab = np.shape(w2)[0]
    dout = np.asarray(grad_out, dtype=np.float64).reshape(-1, vocab)
    ids = np.asarray(token_ids, dtype=np.int64).reshape(-1)
    emb = get_prev_embeddings(w1, ids)
    dw2 = dout.T @ emb
    d_emb = dout @ np.asarray(w2, dtype=np.float64)
    dw1 = np.zeros(np.shape(w1), dtype=np.float64)
    np.add.at(dw1, ids, d_emb)
    return dw1, dw2


def fused_lm_head_exact(hidden, lm_head, w1, w2, token_ids) -> np.ndarray:
    """The unrounded corrected logits with the base logits produced in the
    same pass, in fp64: U = hidden @ lm_head^T (the backbone's base logit,
    "lm_head(hidden_k)" in the module docstring of markov_head.py; the frozen
    vocabulary head of DeepseekV41DSparkModel.compute_logits, whose weight is
    [vocab, hidden]) plus the transition bias of each row's previous token.
    ``hidden`` is (..., d), ``token_ids`` (...); returns (..., V)."""
    h = np.asarray(hidden, dtype=np.float64)
    lm = np.asarray(lm_head, dtype=np.float64)
    lead = h.shape[:-1]
    ids = np.asarray(token_ids, dtype=np.int64).reshape(-1)
    u = h.reshape(-1, h.shape[-1]) @ lm.T
    return (u + compute_step_bias(w1, w2, ids)).reshape(lead + (lm.shape[0],))


def fused_lm_head_logits(hidden, lm_head, w1, w2, token_ids, out_dtype: str) -> np.ndarray:
    """``fused_lm_head_exact`` rounded once to ``out_dtype`` (compute_logits
    returns FP32; the head then adds its bias in that dtype)."""
    return round_to(out_dtype, fused_lm_head_exact(hidden, lm_head, w1, w2, token_ids))


def select_greedy(logits: np.ndarray) -> np.ndarray:
    """argmax over the last axis; the lowest index wins among equal maxima and
    NaN counts as the largest value (numpy's argmax has both properties)."""
    return np.argmax(np.asarray(logits), axis=-1).astype(np.int64)


def temperature_scores(logits_row: np.ndarray, temperature: float, seed: int, b: int, k: int) -> np.ndarray:
    """Gumbel-max score of every id for row b at step k: c / T + g."""
    c = np.asarray(logits_row, dtype=np.float64)
    return c / float(temperature) + gumbel_noise(seed, b, k, c.shape[-1])


def sample_tokens(step_logits: np.ndarray, temperature: Optional[float], seed: int, k: int) -> np.ndarray:
    """``_sample_tokens`` for one step of a (B, V) block row set: greedy when
    ``temperature`` is None or below 1e-5, else one draw per row from
    softmax(logits / T), taken as argmax(logits / T + Gumbel noise)."""
    if temperature is None or temperature < GREEDY_TEMPERATURE:
        return select_greedy(step_logits)
    return np.array([int(np.argmax(temperature_scores(step_logits[b], temperature, seed, b, k)))
                     for b in range(step_logits.shape[0])], dtype=np.int64)


def sample_block_tokens(base_logits, w1, w2, first_prev_token_ids, out_dtype: str,
                        temperature: Optional[float] = 0.0, seed: int = 0,
                        hidden_states=None) -> Tuple[np.ndarray, np.ndarray]:
    """``VanillaMarkov.sample_block_tokens``: left-to-right over the M
    positions of each of the B blocks. Position k is corrected with the bias of
    the token chosen at k-1 (``first_prev_token_ids`` before position 0), and
    its own choice feeds position k+1. Returns (tokens (B, M) int64,
    corrected logits (B, M, V)). With M == 0 it returns an empty (B, 0) token
    array and the input object itself."""
    base = base_logits
    batch, proposal_len = np.shape(base)[:2]
    if proposal_len == 0:
        return np.empty((batch, 0), dtype=np.int64), base_logits
    base = np.asarray(base, dtype=np.float64)
    prev = np.asarray(first_prev_token_ids, dtype=np.int64)
    tokens = np.empty((batch, proposal_len), dtype=np.int64)
    corrected = np.empty(base.shape, dtype=np.float64)
    for k in range(proposal_len):
        step = apply_step_logits(base[:, k, :], w1, w2, prev, out_dtype, hidden_states)
        corrected[:, k, :] = step
        nxt = sample_tokens(step, temperature, seed, k)
        tokens[:, k] = nxt
        prev = nxt
    return tokens, corrected
