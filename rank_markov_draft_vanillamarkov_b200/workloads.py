"""Seeded synthetic inputs for the Markov transition-bias head.

This module only draws inputs. It holds none of the head's arithmetic, and
both the CUDA path and the CPU oracle are fed from it. Everything is drawn on
the CPU from a seeded ``torch.Generator`` so that a given workload is the same
bytes on every machine.

Shapes and value distributions follow the DSpark pages:

* vocabulary 129280 and Markov rank up to 256 come from the DeepSeek-V4.1
  DSpark config (``DeepseekV41TextConfig``: ``vocab_size``,
  ``dspark_markov_rank``), block size 5 from ``dspark_block_size``, the
  weight scale 0.02 from ``initializer_range`` and the padding id 2 from
  ``pad_token_id``;
* the teacher-forced layout ``[B, num_blocks, block_size, V]`` and the
  sampling layout ``[B, M, V]`` come from the markov_head module docs
  (``RNNHead.apply_block_logits``, ``RNNHead.sample_block_tokens``);
* "N(0, s)" means a normal draw with standard deviation ``s``, made in fp32
  and then rounded to the storage dtype; the rounded values are the ground
  truth handed to both sides.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

PAD_TOKEN_ID = 2  # DeepseekV41TextConfig.pad_token_id

_DTYPES = {"bf16": torch.bfloat16, "fp32": torch.float32}


@dataclass(frozen=True)
class Workload:
    """One seeded synthetic workload.

    ``mode`` is ``"apply"`` (teacher-forced, rows = batch * num_blocks *
    block_size), ``"backward"`` (the apply's gradients for W1 and W2; the
    base-logit tensor serves as the incoming gradient), ``"transition"``
    (the bias alone and the embeddings of the same rows, no base logits) or
    ``"sample"`` (left-to-right, ``batch`` blocks of ``proposal_len``
    positions) or ``"fused"`` (teacher-forced, with the base logits made
    from hidden states of width ``hidden`` by an LM-head weight [V, hidden];
    ``logits_dtype`` is then the output dtype).
    """

    name: str
    mode: str
    vocab: int
    rank: int
    batch: int
    num_blocks: int = 1
    block_size: int = 5
    proposal_len: int = 5
    logits_dtype: str = "bf16"
    weight_dtype: str = "bf16"
    logit_std: float = 2.0
    weight_std: float = 0.02
    prev_dist: str = "uniform"  # "uniform" or "zipf1.1"
    spike: float = 0.0  # added at one uniform id per (b, k) before rounding
    pad_frac: float = 0.0  # fraction of (b, block) pairs whose prev ids are the pad id
    temperature: float = 0.0
    philox_seed: int = 0
    data_seed: int = 0
    hidden: int = 0  # fused: width of the hidden states
    hidden_std: float = 1.0  # fused: hidden states ~N(0, hidden_std)
    lm_std: float = 0.02  # fused: LM-head weight ~N(0, lm_std)

    @property
    def rows(self) -> int:
        return self.batch * self.num_blocks * self.block_size

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def bytes_moved(self) -> int:
        """Algorithmic HBM bytes of one call: logits in and out, W2 once,
        the gathered W1 rows and the ids."""
        lb = 2 if self.logits_dtype == "bf16" else 4
        wb = 2 if self.weight_dtype == "bf16" else 4
        if self.mode == "apply":
            r = self.rows
            return 2 * r * self.vocab * lb + self.vocab * self.rank * wb + r * self.rank * wb + r * 8
        if self.mode == "backward":  # grad in, W2 and W1 rows in, ids, two fp32 [V, r] gradients out
            r = self.rows
            return r * self.vocab * lb + self.vocab * self.rank * wb + r * self.rank * wb + r * 8 \
                + 2 * self.vocab * self.rank * 4
        if self.mode == "fused":  # hidden in, LM head and W2 once, W1 rows, ids, logits out
            r = self.rows
            return (r * self.hidden * wb + self.vocab * self.hidden * wb + self.vocab * self.rank * wb
                    + r * self.rank * wb + r * 8 + r * self.vocab * lb)
        if self.mode == "transition":  # bias out, W2, W1 rows in and embeddings out, ids
            r = self.rows
            return r * self.vocab * wb + self.vocab * self.rank * wb + 2 * r * self.rank * wb + r * 8
        r = self.batch * self.proposal_len
        return (2 * r * self.vocab * lb + self.vocab * self.rank * wb + r * self.rank * wb
                + self.batch * 8 + r * 8)

    def flops(self) -> int:
        if self.mode == "fused":
            return 2 * self.rows * self.vocab * (self.hidden + self.rank)
        r = self.rows if self.mode in ("apply", "transition") else self.batch * self.proposal_len
        if self.mode == "backward":  # dW2 and dW1 each cost one product per (row, id, rank) term
            return 4 * self.rows * self.vocab * self.rank
        return 2 * r * self.vocab * self.rank


# The five workloads of the method's hot path, named by what they are.
TINY_FP32 = Workload("tiny_fp32_v1024_r16", "apply", vocab=1024, rank=16, batch=2, num_blocks=1,
                     block_size=5, proposal_len=5, logits_dtype="fp32", weight_dtype="fp32",
                     logit_std=1.0, weight_std=0.02, prev_dist="uniform", data_seed=0)
APPLY_320 = Workload("apply_r320_v129280_k128", "apply", vocab=129280, rank=128, batch=4,
                     num_blocks=16, block_size=5, logit_std=2.0, weight_std=0.02,
                     prev_dist="zipf1.1", data_seed=0)
GREEDY = Workload("greedy_m5_v129280_k128", "sample", vocab=129280, rank=128, batch=32,
                  proposal_len=5, logit_std=2.0, weight_std=0.05, spike=6.0, temperature=0.0,
                  data_seed=0)
TEMPERATURE = Workload("temp0.7_b32_m8_v151936_k64", "sample", vocab=151936, rank=64, batch=32,
                       proposal_len=8, logit_std=1.5, weight_std=0.05, temperature=0.7,
                       philox_seed=1234, data_seed=0)
BACKWARD_320 = Workload("backward_r320_v129280_k128", "backward", vocab=129280, rank=128, batch=4,
                        num_blocks=16, block_size=5, logit_std=1.0, weight_std=0.02, prev_dist="zipf1.1",
                        data_seed=0)
APPLY_320_FP32 = Workload("apply_fp32logits_r320_v129280_k128", "apply", vocab=129280, rank=128, batch=4,
                          num_blocks=16, block_size=5, logits_dtype="fp32", weight_dtype="bf16", logit_std=2.0,
                          weight_std=0.02, prev_dist="zipf1.1", data_seed=0)
TRANSITION_320 = Workload("transition_r320_v129280_k128", "transition", vocab=129280, rank=128, batch=4,
                          num_blocks=16, block_size=5, weight_std=0.02, prev_dist="zipf1.1", data_seed=0)
APPLY_2560 = Workload("apply_r2560_v129280_k256_pad20", "apply", vocab=129280, rank=256, batch=8,
                      num_blocks=64, block_size=5, logit_std=2.0, weight_std=0.02,
                      prev_dist="zipf1.1", pad_frac=0.2, data_seed=0)

# The fused producer on the 320-row layout: hidden width 5120 and the LM head
# [129280, 5120] of DeepseekV41TextConfig (hidden_size, vocab_size), fp32
# output as compute_logits gives.
FUSED_320 = Workload("fused_lmhead_r320_d5120_v129280_k128", "fused", vocab=129280, rank=128, batch=4,
                     num_blocks=16, block_size=5, logits_dtype="fp32", weight_std=0.02, prev_dist="zipf1.1",
                     hidden=5120, hidden_std=1.0, lm_std=0.02, data_seed=0)

GREEDY_BATCHES = (1, 8, 32, 64)


def greedy(batch: int) -> Workload:
    return GREEDY.with_(name=f"greedy_b{batch}_m5_v129280_k128", batch=batch)


def _normal(g: torch.Generator, shape, std: float, dtype: str) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32) * std
    return x.to(_DTYPES[dtype])


def zipf_ids(g: torch.Generator, n: int, vocab: int, s: float = 1.1) -> torch.Tensor:
    """Ids with p(i) proportional to (i+1)^-s on [0, vocab), by inverse CDF
    on the finite support; the id is the rank (no permutation)."""
    w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = torch.rand(n, generator=g, dtype=torch.float64).numpy()
    ids = np.searchsorted(cdf, u, side="right")
    return torch.from_numpy(np.minimum(ids, vocab - 1).astype(np.int64))


def uniform_ids(g: torch.Generator, n: int, vocab: int) -> torch.Tensor:
    return torch.randint(0, vocab, (n,), generator=g, dtype=torch.int64)


def make_weights(wl: Workload, g: Optional[torch.Generator] = None):
    """W1 (embedding, [V, r]) and W2 (Linear(r, V) weight, stored [V, r])."""
    g = g if g is not None else torch.Generator().manual_seed(wl.data_seed)
    w1 = _normal(g, (wl.vocab, wl.rank), wl.weight_std, wl.weight_dtype)
    w2 = _normal(g, (wl.vocab, wl.rank), wl.weight_std, wl.weight_dtype)
    return w1, w2


def make_inputs(wl: Workload) -> dict:
    """All CPU tensors of one workload.

    apply:  base [B, nb, bs, V], prev_ids [B, nb, bs] int64, pad_mask [B, nb]
    sample: base [B, M, V], first_prev [B] int64
    fused:  hidden [B, nb, bs, d], lm_head [V, d], prev_ids [B, nb, bs] int64
    plus w1, w2 [V, r].
    """
    g = torch.Generator().manual_seed(wl.data_seed)
    w1, w2 = make_weights(wl, g)
    out = {"w1": w1, "w2": w2}
    if wl.mode == "fused":
        n = wl.rows
        ids = zipf_ids(g, n, wl.vocab, 1.1) if wl.prev_dist == "zipf1.1" else uniform_ids(g, n, wl.vocab)
        out["prev_ids"] = ids.view(wl.batch, wl.num_blocks, wl.block_size)
        out["hidden"] = _normal(g, (wl.batch, wl.num_blocks, wl.block_size, wl.hidden), wl.hidden_std,
                                wl.weight_dtype)
        out["lm_head"] = _normal(g, (wl.vocab, wl.hidden), wl.lm_std, wl.weight_dtype)
    elif wl.mode == "transition":
        n = wl.rows
        ids = zipf_ids(g, n, wl.vocab, 1.1) if wl.prev_dist == "zipf1.1" else uniform_ids(g, n, wl.vocab)
        out["prev_ids"] = ids.view(wl.batch, wl.num_blocks, wl.block_size)
    elif wl.mode in ("apply", "backward"):
        shape = (wl.batch, wl.num_blocks, wl.block_size, wl.vocab)
        base = _normal(g, shape, wl.logit_std, wl.logits_dtype)
        n = wl.rows
        if wl.prev_dist == "zipf1.1":
            ids = zipf_ids(g, n, wl.vocab, 1.1)
        else:
            ids = uniform_ids(g, n, wl.vocab)
        ids = ids.view(wl.batch, wl.num_blocks, wl.block_size)
        pad = torch.zeros(wl.batch, wl.num_blocks, dtype=torch.bool)
        if wl.pad_frac > 0:
            npairs = wl.batch * wl.num_blocks
            k = int(round(wl.pad_frac * npairs))
            sel = torch.randperm(npairs, generator=g)[:k]
            pad.view(-1)[sel] = True
            ids = ids.clone()
            ids[pad] = PAD_TOKEN_ID
        out.update(base=base, prev_ids=ids, pad_mask=pad)
    else:
        shape = (wl.batch, wl.proposal_len, wl.vocab)
        x = torch.randn(*shape, generator=g, dtype=torch.float32) * wl.logit_std
        if wl.spike:
            at = torch.randint(0, wl.vocab, (wl.batch, wl.proposal_len), generator=g)
            x.scatter_add_(2, at.unsqueeze(-1), torch.full((wl.batch, wl.proposal_len, 1), float(wl.spike)))
        out["base"] = x.to(_DTYPES[wl.logits_dtype])
        out["first_prev"] = uniform_ids(g, wl.batch, wl.vocab)
    return out


def small_variants():
    """Shapes the oracle finishes in seconds that still span several 128-wide
    tiles and leave ragged tails (rows and vocab not multiples of 128)."""
    return [
        Workload("apply_small_r200_v1000_k64", "apply", vocab=1000, rank=64, batch=2, num_blocks=20,
                 block_size=5, weight_std=0.3, prev_dist="zipf1.1", data_seed=11),
        Workload("apply_small_r330_v2056_k128", "apply", vocab=2056, rank=128, batch=3, num_blocks=22,
                 block_size=5, weight_std=0.3, prev_dist="uniform", data_seed=12),
        Workload("apply_small_r135_v4096_k256_pad", "apply", vocab=4096, rank=256, batch=3, num_blocks=9,
                 block_size=5, weight_std=0.2, prev_dist="zipf1.1", pad_frac=0.2, data_seed=13),
    ]
