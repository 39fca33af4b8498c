"""``VanillaMarkov``: the rank-r Markov transition-bias head on B200.

Python face of the C ABI: torch tensors supply device memory and the current
CUDA stream; every step of the computation runs in the library's kernels.

The method (markov_head.py, the vendored DSpark-style low-rank Markov head,
module docstring "WHAT THIS IS"; nemo_automodel ...speculative.dspark.markov_head
API docs, ``VanillaMarkov``): a parallel block drafter gives base logits U_k
for every position k of a block in one pass; the head adds
B(x_{k-1}, :) = W2(W1[x_{k-1}]) with W1 an embedding [V, r] and W2 a
bias-free Linear(r, V) (weight [V, r]). Training uses the teacher-forced
predecessor (``apply_block_logits``); inference samples left to right
(``sample_block_tokens``).
"""
from __future__ import annotations

import functools
import math
import os
from typing import Optional, Tuple

import torch

from . import _native as N

_DT = {torch.float32: N.DSPARK_DTYPE_FP32, torch.bfloat16: N.DSPARK_DTYPE_BF16}

# Every entry point runs inside an NVTX range named "dspark_markov.<method>",
# so that a profiler's timeline shows the library's calls around its kernels.
# DSPARK_NVTX=0 in the environment (read at import) leaves the ranges out.
_NVTX = os.environ.get("DSPARK_NVTX", "1") != "0"


def _ranged(fn):
    name = "dspark_markov." + fn.__name__

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        if not _NVTX:
            return fn(*args, **kwargs)
        torch.cuda.nvtx.range_push(name)
        try:
            return fn(*args, **kwargs)
        finally:
            torch.cuda.nvtx.range_pop()

    return wrapper


def _stream_ptr(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_cuda(t: torch.Tensor, name: str, device: torch.device) -> None:
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class VanillaMarkov:
    """Memoryless low-rank transition bias with caller-owned weights.

    ``w1`` (embedding table) and ``w2`` (``Linear(rank, vocab)`` weight) are
    both ``[vocab, rank]`` CUDA tensors of one dtype (fp32 or bf16). The head
    requires ``rank > 0`` (``VanillaMarkov.__init__`` asserts it).
    """

    markov_head_type = "vanilla"

    def __init__(self, w1: torch.Tensor, w2: torch.Tensor):
        if w1.dim() != 2 or w1.shape != w2.shape:
            raise ValueError("w1 and w2 must both be [vocab, rank]")
        if w1.dtype not in _DT or w2.dtype not in _DT:
            raise ValueError("weights must be float32 or bfloat16")
        if w1.dtype != w2.dtype:
            raise ValueError("w1 and w2 must share a dtype")
        self.vocab_size, self.markov_rank = int(w1.shape[0]), int(w1.shape[1])
        if self.markov_rank <= 0:
            raise ValueError(f"VanillaMarkov requires markov_rank > 0, got {self.markov_rank}")
        _check_cuda(w1, "w1", w1.device)
        _check_cuda(w2, "w2", w1.device)
        self.device = w1.device
        self.markov_w1 = w1
        self.markov_w2 = w2
        self._lib = N.load()

    @property
    def weight_dtype(self) -> torch.dtype:
        return self.markov_w1.dtype

    # ------------------------------------------------------------------ apply
    @_ranged
    def apply_block_logits(self, base_logits: torch.Tensor, *, token_ids: torch.Tensor,
                           hidden_states: Optional[torch.Tensor] = None,
                           out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Teacher-forced corrected logits, shape-agnostic over leading dims:
        ``base_logits`` (..., M, V), ``token_ids`` (..., M). Returns
        ``base_logits`` itself when it is empty or M == 0. ``hidden_states``
        is accepted and ignored (the vanilla head is a function of the
        previous token only). ``out`` may be ``base_logits`` (in place)."""
        del hidden_states
        if base_logits.numel() == 0 or base_logits.shape[-2] == 0:
            return base_logits
        vocab = base_logits.shape[-1]
        if vocab != self.vocab_size:
            raise ValueError(f"vocab mismatch: logits {vocab} vs head {self.vocab_size}")
        if tuple(token_ids.shape) != tuple(base_logits.shape[:-1]):
            raise ValueError("token_ids must match base_logits without its last dim")
        if base_logits.dtype not in _DT:
            raise ValueError("logits must be float32 or bfloat16")
        _check_cuda(base_logits, "base_logits", self.device)
        ids = token_ids if token_ids.dtype == torch.int64 else token_ids.long()
        ids = ids.contiguous()
        _check_cuda(ids, "token_ids", self.device)
        if out is None:
            out = torch.empty_like(base_logits)
        else:
            if out.shape != base_logits.shape or out.dtype != base_logits.dtype:
                raise ValueError("out must match base_logits in shape and dtype")
            _check_cuda(out, "out", self.device)
        rows = base_logits.numel() // vocab
        code = self._lib.dspark_markov_apply_block_logits(
            base_logits.data_ptr(), out.data_ptr(), ids.data_ptr(), rows, vocab, self.markov_w1.data_ptr(),
            self.markov_w2.data_ptr(), self.markov_rank, _DT[base_logits.dtype], _DT[self.weight_dtype],
            _stream_ptr(self.device))
        N.check(code, "dspark_markov_apply_block_logits")
        return out

    @_ranged
    def fused_lm_head_logits(self, hidden_states: torch.Tensor, lm_head_weight: torch.Tensor, *,
                             token_ids: torch.Tensor, out_dtype: torch.dtype = torch.float32,
                             out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Corrected logits with the base logits made in the same kernel:
        round(hidden @ lm_head_weight^T + bias(token_ids)), one fp32
        accumulation and one rounding, the base logits never stored.
        ``hidden_states`` (..., d) and ``lm_head_weight`` [V, d] are bf16 like
        the head's weights; ``token_ids`` (...) are the teacher-forced previous
        tokens. Returns (..., V) in ``out_dtype`` (fp32, as compute_logits
        gives, or bf16)."""
        d = hidden_states.shape[-1]
        if tuple(lm_head_weight.shape) != (self.vocab_size, d):
            raise ValueError(f"lm_head_weight must be [{self.vocab_size}, {d}]")
        if tuple(token_ids.shape) != tuple(hidden_states.shape[:-1]):
            raise ValueError("token_ids must match hidden_states without its last dim")
        if hidden_states.dtype != self.weight_dtype or lm_head_weight.dtype != self.weight_dtype:
            raise ValueError("hidden_states and lm_head_weight must have the head's weight dtype")
        if out_dtype not in _DT:
            raise ValueError("out_dtype must be float32 or bfloat16")
        _check_cuda(hidden_states, "hidden_states", self.device)
        _check_cuda(lm_head_weight, "lm_head_weight", self.device)
        ids = (token_ids if token_ids.dtype == torch.int64 else token_ids.long()).contiguous()
        _check_cuda(ids, "token_ids", self.device)
        shape = tuple(hidden_states.shape[:-1]) + (self.vocab_size,)
        if out is None:
            out = torch.empty(shape, dtype=out_dtype, device=self.device)
        else:
            if tuple(out.shape) != shape or out.dtype != out_dtype:
                raise ValueError("out must be (..., V) of out_dtype")
            _check_cuda(out, "out", self.device)
        rows = hidden_states.numel() // d
        if rows == 0:
            return out
        code = self._lib.dspark_markov_fused_lm_head_logits(
            hidden_states.data_ptr(), ids.data_ptr(), rows, d, self.vocab_size, lm_head_weight.data_ptr(),
            self.markov_w1.data_ptr(), self.markov_w2.data_ptr(), self.markov_rank, out.data_ptr(), _DT[out_dtype],
            _DT[self.weight_dtype], _stream_ptr(self.device))
        N.check(code, "dspark_markov_fused_lm_head_logits")
        return out

    @_ranged
    def apply_step_logits(self, logits: torch.Tensor, *, token_ids: torch.Tensor,
                          hidden_states: Optional[torch.Tensor] = None) -> torch.Tensor:
        """One position (B, V) with its (B,) previous tokens."""
        return self.apply_block_logits(logits.unsqueeze(-2), token_ids=token_ids.unsqueeze(-1),
                                       hidden_states=hidden_states).squeeze(-2)

    @_ranged
    def apply_block_logits_backward(self, grad_out: torch.Tensor, *, token_ids: torch.Tensor,
                                    grad_w1: Optional[torch.Tensor] = None, grad_w2: Optional[torch.Tensor] = None,
                                    accumulate: bool = False, want_w1: bool = True, want_w2: bool = True):
        """Gradients of ``apply_block_logits`` with respect to W1 and W2 (fp32,
        [V, r]) for ``grad_out`` (..., M, V) and the teacher-forced
        ``token_ids`` (..., M); the gradient of the base logits is
        ``grad_out`` itself. ``accumulate`` adds into given buffers."""
        vocab, rank = self.vocab_size, self.markov_rank
        if grad_out.shape[-1] != vocab or tuple(token_ids.shape) != tuple(grad_out.shape[:-1]):
            raise ValueError("grad_out must be (..., V) with token_ids (...)")
        if grad_out.dtype not in _DT:
            raise ValueError("grad_out must be float32 or bfloat16")
        g = grad_out.contiguous()
        _check_cuda(g, "grad_out", self.device)
        ids = (token_ids if token_ids.dtype == torch.int64 else token_ids.long()).contiguous()
        _check_cuda(ids, "token_ids", self.device)
        outs = []
        for want, buf, name in ((want_w1, grad_w1, "grad_w1"), (want_w2, grad_w2, "grad_w2")):
            if not want:
                outs.append(None)
                continue
            if buf is None:
                if accumulate:
                    raise ValueError(f"accumulate needs {name}")
                buf = torch.empty(vocab, rank, dtype=torch.float32, device=self.device)
            elif tuple(buf.shape) != (vocab, rank) or buf.dtype != torch.float32:
                raise ValueError(f"{name} must be fp32 (V, r)")
            _check_cuda(buf, name, self.device)
            outs.append(buf)
        code = self._lib.dspark_markov_apply_block_logits_backward(
            g.data_ptr(), ids.data_ptr(), ids.numel(), vocab, self.markov_w1.data_ptr(), self.markov_w2.data_ptr(),
            rank, outs[0].data_ptr() if outs[0] is not None else None,
            outs[1].data_ptr() if outs[1] is not None else None, 1 if accumulate else 0, _DT[g.dtype],
            _DT[self.weight_dtype], _stream_ptr(self.device))
        N.check(code, "dspark_markov_apply_block_logits_backward")
        return outs[0], outs[1]

    @_ranged
    def transition_logits(self, token_ids: torch.Tensor, *, with_embeddings: bool = True,
                          out: Optional[torch.Tensor] = None,
                          out_embeddings: Optional[torch.Tensor] = None):
        """The bias alone and its conditioning embeddings, for token ids of
        any shape (...): returns (transition (..., V), embeddings (..., r) or
        None), both in the weights' dtype (_DeepseekV41DSparkMarkovHead.forward).
        The bias is accumulated in fp32 and rounded once."""
        ids = token_ids if token_ids.dtype == torch.int64 else token_ids.long()
        ids = ids.contiguous()
        _check_cuda(ids, "token_ids", self.device)
        shape = tuple(ids.shape)
        wdt = self.weight_dtype
        if out is None:
            out = torch.empty(*shape, self.vocab_size, dtype=wdt, device=self.device)
        elif tuple(out.shape) != shape + (self.vocab_size,) or out.dtype != wdt:
            raise ValueError("out must be (..., V) in the weights' dtype")
        emb = None
        if with_embeddings:
            emb = out_embeddings if out_embeddings is not None else \
                torch.empty(*shape, self.markov_rank, dtype=wdt, device=self.device)
            if tuple(emb.shape) != shape + (self.markov_rank,) or emb.dtype != wdt:
                raise ValueError("out_embeddings must be (..., r) in the weights' dtype")
            _check_cuda(emb, "out_embeddings", self.device)
        _check_cuda(out, "out", self.device)
        rows = ids.numel()
        if rows == 0:
            return out, emb
        code = self._lib.dspark_markov_transition_logits(
            ids.data_ptr(), rows, self.vocab_size, self.markov_w1.data_ptr(), self.markov_w2.data_ptr(),
            self.markov_rank, out.data_ptr(), emb.data_ptr() if emb is not None else None, _DT[wdt],
            _stream_ptr(self.device))
        N.check(code, "dspark_markov_transition_logits")
        return out, emb

    # ----------------------------------------------------------------- sample
    @_ranged
    def sample_block_tokens(self, base_logits: torch.Tensor, *, first_prev_token_ids: torch.Tensor,
                            hidden_states: Optional[torch.Tensor] = None, temperature: Optional[float] = 0.0,
                            seed: int = 0, out_tokens: Optional[torch.Tensor] = None,
                            out_logits: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
        """Left-to-right sampling of ``base_logits`` (B, M, V). Returns
        (sampled_tokens (B, M) int64, corrected_logits (B, M, V)). With M == 0
        returns an empty (B, 0) token tensor and ``base_logits`` itself.
        ``temperature`` None or below 1e-5 is greedy; otherwise each token is
        a Gumbel-max draw from softmax(c / T) with Philox noise keyed by
        ``seed``. ``hidden_states`` is accepted and ignored."""
        del hidden_states
        if base_logits.dim() != 3:
            raise ValueError("base_logits must be (B, M, V)")
        batch, m, vocab = base_logits.shape
        if m == 0:
            return torch.empty(batch, 0, dtype=torch.long, device=base_logits.device), base_logits
        if vocab != self.vocab_size:
            raise ValueError(f"vocab mismatch: logits {vocab} vs head {self.vocab_size}")
        if base_logits.dtype not in _DT:
            raise ValueError("logits must be float32 or bfloat16")
        _check_cuda(base_logits, "base_logits", self.device)
        prev = first_prev_token_ids if first_prev_token_ids.dtype == torch.int64 else first_prev_token_ids.long()
        prev = prev.contiguous()
        if tuple(prev.shape) != (batch,):
            raise ValueError("first_prev_token_ids must be (B,)")
        _check_cuda(prev, "first_prev_token_ids", self.device)
        t = 0.0 if temperature is None else float(temperature)
        if math.isnan(t):
            raise ValueError("temperature is NaN")
        tokens = out_tokens if out_tokens is not None else torch.empty(batch, m, dtype=torch.long, device=self.device)
        corrected = out_logits if out_logits is not None else torch.empty_like(base_logits)
        code = self._lib.dspark_markov_sample_block(
            base_logits.data_ptr(), prev.data_ptr(), batch, m, vocab, self.markov_w1.data_ptr(),
            self.markov_w2.data_ptr(), self.markov_rank, t, seed & 0xFFFFFFFFFFFFFFFF, tokens.data_ptr(),
            corrected.data_ptr(), _DT[base_logits.dtype], _DT[self.weight_dtype], _stream_ptr(self.device))
        N.check(code, "dspark_markov_sample_block")
        return tokens, corrected

    @_ranged
    def sample_block_tokens_noalloc(self, base_logits: torch.Tensor, *, first_prev_token_ids: torch.Tensor,
                                    out_tokens: torch.Tensor, out_logits: torch.Tensor,
                                    temperature: Optional[float] = 0.0, seed: int = 0) -> None:
        """``sample_block_tokens`` for callers that must not allocate device
        memory during the call (memory reserved up front, an allocator lock
        held): the outputs are caller-provided, ``first_prev_token_ids`` must
        already be contiguous int64 on the head's device, and the library's
        fixed static scratch replaces its growable workspace. Requires
        B * M <= 8192 and a shape the tensor-core sampler takes. Calls that
        overlap on one device race on the shared scratch; the first call on a
        device should come before any stream capture."""
        if base_logits.dim() != 3:
            raise ValueError("base_logits must be (B, M, V)")
        batch, m, vocab = base_logits.shape
        if vocab != self.vocab_size:
            raise ValueError(f"vocab mismatch: logits {vocab} vs head {self.vocab_size}")
        if base_logits.dtype not in _DT:
            raise ValueError("logits must be float32 or bfloat16")
        prev = first_prev_token_ids
        if prev.dtype != torch.int64 or not prev.is_contiguous() or tuple(prev.shape) != (batch,):
            raise ValueError("first_prev_token_ids must be contiguous int64 (B,)")
        if tuple(out_tokens.shape) != (batch, m) or out_tokens.dtype != torch.int64 or not out_tokens.is_contiguous():
            raise ValueError("out_tokens must be contiguous int64 (B, M)")
        if out_logits.shape != base_logits.shape or out_logits.dtype != base_logits.dtype or \
                not out_logits.is_contiguous():
            raise ValueError("out_logits must be contiguous with the shape and dtype of base_logits")
        for t, name in ((base_logits, "base_logits"), (prev, "first_prev_token_ids"), (out_tokens, "out_tokens"),
                        (out_logits, "out_logits")):
            _check_cuda(t, name, self.device)
        t = 0.0 if temperature is None else float(temperature)
        if math.isnan(t):
            raise ValueError("temperature is NaN")
        code = self._lib.dspark_markov_sample_block_noalloc(
            base_logits.data_ptr(), prev.data_ptr(), batch, m, vocab, self.markov_w1.data_ptr(),
            self.markov_w2.data_ptr(), self.markov_rank, t, seed & 0xFFFFFFFFFFFFFFFF, out_tokens.data_ptr(),
            out_logits.data_ptr(), _DT[base_logits.dtype], _DT[self.weight_dtype], _stream_ptr(self.device))
        N.check(code, "dspark_markov_sample_block_noalloc")


def build_markov_head(w1: Optional[torch.Tensor], w2: Optional[torch.Tensor], markov_rank: int,
                      head_type: str = "vanilla") -> Optional[VanillaMarkov]:
    """``build_markov_head``: None when ``markov_rank == 0`` (head disabled);
    a negative rank is an error; only the vanilla head is built here."""
    markov_rank = int(markov_rank)
    if markov_rank < 0:
        raise ValueError(f"markov_rank must be >= 0, got {markov_rank}")
    if markov_rank == 0:
        return None
    if str(head_type).lower() != "vanilla":
        raise ValueError(f"Unsupported markov_head_type={head_type!r}; only 'vanilla' is built")
    return VanillaMarkov(w1, w2)


def device_status(device: Optional[torch.device] = None) -> int:
    """Synchronise the current stream, then read and clear the device status
    word (DSPARK_STATUS_* bits)."""
    import ctypes
    dev = device or torch.device("cuda", torch.cuda.current_device())
    out = ctypes.c_int32(0)
    with torch.cuda.device(dev):
        N.check(N.load().dspark_markov_get_status(_stream_ptr(dev), ctypes.byref(out)), "dspark_markov_get_status")
    return int(out.value)


def set_algo(algo: int) -> int:
    return int(N.load().dspark_markov_set_algo(int(algo)))


def launch_count() -> int:
    return int(N.load().dspark_markov_launch_count())


def last_algo() -> int:
    return int(N.load().dspark_markov_last_algo())


def last_variant() -> int:
    """DSPARK_VARIANT_* bits of the tensor-core variants the last call on this
    thread launched."""
    return int(N.load().dspark_markov_last_variant())


def set_debug(flags: int, wait_limit_ns: int = 0) -> None:
    N.check(N.load().dspark_markov_set_debug(int(flags), int(wait_limit_ns)), "dspark_markov_set_debug")
