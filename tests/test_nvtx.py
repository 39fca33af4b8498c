"""The binding's entry points run inside NVTX ranges named after them (the
tracing row of the survey's auxiliary subsystems). Host logic only: the NVTX
calls are recorded, not sent to a profiler."""
import pytest
import torch

from rank_markov_draft_vanillamarkov_b200 import head as H
from rank_markov_draft_vanillamarkov_b200.head import VanillaMarkov


@pytest.fixture
def recorder(monkeypatch):
    calls = []
    monkeypatch.setattr(torch.cuda.nvtx, "range_push", lambda name: calls.append(("push", name)))
    monkeypatch.setattr(torch.cuda.nvtx, "range_pop", lambda: calls.append(("pop", None)))
    monkeypatch.setattr(H, "_NVTX", True)
    return calls


def test_range_wraps_the_call_and_keeps_its_result(recorder):
    @H._ranged
    def apply_block_logits(x, *, y):
        recorder.append(("body", x + y))
        return x * y

    assert apply_block_logits(3, y=4) == 12
    assert recorder == [("push", "dspark_markov.apply_block_logits"), ("body", 7), ("pop", None)]


def test_range_is_popped_when_the_call_raises(recorder):
    @H._ranged
    def sample_block_tokens():
        raise ValueError("bad shape")

    with pytest.raises(ValueError):
        sample_block_tokens()
    assert recorder == [("push", "dspark_markov.sample_block_tokens"), ("pop", None)]


def test_disabled_ranges_make_no_calls(recorder, monkeypatch):
    monkeypatch.setattr(H, "_NVTX", False)

    @H._ranged
    def transition_logits():
        return "ok"

    assert transition_logits() == "ok" and recorder == []


@pytest.mark.parametrize("method", ["apply_block_logits", "fused_lm_head_logits", "apply_step_logits",
                                    "apply_block_logits_backward", "transition_logits", "sample_block_tokens",
                                    "sample_block_tokens_noalloc"])
def test_every_entry_point_is_ranged(method):
    fn = getattr(VanillaMarkov, method)
    assert fn.__wrapped__.__name__ == method  # functools.wraps of _ranged
