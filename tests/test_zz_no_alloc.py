"""The no-allocation sampler entry (dspark_markov_sample_block_noalloc) against
the allocating one (dspark_markov_sample_block), through the C ABI, on B200.

Both run the same tensor-core kernel; only where the step maxima and the
barrier counter live differs (a fixed static scratch instead of a growable
workspace). So two calls in a row of the no-allocation entry must each give
exactly the tokens of the allocating entry and logits within one bf16 ulp
(in practice identical). This file is collected last so that it also runs
after every other test in the same process; it must pass alone as well.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle.checks import check_sampled_block
from rank_markov_draft_vanillamarkov_b200 import VanillaMarkov, device_status, set_algo
from rank_markov_draft_vanillamarkov_b200 import _native as N
from rank_markov_draft_vanillamarkov_b200 import workloads as W
from rank_markov_draft_vanillamarkov_b200.build import build

from _helpers import f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    build()
    lib = N.load()
    set_algo(N.DSPARK_ALGO_AUTO)
    return lib


def _call(lib, fn_name, d, base, first, temperature, seed, tokens, corr):
    stream = torch.cuda.current_stream().cuda_stream
    fn = getattr(lib, fn_name)
    return fn(base.data_ptr(), first.data_ptr(), base.shape[0], base.shape[1], base.shape[2], d["w1"].data_ptr(),
              d["w2"].data_ptr(), d["w1"].shape[1], float(temperature), seed, tokens.data_ptr(), corr.data_ptr(),
              N.DSPARK_DTYPE_BF16, N.DSPARK_DTYPE_BF16, stream)


def _within_one_ulp(a: torch.Tensor, b: torch.Tensor) -> bool:
    a64, b64 = f64(a), f64(b)
    mag = np.maximum(np.abs(a64), np.abs(b64))
    ulp = np.exp2(np.floor(np.log2(np.maximum(mag, 2.0 ** -126))) - 7)
    return bool(np.all(np.abs(a64 - b64) <= ulp))


def _inputs(wl):
    d = W.make_inputs(wl)
    return {"w1": d["w1"].cuda(), "w2": d["w2"].cuda()}, d["base"].cuda(), d["first_prev"].cuda()


@pytest.mark.parametrize("wl", [W.greedy(32), W.greedy(1), W.TEMPERATURE], ids=lambda w: w.name)
def test_noalloc_matches_allocating_entry_twice(lib, wl):
    d, base, first = _inputs(wl)
    ref_tok = torch.empty(base.shape[:2], dtype=torch.long, device="cuda")
    ref_cor = torch.empty_like(base)
    seed = wl.philox_seed
    assert _call(lib, "dspark_markov_sample_block", d, base, first, wl.temperature, seed, ref_tok, ref_cor) == 0
    for _ in range(2):
        tok = torch.full_like(ref_tok, -1)
        cor = torch.zeros_like(ref_cor)
        assert _call(lib, "dspark_markov_sample_block_noalloc", d, base, first, wl.temperature, seed, tok, cor) == 0
        torch.cuda.synchronize()
        assert torch.equal(tok, ref_tok)
        assert _within_one_ulp(cor, ref_cor)
    assert device_status() == 0


def test_noalloc_allocates_nothing_after_setup(lib):
    d, base, first = _inputs(W.greedy(8))
    tok = torch.empty(base.shape[:2], dtype=torch.long, device="cuda")
    cor = torch.empty_like(base)
    assert _call(lib, "dspark_markov_sample_block_noalloc", d, base, first, 0.0, 0, tok, cor) == 0  # set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        assert _call(lib, "dspark_markov_sample_block_noalloc", d, base, first, 0.0, 0, tok, cor) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_against_oracle_small(lib):
    wl = W.GREEDY.with_(name="noalloc_small", batch=5, vocab=2056, rank=128, proposal_len=6, weight_std=0.3,
                        data_seed=7)
    cpu = W.make_inputs(wl)
    head = VanillaMarkov(cpu["w1"].cuda(), cpu["w2"].cuda())
    base, first = cpu["base"].cuda(), cpu["first_prev"].cuda()
    for temperature, seed in ((0.0, 0), (0.7, 99)):
        tok = torch.empty(5, 6, dtype=torch.long, device="cuda")
        cor = torch.empty_like(base)
        head.sample_block_tokens_noalloc(base, first_prev_token_ids=first, out_tokens=tok, out_logits=cor,
                                         temperature=temperature, seed=seed)
        torch.cuda.synchronize()
        rep = check_sampled_block(tok.cpu().numpy(), f64(cor), f64(cpu["base"]), f64(cpu["w1"]), f64(cpu["w2"]),
                                  cpu["first_prev"].numpy(), "bf16", temperature, seed)
        assert rep.logits.ok, (rep.logits.bad, rep.logits.first_bad, rep.logits.max_abs)
        assert rep.bad == 0, (rep.bad, rep.exact_required, rep.near_ties)


def test_noalloc_rejects_oversize_and_unsupported(lib):
    p = ctypes.c_void_p(16)  # never dereferenced: the checks fail first
    fn = lib.dspark_markov_sample_block_noalloc
    # batch * proposal_len above the scratch's capacity
    assert fn(p, p, 256, 33, 1024, p, p, 64, 0.0, 0, p, ctypes.c_void_p(1 << 40), 1, 1, None) == \
        N.DSPARK_ERR_UNSUPPORTED
    assert 256 * 33 > N.DSPARK_NOALLOC_MAX_KEYS
    # fp32 logits: the tensor-core sampler does not take them, and there is no other path here
    assert fn(p, p, 2, 5, 1024, p, p, 64, 0.0, 0, p, ctypes.c_void_p(1 << 40), 0, 1, None) == \
        N.DSPARK_ERR_UNSUPPORTED
