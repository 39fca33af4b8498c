"""Parity of the CUDA teacher-forced apply against the fp64 oracle (B200).

Every comparison is element by element against ``oracle.exact_block_logits``
under the tolerance rule of ``oracle.checks`` (bf16: one round-to-nearest-even
of a sum within the fp32 accumulation bound of the exact sum, and within
2e-2 + ulp/2 of it; fp32: 1e-4).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import markov as om
from oracle.checks import check_logits
from rank_markov_draft_vanillamarkov_b200 import (VanillaMarkov, device_status, last_algo, last_variant, set_algo,
                                                 set_debug)
from rank_markov_draft_vanillamarkov_b200 import _native as N
from rank_markov_draft_vanillamarkov_b200 import workloads as W
from rank_markov_draft_vanillamarkov_b200.build import build

from _helpers import dtype_name, f64

pytestmark = pytest.mark.gpu

TC, GEN = N.DSPARK_ALGO_TENSOR_CORE, N.DSPARK_ALGO_GENERIC


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    assert torch.cuda.is_available()
    N.load()
    yield
    set_algo(N.DSPARK_ALGO_AUTO)


_VARIANT = {}


@pytest.fixture(params=["narrow", "wide"])
def kernel(request):
    """The tensor-core apply with 128-id units (the default) or, on request,
    256-id units."""
    set_debug(N.DSPARK_DEBUG_APPLY_WIDE if request.param == "wide" else 0, 0)
    yield request.param
    set_debug(0, 0)


def _run(d, algo, base=None, ids=None, out=None):
    set_algo(algo)
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    base = (d["base"] if base is None else base).cuda()
    ids = (d["prev_ids"] if ids is None else ids).cuda()
    got = head.apply_block_logits(base, token_ids=ids, out=out)
    _VARIANT["last"] = last_variant()
    torch.cuda.synchronize()
    used = last_algo()
    st = device_status()
    return got, used, st


def _wide_ran() -> bool:
    return bool(_VARIANT["last"] & N.DSPARK_VARIANT_APPLY_WIDE)


def _operands(d, base=None, ids=None, rows=None):
    base = d["base"] if base is None else base
    ids = d["prev_ids"] if ids is None else ids
    v = base.shape[-1]
    b = f64(base).reshape(-1, v)
    i = ids.reshape(-1).numpy()
    if rows is not None:
        b, i = b[rows], i[rows]
    return b, i


def _exact(d, base=None, ids=None, rows=None):
    b, i = _operands(d, base, ids, rows)
    return om.exact_block_logits(b, f64(d["w1"]), f64(d["w2"]), i)


def _acc(d, base=None, ids=None, rows=None):
    """fp32 accumulation error bound of every element (oracle.checks)."""
    b, i = _operands(d, base, ids, rows)
    return oracle.accumulation_bound(b, f64(d["w1"]), f64(d["w2"]), i)


def _assert_ok(rep, what):
    assert rep.ok, f"{what}: {rep.bad} of {rep.n} outside tolerance, first at {rep.first_bad}, " \
                   f"max_abs {rep.max_abs:.3g}, max_ulps {rep.max_ulps_vs_rne:.2f}"


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
@pytest.mark.parametrize("wl", W.small_variants(), ids=lambda w: w.name)
def test_small_variants(wl, algo, kernel):
    d = W.make_inputs(wl)
    got, used, st = _run(d, algo)
    assert used == (2 if algo == TC else 1)
    assert st == 0
    if algo == TC:
        assert _wide_ran() == (kernel == "wide")
    exact = _exact(d)
    _assert_ok(check_logits(f64(got).reshape(exact.shape), exact, "bf16", _acc(d)), wl.name)


def test_tiny_fp32_workload():
    """The fp32 tiny workload: logits within 1e-4 of the exact sum."""
    d = W.make_inputs(W.TINY_FP32)
    got, used, st = _run(d, N.DSPARK_ALGO_AUTO)
    assert used == 1 and st == 0 and got.dtype == torch.float32
    exact = _exact(d)
    _assert_ok(check_logits(f64(got).reshape(exact.shape), exact, "fp32"), "tiny fp32")


@pytest.mark.parametrize("ldt,wdt", [(torch.float32, torch.bfloat16), (torch.bfloat16, torch.float32)])
def test_mixed_dtypes(ldt, wdt):
    wl = W.small_variants()[0]
    d = W.make_inputs(wl)
    d = dict(d, base=d["base"].to(ldt), w1=d["w1"].to(wdt), w2=d["w2"].to(wdt))
    got, used, st = _run(d, N.DSPARK_ALGO_AUTO)
    # fp32 logits with bf16 weights run on the tensor-core kernel, the other pairs on the generic one
    assert used == (2 if (ldt == torch.float32 and wdt == torch.bfloat16) else 1) and st == 0
    exact = _exact(d)
    _assert_ok(check_logits(f64(got).reshape(exact.shape), exact, dtype_name(ldt), _acc(d)), "mixed")


_NON_RESIDENT = W.APPLY_320.with_(name="apply_small_r1100_v1000_k64", vocab=1000, rank=64, batch=4, num_blocks=55,
                                  weight_std=0.3, data_seed=14)  # 9 row tiles: per-unit A


@pytest.mark.parametrize("wl", W.small_variants() + [_NON_RESIDENT], ids=lambda w: w.name)
def test_fp32_logits_tensor_core(wl):
    """fp32 logits with a bf16 head (the stage's compute_logits returns fp32)
    on the tensor-core kernel: ragged tiles, resident and per-unit A, in place."""
    d = W.make_inputs(wl)
    d = dict(d, base=d["base"].float())
    got, used, st = _run(d, TC)
    assert used == 2 and st == 0 and got.dtype == torch.float32
    exact = _exact(d)
    _assert_ok(check_logits(f64(got).reshape(exact.shape), exact, "fp32", _acc(d)), "fp32 logits")
    base = d["base"].clone().cuda()
    same, used, st = _run(d, TC, base=base, out=base)
    assert same.data_ptr() == base.data_ptr() and torch.equal(same.cpu(), got.cpu())


def test_apply_320_fp32_logits_full_size():
    d = W.make_inputs(W.APPLY_320_FP32)
    got, used, st = _run(d, N.DSPARK_ALGO_AUTO)
    assert used == 2 and st == 0
    exact = _exact(d)
    _assert_ok(check_logits(f64(got).reshape(exact.shape), exact, "fp32", _acc(d)), "apply 320 fp32 logits")


def test_apply_320_full_size(kernel):
    """320 rows x 129280 ids x rank 128, every element against the oracle."""
    d = W.make_inputs(W.APPLY_320)
    got, used, st = _run(d, N.DSPARK_ALGO_AUTO)
    assert used == 2 and st == 0 and _wide_ran() == (kernel == "wide")
    exact = _exact(d)
    _assert_ok(check_logits(f64(got).reshape(exact.shape), exact, "bf16", _acc(d)), "apply 320")


def _check_all_rows(d, got, what, base=None, chunk=128):
    """Every row of a large output against the oracle, 128 rows at a time so
    that the fp64 operands stay small. Returns the largest |exact| seen."""
    base = d["base"] if base is None else base
    v = base.shape[-1]
    bv, iv, gv = base.reshape(-1, v), d["prev_ids"].reshape(-1), got.view(-1, v)
    w1, w2 = f64(d["w1"]), f64(d["w2"])
    peak = 0.0
    for r0 in range(0, bv.shape[0], chunk):
        r1 = min(bv.shape[0], r0 + chunk)
        b, i = f64(bv[r0:r1]), iv[r0:r1].numpy()
        exact = om.exact_block_logits(b, w1, w2, i)
        rep = check_logits(f64(gv[r0:r1]), exact, "bf16", oracle.accumulation_bound(b, w1, w2, i))
        _assert_ok(rep, f"{what}, rows {r0}..{r1 - 1}")
        peak = max(peak, float(np.abs(exact).max()))
    return peak


def test_apply_2560_every_row(kernel):
    """2560 rows x 129280 ids x rank 256, 20% padding blocks (computed like
    any other): every element against the oracle."""
    wl = W.APPLY_2560
    d = W.make_inputs(wl)
    assert d["pad_mask"].float().mean() > 0.1
    got, used, st = _run(d, N.DSPARK_ALGO_AUTO)
    assert used == 2 and st == 0 and _wide_ran() == (kernel == "wide")
    _check_all_rows(d, got, "apply 2560")


@pytest.mark.parametrize("wl", [W.APPLY_320, W.APPLY_2560], ids=lambda w: w.name)
def test_bias_probe_zero_logits(wl, kernel):
    """U = 0: the output is the bias alone, so a kernel that dropped or
    garbled the bias cannot hide under the logits tolerance. Every element is
    checked with the one-rounding rule, and the largest bias must be well
    above the tolerance for the probe to have power."""
    d = W.make_inputs(wl)
    zero = torch.zeros_like(d["base"])
    got, used, st = _run(d, N.DSPARK_ALGO_AUTO, base=zero)
    assert used == 2 and st == 0
    assert _check_all_rows(d, got, "bias probe", base=zero) > 1e-2


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_strong_bias_full_vocab(algo, kernel):
    """Weights ~N(0, 0.3): bias std about 1, comparable to the logits."""
    wl = W.APPLY_320.with_(weight_std=0.3, batch=1, num_blocks=40, data_seed=5)
    d = W.make_inputs(wl)
    got, used, st = _run(d, algo)
    assert st == 0
    exact = _exact(d)
    _assert_ok(check_logits(f64(got).reshape(exact.shape), exact, "bf16", _acc(d)), "strong bias")


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_zero_w2_is_bit_exact_passthrough(algo):
    wl = W.small_variants()[1]
    d = W.make_inputs(wl)
    d["w2"] = torch.zeros_like(d["w2"])
    got, used, st = _run(d, algo)
    assert torch.equal(got.cpu(), d["base"])


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_in_place(algo):
    wl = W.small_variants()[1]
    d = W.make_inputs(wl)
    base = d["base"].cuda()
    set_algo(algo)
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    ref = head.apply_block_logits(base.clone(), token_ids=d["prev_ids"].cuda())
    out = head.apply_block_logits(base, token_ids=d["prev_ids"].cuda(), out=base)
    torch.cuda.synchronize()
    assert out.data_ptr() == base.data_ptr()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_canaries_untouched(algo):
    """The kernel writes exactly rows x vocab elements: guard bands on both
    sides of the output keep their pattern."""
    wl = W.small_variants()[0]
    d = W.make_inputs(wl)
    n = wl.rows * wl.vocab
    guard = 4096
    buf = torch.full((n + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[guard:guard + n].view(d["base"].shape)
    _run(d, algo, out=out)
    assert (buf[:guard] == 7.0).all() and (buf[guard + n:] == 7.0).all()


@pytest.mark.parametrize("algo", [TC, GEN], ids=["tc", "generic"])
def test_out_of_range_ids_report_status(algo):
    """An id outside [0, V) sets the TOKEN_RANGE status bit (no trap); the
    other rows are still correct."""
    wl = W.small_variants()[0]
    d = W.make_inputs(wl)
    ids = d["prev_ids"].clone()
    flat = ids.view(-1)
    flat[3] = wl.vocab
    flat[7] = -5
    got, used, st = _run(d, algo, ids=ids)
    assert st & N.DSPARK_STATUS_TOKEN_RANGE
    keep = np.setdiff1d(np.arange(wl.rows), [3, 7])
    fixed = ids.clamp(0, wl.vocab - 1)
    exact = _exact(d, ids=fixed, rows=keep)
    _assert_ok(check_logits(f64(got.view(-1, wl.vocab)[torch.from_numpy(keep).cuda()]), exact, "bf16",
                            _acc(d, ids=fixed, rows=keep)), "rest")
    assert device_status() == 0  # cleared by the previous read


def test_empty_inputs_return_the_same_object():
    d = W.make_inputs(W.small_variants()[0])
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    e1 = torch.zeros(2, 0, 1000, dtype=torch.bfloat16, device="cuda")
    assert head.apply_block_logits(e1, token_ids=torch.zeros(2, 0, dtype=torch.long, device="cuda")) is e1
    e2 = torch.zeros(0, 3, 1000, dtype=torch.bfloat16, device="cuda")
    assert head.apply_block_logits(e2, token_ids=torch.zeros(0, 3, dtype=torch.long, device="cuda")) is e2


def test_hidden_states_are_ignored():
    wl = W.small_variants()[0]
    d = W.make_inputs(wl)
    head = VanillaMarkov(d["w1"].cuda(), d["w2"].cuda())
    base, ids = d["base"].cuda(), d["prev_ids"].cuda()
    a = head.apply_block_logits(base, token_ids=ids)
    hid = torch.randn(*ids.shape, 64, device="cuda")
    b = head.apply_block_logits(base, token_ids=ids, hidden_states=hid)
    assert torch.equal(a, b)


def test_tc_and_generic_agree():
    wl = W.small_variants()[2]
    d = W.make_inputs(wl)
    a, ua, _ = _run(d, TC)
    b, ub, _ = _run(d, GEN)
    assert (ua, ub) == (2, 1)
    diff = np.abs(f64(a) - f64(b)).reshape(-1, wl.vocab)
    # both are one rounding of an fp32 sum: one ulp apart at most, plus the
    # accumulation error bound where U and the bias cancel
    ulp = oracle.ulp_bfloat16(f64(a)).reshape(diff.shape)
    assert (diff <= ulp + 2 * _acc(d)).all()
    assert (diff == 0).mean() > 0.99


def test_deterministic_rerun():
    d = W.make_inputs(W.small_variants()[1])
    a, _, _ = _run(d, TC)
    b, _, _ = _run(d, TC)
    assert torch.equal(a, b)
