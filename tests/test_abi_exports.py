"""The C-ABI library loads and exports every symbol include/dspark_markov.h
declares; host-side argument checks run without a GPU (no kernel launches)."""
import ctypes
import os
import re

import pytest

from rank_markov_draft_vanillamarkov_b200 import _native as N
from rank_markov_draft_vanillamarkov_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dspark_markov.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dspark_markov_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    B.build()  # no-op when up to date; nvcc cross-compiles without a GPU
    return N.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
        assert n in N.SIGNATURES, f"binding lacks a signature for {n}"


def test_header_constants_match_binding():
    text = open(HEADER).read()
    for name in ["DSPARK_OK", "DSPARK_ERR_INVALID_ARG", "DSPARK_ERR_UNSUPPORTED", "DSPARK_ERR_CUDA",
                 "DSPARK_STATUS_TOKEN_RANGE", "DSPARK_STATUS_TIMEOUT", "DSPARK_DTYPE_FP32", "DSPARK_DTYPE_BF16",
                 "DSPARK_ALGO_AUTO", "DSPARK_ALGO_GENERIC", "DSPARK_ALGO_TENSOR_CORE",
                 "DSPARK_DEBUG_SKIP_BARRIER_ARRIVAL", "DSPARK_NOALLOC_MAX_KEYS", "DSPARK_VARIANT_BWD_RESIDENT_W1",
                 "DSPARK_VARIANT_SAMPLE_ROWS", "DSPARK_VARIANT_APPLY_WIDE", "DSPARK_DEBUG_APPLY_WIDE",
                 "DSPARK_DEBUG_SAMPLE_ROWS", "DSPARK_DEBUG_SAMPLE_TILE"]:
        m = re.search(rf"#define {name} (\d+)", text)
        assert m, name
        assert int(m.group(1)) == getattr(N, name), name


def test_argument_errors_are_caught_on_the_host(lib):
    p = ctypes.c_void_p(16)  # never dereferenced: every call below fails its checks first
    ap = lib.dspark_markov_apply_block_logits
    assert ap(p, p, p, 4, 128, p, p, 0, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG  # rank 0
    assert ap(p, p, p, 4, 128, p, p, -3, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert ap(p, p, p, -1, 128, p, p, 16, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert ap(p, p, p, 4, 0, p, p, 16, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert ap(p, p, p, 4, 128, p, p, 16, 7, 1, None) == N.DSPARK_ERR_INVALID_ARG  # bad dtype
    assert ap(None, p, p, 4, 128, p, p, 16, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert ap(None, None, None, 0, 128, None, None, 16, 1, 1, None) == N.DSPARK_OK  # empty: nothing enqueued
    sp = lib.dspark_markov_sample_block
    nan = float("nan")
    assert sp(p, p, 2, 5, 128, p, p, 16, nan, 0, p, p, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert sp(p, p, 2, 5, 128, p, p, 0, 0.0, 0, p, p, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert sp(None, None, 2, 0, 128, None, None, 16, 0.0, 0, None, None, 1, 1, None) == N.DSPARK_OK
    assert sp(None, None, 0, 5, 128, None, None, 16, 0.0, 0, None, None, 1, 1, None) == N.DSPARK_OK
    # corrected logits overlapping the base logits are refused
    q = ctypes.c_void_p(4096)
    assert sp(q, p, 2, 5, 128, p, p, 16, 0.0, 0, p, q, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    # the no-allocation sampler: same argument checks, and its scratch bound
    na = lib.dspark_markov_sample_block_noalloc
    assert na(p, p, 2, 5, 128, p, p, 16, nan, 0, p, p, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert na(None, None, 2, 0, 128, None, None, 16, 0.0, 0, None, None, 1, 1, None) == N.DSPARK_OK
    assert na(q, p, 2, 5, 128, p, p, 16, 0.0, 0, p, q, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert na(p, p, 256, 33, 128, p, p, 64, 0.0, 0, p, ctypes.c_void_p(1 << 40), 1, 1, None) == \
        N.DSPARK_ERR_UNSUPPORTED


def test_transition_argument_checks(lib):
    p = ctypes.c_void_p(16)  # never dereferenced
    tr = lib.dspark_markov_transition_logits
    assert tr(None, 0, 128, None, None, 16, None, None, 1, None) == N.DSPARK_OK  # empty: nothing enqueued
    assert tr(p, 4, 128, p, p, 0, p, None, 1, None) == N.DSPARK_ERR_INVALID_ARG  # rank 0
    assert tr(p, 4, 0, p, p, 16, p, None, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert tr(p, -1, 128, p, p, 16, p, None, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert tr(p, 4, 128, p, p, 16, p, None, 5, None) == N.DSPARK_ERR_INVALID_ARG  # bad dtype
    assert tr(p, 4, 128, p, p, 16, None, p, 1, None) == N.DSPARK_ERR_INVALID_ARG  # no output


def test_backward_argument_checks(lib):
    p = ctypes.c_void_p(16)  # never dereferenced
    bw = lib.dspark_markov_apply_block_logits_backward
    assert bw(p, p, 4, 128, p, p, 16, None, None, 0, 1, 1, None) == N.DSPARK_OK  # nothing wanted
    assert bw(p, p, 4, 128, p, p, 0, p, p, 0, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG  # rank 0
    assert bw(p, p, -1, 128, p, p, 16, p, p, 0, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG
    assert bw(p, p, 4, 128, p, p, 16, p, p, 0, 9, 1, None) == N.DSPARK_ERR_INVALID_ARG  # bad dtype
    assert bw(None, p, 4, 128, p, p, 16, p, p, 0, 1, 1, None) == N.DSPARK_ERR_INVALID_ARG


def test_host_utilities(lib):
    assert lib.dspark_markov_strerror(0) == b"ok"
    assert lib.dspark_markov_strerror(N.DSPARK_ERR_UNSUPPORTED).startswith(b"unsupported")
    prev = lib.dspark_markov_set_algo(N.DSPARK_ALGO_GENERIC)
    assert lib.dspark_markov_set_algo(prev) == N.DSPARK_ALGO_GENERIC
    assert lib.dspark_markov_set_algo(99) == -1
    assert lib.dspark_markov_launch_count() >= 0
    assert lib.dspark_markov_set_debug(0, 0) == N.DSPARK_OK


def test_missing_library_fails_loudly(tmp_path):
    saved = N._lib
    N._lib = None
    try:
        with pytest.raises(RuntimeError, match="not built"):
            N.load(str(tmp_path / "nope.so"))
    finally:
        N._lib = saved
