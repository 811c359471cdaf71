"""The C-ABI library loads without a GPU, exports every declared symbol, and rejects bad
arguments before it touches a device (no compute call is made here)."""
import ctypes
import glob
import os
import re

import pytest

import linear_attention_linattn_b200 as la
from linear_attention_linattn_b200 import build as labuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        with open(h) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(linattn_[a-z0-9_]+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    if labuild.needs_build():
        labuild.build()
    return la.load_library()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_symbols()
    assert {"linattn_forward", "linattn_decode_step"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(la.SIGNATURES), "binding and header disagree"


def test_state_bytes_closed_form(lib):
    # D*d*4 + D*4 bytes: 16,640 at d = D = 64 (page "Linear Attention > Memory Efficiency")
    assert lib.linattn_state_bytes(64) == 16640
    assert lib.linattn_state_bytes(128) == 66048


def test_status_strings(lib):
    for s in range(5):
        assert lib.linattn_status_string(s)
    assert lib.linattn_version() >= 100


FAKE = 0x10000  # 16-byte aligned, never dereferenced: the checks return first


@pytest.mark.parametrize("args,want", [
    ((0, FAKE, FAKE, FAKE, 1, 1, 8, 64, 0, 1), la.LINATTN_ERR_INVALID_ARG),   # null q
    ((FAKE + 4, FAKE, FAKE, FAKE, 1, 1, 8, 64, 0, 1), la.LINATTN_ERR_INVALID_ARG),  # misaligned
    ((FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 64, 0, 1), la.LINATTN_ERR_INVALID_ARG),  # B = 0
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 64, 0, 1), la.LINATTN_ERR_INVALID_ARG),  # n = 0
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 2, 1), la.LINATTN_ERR_INVALID_ARG),  # causal = 2
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 0, 7), la.LINATTN_ERR_INVALID_ARG),  # dtype
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 96, 0, 1), la.LINATTN_ERR_UNSUPPORTED),  # d = 96
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 1 << 31, 64, 0, 1), la.LINATTN_ERR_INVALID_ARG),  # n too big
])
def test_forward_argument_checks(lib, args, want):
    assert lib.linattn_forward(*args, None) == want


def test_decode_and_state_argument_checks(lib):
    assert lib.linattn_decode_step(0, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 64, None) == \
        la.LINATTN_ERR_INVALID_ARG
    assert lib.linattn_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 32, None) == \
        la.LINATTN_ERR_UNSUPPORTED
    assert lib.linattn_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, 1, 64, None) == \
        la.LINATTN_ERR_INVALID_ARG
    assert lib.linattn_forward_state(FAKE, FAKE, FAKE, 0, 1, 1, 8, 64, 1, None) == \
        la.LINATTN_ERR_INVALID_ARG
    assert lib.linattn_forward_ex(FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 1, 1, -64, None) == \
        la.LINATTN_ERR_INVALID_ARG
    # segments are whole 128-token chunks of the causal kernel
    assert lib.linattn_forward_ex(FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 1, 1, 64, None) == \
        la.LINATTN_ERR_INVALID_ARG


def test_backward_init_and_sum_argument_checks(lib):
    bad = la.LINATTN_ERR_INVALID_ARG
    # backward: null dq, misaligned dout, causal out of range, d unsupported
    assert lib.linattn_backward(FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, 1, 1, 8, 64, 1, 0,
                                None) == bad
    assert lib.linattn_backward(FAKE, FAKE, FAKE, FAKE + 8, FAKE, FAKE, FAKE, 1, 1, 8, 64, 1, 0,
                                None) == bad
    assert lib.linattn_backward(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 2, 0,
                                None) == bad
    assert lib.linattn_backward(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 96, 1, 0,
                                None) == la.LINATTN_ERR_UNSUPPORTED
    # backward segments: whole 64-token chunks, not negative
    for seg in (-64, 100):
        assert lib.linattn_backward_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 1,
                                       1, seg, None) == bad
    # block aggregates: the buffer is required; sizes for unsupported shapes are 0
    assert lib.linattn_forward_state_keep(FAKE, FAKE, FAKE, FAKE, 0, 1, 1, 8, 64, 1,
                                          None) == bad
    assert lib.linattn_forward_init_from(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8, 1, 1, 8,
                                         64, 1, 1, None) == bad
    assert lib.linattn_block_aggregates_bytes(1, 1, 8, 96, 1) == 0
    assert lib.linattn_block_aggregates_bytes(1, 1, 0, 64, 1) == 0
    # fp32: one (d*d + d)-float state per 64-token chunk
    assert lib.linattn_block_aggregates_bytes(2, 3, 130, 64, 0) == 2 * 3 * 3 * (64 * 64 + 64) * 4
    # forward from a state: the state pointers are required
    assert lib.linattn_forward_init(FAKE, FAKE, FAKE, FAKE, 0, FAKE, 1, 1, 8, 64, 1, 1,
                                    None) == bad
    # state sums: negative count, skip below -1, unsupported d
    assert lib.linattn_sum_states(FAKE, -1, -1, 1, 1, 64, FAKE, FAKE, None) == bad
    assert lib.linattn_sum_states(FAKE, 2, -2, 1, 1, 64, FAKE, FAKE, None) == bad
    assert lib.linattn_sum_states(FAKE, 2, -1, 1, 1, 80, FAKE, FAKE, None) == \
        la.LINATTN_ERR_UNSUPPORTED


def test_forward_host_argument_checks(lib):
    """Host buffers need no alignment; null pointers and bad shapes are rejected before any
    device call."""
    bad = la.LINATTN_ERR_INVALID_ARG
    assert lib.linattn_forward_host(0, FAKE, FAKE, FAKE, 1, 1, 8, 64, 1, 1, None) == bad
    assert lib.linattn_forward_host(FAKE, FAKE, FAKE, 0, 1, 1, 8, 64, 1, 1, None) == bad
    assert lib.linattn_forward_host(FAKE + 2, FAKE, FAKE, FAKE, 1, 0, 8, 64, 1, 1, None) == bad
    assert lib.linattn_forward_host(FAKE + 2, FAKE, FAKE, FAKE, 1, 1, 8, 64, 3, 1, None) == bad
    assert lib.linattn_forward_host(FAKE + 2, FAKE, FAKE, FAKE, 1, 1, 8, 96, 1, 1, None) == \
        la.LINATTN_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError):
        la.load_library(str(tmp_path / "nope.so"))
