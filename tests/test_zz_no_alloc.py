"""The forward entry point that allocates nothing (dspark_attn_fwd_noalloc).

It serves callers that only get their input and output buffers and may not
allocate device memory themselves (for example a plugin inside another
framework's execution hook, or a loop that cannot afford cudaMalloc's device
synchronisation). Its workspace is a fixed array compiled into the library.
These tests call it through the C ABI and check that it gives the regular
forward's results on consecutive calls of different shapes and dtypes (the
array keeps the previous call's contents), that it rejects problems whose
scratch would not fit, and that it reports a bad anchor through the error
word output.

This file is collected last on purpose: a run that stops at the first failure
has already run every other test.
"""
import ctypes

import pytest
import torch

from parity import assert_close, to_dev
from speculative_draft_mla_b200 import build as dbuild
from speculative_draft_mla_b200 import capi, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dbuild.build()
    return capi.load()


def _cases():
    page = synth.random_case(71, 1, 300, 20, 128, 2, 192, 64, 256, "bf16", keep_frac=0.9)
    page["anchors"][0, 0] = 0
    tiny = synth.make_inputs(synth.WORKLOADS[1])
    return [(page, 300, 128, torch.bfloat16), (tiny, 64, 16, torch.float32)]


def test_matches_regular_forward_on_consecutive_calls():
    cases = _cases()
    err = torch.full((1,), 0xFFFFFFFF, dtype=torch.int64, device="cuda").to(torch.int32)
    results = []
    # two (here three) no-alloc calls in a row, of different sizes and dtypes
    for c, S, W, dt in cases + cases[:1]:
        d = to_dev(c)
        o, lse = capi.attn_fwd_noalloc(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], S, W,
                                       error_word=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        results.append((o.cpu(), lse.cpu()))
    for (c, S, W, dt), (o, lse) in zip(cases + cases[:1], results):
        d = to_dev(c)
        ro, rl, ws = capi.attn_fwd(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], S, W)
        capi.get_error(ws)
        assert_close(o, ro.cpu().double().numpy(), dt, "o")
        assert_close(lse, rl.cpu().double().numpy(), dt, "lse")


def test_rejects_problem_larger_than_scratch():
    lib = capi.load()
    # a 65536-position RoPE table alone needs more than the 16 MiB array
    big = capi.problem(8, 64, 65536, 2048, 128, 192, 64, 256, 10000.0, capi.BF16)
    assert capi.workspace_size(big) > (16 << 20)
    st = lib.dspark_attn_fwd_noalloc(ctypes.byref(big), None, None, None, None, None, None, None, None, None, None)
    assert st == 9  # DSPARK_ERR_UNSUPPORTED, before any device work
    bad = capi.problem(1, 2, 0, 4, 16, 32, 16, 32, 10000.0, capi.F32)  # S = 0
    st = lib.dspark_attn_fwd_noalloc(ctypes.byref(bad), None, None, None, None, None, None, None, None, None, None)
    assert st == 2  # DSPARK_ERR_SHAPE, the regular host check


def test_reports_bad_anchor_in_error_word():
    c = synth.random_case(72, 1, 32, 4, 8, 2, 16, 8, 16, "f32")
    c["anchors"][0, 2] = 31  # S - 1 is not a valid anchor
    d = to_dev(c)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = capi.attn_fwd_noalloc(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], 32, 8,
                                   error_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 1
    assert torch.count_nonzero(o[0, :, 10:15]) == 0 and torch.isneginf(lse[0, :, 10:15]).all()
