"""The time-out path of the tensor-core kernels' bounded waits, exercised
without a stalled device.

A pipeline-wait limit of 1 ns, far below the latency of any copy or MMA,
makes the waits give up: the MMA issuer of every CTA sits idle for
microseconds at its start, waiting for the first tiles. Each CTA then raises
its abort flag, lets the copies and MMAs it issued complete (those waits keep
their 2 s limit), releases its tensor memory and exits; the call reports
DSPARK_ERR_DEVICE. With the default limit restored, the same inputs must give
the results they gave before, which shows that no CTA left tensor memory
allocated or a copy in flight and that the context is still usable.
"""
import pytest
import torch

from parity import run_gpu, to_dev
from speculative_draft_mla_b200 import build as dbuild
from speculative_draft_mla_b200 import capi, synth

pytestmark = pytest.mark.gpu
ERR_DEVICE = 7


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dbuild.build()
    return capi.load()


def _same(a, b):
    for k in a:
        if k == "dq":  # fp32 sums of per-tile contributions, order not fixed
            x, y = a[k].float(), b[k].float()
            assert ((x - y).abs() <= torch.maximum(x.abs(), y.abs()) * 2.0 ** -7 + 1e-6).all(), k
        else:
            assert torch.equal(a[k], b[k]), k


def test_wait_limit_runs_out_and_context_recovers():
    wl = synth.WORKLOADS[2]  # bf16 at the page's dims: the tensor-core kernels
    c = synth.make_inputs(wl)
    before = run_gpu(c, wl.S, wl.W)
    d = to_dev(c)
    prev = capi.set_wait_limit_ns(1)
    try:
        o, lse, ws = capi.attn_fwd(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], wl.S, wl.W)
        with pytest.raises(capi.DsparkError) as e:
            capi.get_error(ws)
        assert e.value.status == ERR_DEVICE
        # the backward on the forward's correct outputs; the descriptor built
        # by the forward above is intact (its kernels have no waits)
        o_ok, lse_ok = before["o"].cuda(), before["lse"].cuda()
        capi.attn_bwd(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], o_ok, lse_ok, d["dout"], wl.S,
                      wl.W, workspace=ws, flags=capi.FLAG_REUSE_DESCRIPTOR)
        with pytest.raises(capi.DsparkError) as e:
            capi.get_error(ws)
        assert e.value.status == ERR_DEVICE
    finally:
        assert capi.set_wait_limit_ns(prev) == 1
    torch.cuda.synchronize()
    after = run_gpu(c, wl.S, wl.W)  # raises if the error word is set
    _same(before, after)


def test_wait_limit_loss_cluster_kernel():
    """The loss kernel's CTAs wait for their row copies with the same bounded
    waits; one that gives up stops issuing copies but keeps taking part in
    every cluster barrier (the cluster's CTAs run the same rows), drains its
    copies and reports the device error; the next call is clean."""
    g = torch.Generator(device="cuda").manual_seed(3)
    R, V = 64, 154880
    L = torch.randn(R, V, generator=g, device="cuda").to(torch.bfloat16)
    T = torch.randn(R, V, generator=g, device="cuda").to(torch.bfloat16)
    y = torch.randint(0, V, (R,), generator=g, device="cuda", dtype=torch.int32)
    c = torch.randn(R, generator=g, device="cuda")
    m = torch.ones(R, dtype=torch.uint8, device="cuda")
    out0, g0, gc0, ws = capi.dspark_loss(L, T, y, c, m)
    capi.get_error(ws)
    prev = capi.set_wait_limit_ns(1)
    try:
        capi.dspark_loss(L, T, y, c, m, workspace=ws)
        with pytest.raises(capi.DsparkError) as e:
            capi.get_error(ws)
        assert e.value.status == ERR_DEVICE
    finally:
        assert capi.set_wait_limit_ns(prev) == 1
    out1, g1, gc1, ws = capi.dspark_loss(L, T, y, c, m, workspace=ws)
    capi.get_error(ws)
    assert torch.equal(out0, out1) and torch.equal(g0, g1) and torch.equal(gc0, gc1)
