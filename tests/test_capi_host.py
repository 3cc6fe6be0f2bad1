"""Host-side tests of the C ABI (no GPU needed, no kernel launched).

- the library loads and exports every function declared in include/*.h;
- argument validation returns the documented status before any CUDA call;
- the host anchor sampler follows the page's §2 rule (checked against the
  oracle's candidate enumeration) and the §3 padding convention.
"""
import ctypes
import glob
import os
import re

import numpy as np
import pytest
import torch

from speculative_draft_mla_b200 import build as dbuild
from speculative_draft_mla_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dbuild.build()
    return capi.load()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        names += re.findall(r"DSPARK_API\s+[\w\s\*]+?\b(dspark_\w+)\s*\(", open(h).read())
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(capi.EXPORTS) <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    out = os.popen("nm -D --defined-only %s" % capi.LIB_PATH).read()
    for n in names:
        assert re.search(r" T %s$" % n, out, re.M), n


def test_built_for_sm100a(lib):
    # the build flags name the one target architecture
    assert dbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def P(**kw):
    d = dict(B=1, n_h=2, S=64, N=4, W=16, d_c=32, d_r=16, d_v=32, rope_base=10000.0, dtype=capi.F32)
    d.update(kw)
    return capi.problem(**d)


def test_workspace_size(lib):
    assert capi.workspace_size(P()) > 0
    assert capi.workspace_size(P(n_h=0)) == 0
    assert capi.workspace_size(P(d_r=3)) == 0
    assert capi.workspace_size(P(dtype=7)) == 0
    assert capi.workspace_size(P(W=5000)) == 0
    big = P(B=4, S=4096, N=512, n_h=64, d_c=192, d_r=64, d_v=256, W=128, dtype=capi.BF16)
    assert capi.workspace_size(big) > capi.workspace_size(P())
    assert capi.workspace_size(big) % 256 == 0


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails validation first


def fwd(lib, prob, ws_bytes=1 << 20, q=FAKE, ws=ctypes.c_void_p(0x100000), anchors=FAKE):
    return lib.dspark_attn_fwd(ctypes.byref(prob), q, FAKE, FAKE, FAKE, anchors, FAKE, FAKE, FAKE, ws, ws_bytes, 0,
                               None)


def test_validation_statuses(lib):
    assert lib.dspark_attn_fwd(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, None) == 1
    assert fwd(lib, P(dtype=5)) == 3
    assert fwd(lib, P(S=0)) == 2
    assert fwd(lib, P(d_r=5)) == 2
    assert fwd(lib, P(rope_base=-1.0)) == 2
    assert fwd(lib, P(d_c=200, d_r=64)) == 9
    assert fwd(lib, P(d_v=512)) == 9
    assert fwd(lib, P(N=9000)) == 9
    assert fwd(lib, P(), ws_bytes=16) == 5
    assert fwd(lib, P(), ws=None) == 5
    assert fwd(lib, P(), ws=ctypes.c_void_p(0x100010)) == 5  # not 256-aligned
    need = capi.workspace_size(P())
    assert fwd(lib, P(), ws_bytes=need, q=None) == 1
    assert fwd(lib, P(), ws_bytes=need, q=ctypes.c_void_p(0x1008)) == 8
    assert fwd(lib, P(), ws_bytes=need, anchors=None) == 1
    prob = P()
    assert lib.dspark_build_descriptor(ctypes.byref(prob), None, None, ctypes.c_void_p(0x100000), need, None) == 1
    assert lib.dspark_attn_bwd(ctypes.byref(P(W=0)), *([FAKE] * 14), 0, 0, None) == 2
    assert lib.dspark_get_error(None, None) == 5
    for s in range(10):
        assert len(capi.status_string(s)) > 0


def test_sampler_follows_page_rule(lib, oracle_mod):
    g = torch.Generator().manual_seed(5)
    for S, N, pm in [(64, 8, 0.7), (300, 40, 0.9), (20, 30, 0.5), (2, 3, 1.0), (1, 2, 1.0)]:
        lm = (torch.rand(3, S, generator=g) < pm).to(torch.uint8)
        an, kp = capi.sample_anchors(lm, N, seed=123)
        for b in range(3):
            cand = oracle_mod.anchor_candidates(lm[b].numpy())
            take = min(N, len(cand))
            assert kp[b, :take].tolist() == [1] * take and kp[b, take:].tolist() == [0] * (N - take)
            drawn = an[b, :take].tolist()
            assert len(set(drawn)) == take and set(drawn) <= set(cand.tolist())
            assert an[b, take:].tolist() == [0] * (N - take)
        an2, kp2 = capi.sample_anchors(lm, N, seed=123)
        assert torch.equal(an, an2) and torch.equal(kp, kp2)


def test_sampler_uniform(lib):
    """Each candidate is drawn with probability N / #candidates."""
    S, N, trials = 12, 3, 4000
    lm = torch.ones(1, S, dtype=torch.uint8)
    counts = np.zeros(S)
    for t in range(trials):
        an, _ = capi.sample_anchors(lm, N, seed=t)
        counts[an[0].numpy()] += 1
    cand = S - 2  # A in [0, S-3] once loss_mask[S-1] is read as 0
    assert counts[cand:].sum() == 0
    expect = trials * N / cand
    chi2 = ((counts[:cand] - expect) ** 2 / expect).sum()
    assert chi2 < 30.0, chi2  # 9 degrees of freedom; p ~ 5e-4 at 30


def test_wait_limit_setter(lib):
    """The pipeline-wait limit is process-wide; 0 and values above the 2 s
    default restore the default; each call returns the limit it replaced."""
    default = 2_000_000_000
    prev = capi.set_wait_limit_ns(0)
    assert prev == default
    assert capi.set_wait_limit_ns(1000) == default
    assert capi.set_wait_limit_ns(5 * default) == 1000
    assert capi.set_wait_limit_ns(0) == default
    assert capi.set_wait_limit_ns(0) == default


def test_draft_input_validation(lib):
    """Host checks of the GPU sampler and builder return before any device work."""
    vp = ctypes.c_void_p
    odd = vp(0x1001)  # never dereferenced: every call below fails its host checks
    ok = vp(0x1000)
    S_, N_ = 100, 10
    assert lib.dspark_sample_anchors_gpu(ok, -1, S_, N_, 1, ok, ok, None) == 2
    assert lib.dspark_sample_anchors_gpu(ok, 1, 0, N_, 1, ok, ok, None) == 2
    assert lib.dspark_sample_anchors_gpu(ok, 1, S_, 9000, 1, ok, ok, None) == 9
    assert lib.dspark_sample_anchors_gpu(None, 1, S_, N_, 1, ok, ok, None) == 1
    assert lib.dspark_sample_anchors_gpu(ok, 1, S_, N_, 1, odd, ok, None) == 8
    assert lib.dspark_sample_anchors_gpu(None, 0, S_, N_, 1, None, None, None) == 0  # nothing to do
    args = [ok, ok, 1, S_, N_, ok, ok, 154821, ok, ok, ok, ok, ok, None]
    assert lib.dspark_build_draft_inputs(*args[:2], -1, *args[3:]) == 2
    bad = list(args)
    bad[8] = None
    assert lib.dspark_build_draft_inputs(*bad) == 1
    bad = list(args)
    bad[10] = odd
    assert lib.dspark_build_draft_inputs(*bad) == 8
    assert lib.dspark_build_draft_inputs(*args[:4], 0, *args[5:]) == 0
