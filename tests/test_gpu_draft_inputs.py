"""GPU anchor sampler and draft-input builder through the C ABI against the
oracle (bit-exact: integer work) and against the hand-worked golden fixture."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import draft_inputs as odi
from speculative_draft_mla_b200 import build as dbuild
from speculative_draft_mla_b200 import capi

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "draft_inputs_small.json")
KEYS = ("draft_ids", "position_ids", "labels", "prev_ids", "eval_mask")


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dbuild.build()
    return capi.load()


def _mask(rng, B, S, p, last_zero=True):
    lm = (rng.random((B, S)) < p).astype(np.uint8)
    if last_zero and S:
        lm[:, -1] = 0
    return lm


# (B, S, N, loss_mask density, seed): small and ragged cases, fewer candidates
# than N, and the shapes of the benchmark workloads
CASES = [(1, 64, 8, 0.7, 1), (3, 300, 40, 0.9, 2), (2, 20, 30, 0.5, 3), (1, 2, 3, 1.0, 4), (1, 1, 2, 1.0, 5),
         (2, 1000, 1, 1.0, 6), (1, 3000, 2999, 1.0, 7), (2, 2048, 128, 0.9, 8), (2, 8192, 512, 1.0, 9),
         (4, 4096, 512, 0.8, 10), (1, 32768, 1024, 1.0, 11), (2, 5000, 8192, 0.95, 2 ** 63 + 5)]


@pytest.mark.parametrize("case", CASES, ids=["B%d_S%d_N%d" % c[:3] for c in CASES])
def test_sampler_matches_oracle(case):
    B, S, N, p, seed = case
    lm = _mask(np.random.default_rng(seed % 1000), B, S, p)
    an, kp = capi.sample_anchors_gpu(torch.from_numpy(lm).cuda(), N, seed)
    oan, okp = odi.sample_anchors(lm, N, seed)
    assert np.array_equal(an.cpu().numpy(), oan)
    assert np.array_equal(kp.cpu().numpy(), okp)


def test_sampler_edge_masks():
    for lm in (np.zeros((2, 100), np.uint8), np.ones((1, 100), np.uint8)):
        for N in (0, 1, 98, 99, 200):
            an, kp = capi.sample_anchors_gpu(torch.from_numpy(lm).cuda(), N, 3)
            oan, okp = odi.sample_anchors(lm, N, 3)
            assert np.array_equal(an.cpu().numpy(), oan) and np.array_equal(kp.cpu().numpy(), okp), N


def test_builder_golden():
    g = json.load(open(GOLDEN))
    d = lambda k, t: torch.tensor(g[k], dtype=t).cuda()
    out = capi.build_draft_inputs(d("input_ids", torch.int32), d("loss_mask", torch.uint8), d("anchors", torch.int32),
                                  d("keep", torch.uint8), g["mask_id"])
    for k in KEYS:
        assert out[k].cpu().tolist() == g[k], k


@pytest.mark.parametrize("case", CASES[:10], ids=["B%d_S%d_N%d" % c[:3] for c in CASES[:10]])
def test_builder_matches_oracle(case):
    B, S, N, p, seed = case
    rng = np.random.default_rng(100 + seed % 1000)
    lm = _mask(rng, B, S, p, last_zero=False)
    ids = rng.integers(0, 154880, size=(B, S)).astype(np.int32)
    an, kp = odi.sample_anchors(lm, N, seed)
    if N > 2:  # a padding block and anchors outside the page's range
        kp[:, 1] = 0
        an[0, 2] = S - 1
        an[-1, -1] = -3
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = capi.build_draft_inputs(dev(ids), dev(lm), dev(an), dev(kp))
    want = odi.build_draft_inputs(ids, lm, an, kp)
    for k in KEYS:
        assert np.array_equal(out[k].cpu().numpy(), want[k]), k


def test_sampler_then_builder_feed_attention_layout():
    """The sampled anchors and the built positions agree with what the
    attention descriptor expects: kept anchors in [0, S-2], positions A..A+4."""
    lm = _mask(np.random.default_rng(0), 2, 8192, 1.0)
    an, kp = capi.sample_anchors_gpu(torch.from_numpy(lm).cuda(), 512, 42)
    ids = torch.randint(0, 154880, (2, 8192), dtype=torch.int32).cuda()
    out = capi.build_draft_inputs(ids, torch.from_numpy(lm).cuda(), an, kp)
    a = an.cpu().numpy()
    assert (a[kp.cpu().numpy() == 1] <= 8192 - 2).all() and (a >= 0).all()
    pos = out["position_ids"].cpu().numpy().reshape(2, 512, 5)
    assert np.array_equal(pos, a[:, :, None] + np.arange(5)[None, None, :])
