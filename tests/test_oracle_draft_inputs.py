"""Pins of the draft-input oracle (anchor sampling and the draft block's
inputs, labels and eval_mask) against what the page and the generator's
published definition fix; no GPU."""
import json
import os

import numpy as np

from oracle import draft_inputs as di

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "draft_inputs_small.json")


def test_splitmix64_published_outputs():
    # the first outputs of the SplitMix64 reference generator started from
    # state 0 (Steele, Lea and Flood, OOPSLA 2014; the public reference code)
    assert [di.splitmix64_output(0, k) for k in range(3)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_candidates_page_rule():
    g = json.load(open(GOLDEN))
    for row, want in zip(g["loss_mask"], g["candidates"]):
        assert di.candidates(row) == want
    assert di.candidates([1, 1]) == []           # loss_mask[S-1] is read as 0
    assert di.candidates([1]) == []
    assert di.candidates([0] * 10) == []
    assert di.candidates([1, 1, 1]) == [0]       # A = S-2 needs loss_mask[S-1]


def test_builder_golden():
    g = json.load(open(GOLDEN))
    out = di.build_draft_inputs(np.array(g["input_ids"]), np.array(g["loss_mask"]), np.array(g["anchors"]),
                                np.array(g["keep"]), g["mask_id"])
    for k in ("draft_ids", "position_ids", "labels", "prev_ids", "eval_mask"):
        assert out[k].tolist() == g[k], k


def test_sampler_invariants():
    rng = np.random.default_rng(3)
    for S, N, p in [(64, 8, 0.7), (300, 40, 0.9), (20, 30, 0.5), (2, 3, 1.0), (1, 2, 1.0), (50, 0, 1.0)]:
        lm = (rng.random((3, S)) < p).astype(np.uint8)
        an, kp = di.sample_anchors(lm, N, seed=11)
        for b in range(3):
            cand = di.candidates(lm[b])
            take = min(N, len(cand))
            assert kp[b].tolist() == [1] * take + [0] * (N - take)
            got = an[b, :take].tolist()
            assert got == sorted(set(got)) and set(got) <= set(cand)   # ascending, distinct, valid
            assert an[b, take:].tolist() == [0] * (N - take)
        assert np.array_equal(di.sample_anchors(lm, N, seed=11)[0], an)


def test_sampler_uniform():
    """Each candidate is chosen with probability N / #candidates, and pairs of
    candidates with probability N (N - 1) / (C (C - 1)) (a uniform draw
    without replacement), over seeds."""
    S, N, trials = 12, 3, 3000
    lm = np.ones((1, S), np.uint8)
    C = S - 2
    counts = np.zeros(C)
    pair01 = 0
    for t in range(trials):
        an, _ = di.sample_anchors(lm, N, seed=1000 + 7 * t)
        counts[an[0]] += 1
        pair01 += int(0 in an[0] and 1 in an[0])
    expect = trials * N / C
    chi2 = ((counts - expect) ** 2 / expect).sum()
    assert chi2 < 30.0, chi2  # 9 degrees of freedom
    p_pair = N * (N - 1) / (C * (C - 1))
    assert abs(pair01 / trials - p_pair) < 4 * np.sqrt(p_pair * (1 - p_pair) / trials)


def test_sampler_takes_all_when_few():
    lm = np.array([[1, 1, 0, 1, 1, 1, 0, 1]], np.uint8)
    an, kp = di.sample_anchors(lm, 6, seed=5)
    assert an[0].tolist() == [0, 3, 4, 0, 0, 0] and kp[0].tolist() == [1, 1, 1, 0, 0, 0]
