"""Pins from numbers the DSpark design page prints (tests/golden/page_facts.json).

The page gives no worked attention example, but its parameter and KV-cache
figures fix the head dimensions the workloads use, and its §2/§3 text fixes the
anchor rule and the window size. These tests recompute the printed figures.
"""
import json
import os

import numpy as np

from speculative_draft_mla_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))
FACTS = json.load(open(os.path.join(HERE, "golden", "page_facts.json")))


def test_mla_parameter_count_fixes_head_dims():
    f = FACTS
    d, nh, ql, kvl, dc, dr, dv = f["d"], f["n_h"], f["q_lora"], f["kv_lora"], f["d_c"], f["d_r"], f["d_v"]
    mla = d * ql + ql * nh * (dc + dr) + d * (kvl + dr) + kvl * nh * (dc + dv) + nh * dv * d
    assert round(mla / 1e6) == f["mla_params_per_layer_M"]
    # a single shared k^R per position: a per-head rope key would not match
    per_head_rope = d * ql + ql * nh * (dc + dr) + d * (kvl + nh * dr) + kvl * nh * (dc + dv) + nh * dv * d
    assert round(per_head_rope / 1e6) != f["mla_params_per_layer_M"]
    assert round(f["hidden_states_width"] * d / 1e6) == f["main_proj_params_M"]
    assert round(3 * d * f["ffn"] / 1e6) == f["swiglu_params_per_layer_M"]
    assert round(2 * f["vocab"] * f["markov_rank"] / 1e6) == f["markov_params_M"]


def test_kv_cache_figures():
    f = FACTS
    assert f["kv_lora"] + f["d_r"] == f["kv_cache_numbers_per_layer"]
    assert round(3 * 576 * 2 / 1024, 1) == f["draft_kv_cache_kib_per_token"]
    assert round(f["target_layers"] * 576 * 2 / 1024, 1) == f["target_kv_cache_kib_per_token"]


def test_workload_dims_follow_page():
    f = FACTS
    for wid in (2, 3, 4, 5):
        wl = synth.WORKLOADS[wid]
        assert (wl.n_h, wl.d_c, wl.d_r, wl.d_v, wl.W) == (f["n_h"], f["d_c"], f["d_r"], f["d_v"], f["W"])
    assert f["W"] - 1 == f["visible_context_max"]
    assert (f["d_c"] + f["d_r"]) ** -0.5 == 1.0 / 16


def test_anchor_candidates_rule(oracle_mod):
    """Page §2: A in [0, S-2], loss_mask[A] = loss_mask[A+1] = 1, with
    loss_mask[S-1] read as 0 (so A = S-2 is never a candidate)."""
    lm = np.array([1, 1, 0, 1, 1, 1, 0, 1, 1], np.uint8)
    assert oracle_mod.anchor_candidates(lm).tolist() == [0, 3, 4]
    lm = np.ones(10, np.uint8)
    assert oracle_mod.anchor_candidates(lm).tolist() == list(range(8))
    assert oracle_mod.anchor_candidates(np.ones(2, np.uint8)).tolist() == []


def test_synth_anchors_are_candidates(oracle_mod):
    for wid in (2, 5):
        wl = synth.WORKLOADS[wid].with_(n_h=1, d_c=2, d_r=2, d_v=2)
        c = synth.make_inputs(wl, with_grad=False)
        for b in range(wl.B):
            cand = set(oracle_mod.anchor_candidates(c["loss_mask"][b].numpy()).tolist())
            an = c["anchors"][b].numpy()
            assert len(set(an.tolist())) == wl.N  # without replacement
            assert set(an.tolist()) <= cand
        if wid == 5:
            assert int((c["keep"] == 0).sum()) == wl.B * (wl.N // 10)
    wl = synth.WORKLOADS[4].with_(n_h=1, d_c=2, d_r=2, d_v=2)
    c = synth.make_inputs(wl, with_grad=False)
    an = c["anchors"][0].numpy()
    assert (an < 127).sum() == 16 and 0 in an and an.max() <= wl.S - 2 and len(set(an.tolist())) == wl.N
