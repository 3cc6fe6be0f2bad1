"""Pins of the oracle against textbook special cases and invariants.

Special cases reduce the DSpark draft attention to plain softmax attention,
computed here by torch's scaled_dot_product_attention (a library routine, fp64
CPU) with RoPE applied as a complex multiplication (torch.polar). Invariants come
from the §3 mask rules and from RoPE being a relative-position encoding.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from speculative_draft_mla_b200 import synth

BASE = 10000.0


def rope_polar(x, pos, base=BASE):
    """Interleaved-pair RoPE as complex multiplication (torch.polar)."""
    d_r = x.shape[-1]
    if d_r == 0:
        return x
    theta = base ** (-2.0 * torch.arange(d_r // 2, dtype=torch.float64) / d_r)
    z = torch.view_as_complex(x.reshape(*x.shape[:-1], d_r // 2, 2).contiguous())
    rot = torch.polar(torch.ones_like(theta), pos.to(torch.float64)[..., None] * theta)
    return torch.view_as_real(z * rot).reshape(x.shape)


def _np(c):
    return [c[k].double().numpy() for k in ("q", "kc", "kr", "v")]


def sdpa_rows(c, b, h, n, keys, key_pos, a, d_c):
    """Textbook attention of block n's 5 rows over an explicit key list."""
    q = c["q"][b, h, 5 * n:5 * n + 5].double()
    qpos = torch.arange(5, dtype=torch.float64) + a
    q = torch.cat([q[:, :d_c], rope_polar(q[:, d_c:], qpos)], dim=-1)
    keys = torch.as_tensor(keys)
    k = torch.cat([c["kc"][b, h, keys].double(),
                   rope_polar(c["kr"][b, keys].double(), torch.as_tensor(key_pos, dtype=torch.float64))], dim=-1)
    v = c["v"][b, h, keys].double()
    return F.scaled_dot_product_attention(q[None], k[None], v[None])[0]


@pytest.mark.parametrize("d_r", [0, 8])
def test_anchor_zero_is_plain_block_attention(oracle_mod, d_r):
    """A = 0: the context window is empty, so each row is ordinary softmax
    attention over its block's 5 positions (bidirectional)."""
    S, N, W, n_h, d_c, d_v = 16, 3, 8, 2, 6, 5
    c = synth.random_case(11, 1, S, N, W, n_h, d_c, d_r, d_v, "f32")
    c["anchors"][0] = torch.tensor([0, 7, 0], dtype=torch.int32)
    o, _ = oracle_mod.attn_fwd(*_np(c), c["anchors"].numpy(), c["keep"].numpy(), S, W, BASE)
    for h in range(n_h):
        for n in (0, 2):
            keys = [S + 5 * n + i for i in range(5)]
            ref = sdpa_rows(c, 0, h, n, keys, [0, 1, 2, 3, 4], 0, d_c)
            np.testing.assert_allclose(o[0, h, 5 * n:5 * n + 5], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_window_one_is_block_only(oracle_mod):
    """W = 1: no context position is visible for any anchor."""
    S, N, W, n_h, d_c, d_r, d_v = 40, 4, 1, 2, 4, 4, 3
    c = synth.random_case(12, 1, S, N, W, n_h, d_c, d_r, d_v, "f32")
    an = c["anchors"].numpy()
    o, _ = oracle_mod.attn_fwd(*_np(c), an, c["keep"].numpy(), S, W, BASE)
    for h in range(n_h):
        for n in range(N):
            a = int(an[0, n])
            ref = sdpa_rows(c, 0, h, n, [S + 5 * n + i for i in range(5)], [a + i for i in range(5)], a, d_c)
            np.testing.assert_allclose(o[0, h, 5 * n:5 * n + 5], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_general_row_is_sdpa_over_window(oracle_mod):
    """Any anchor: SDPA over [max(0,A-W+1), A) plus the own block, with RoPE
    positions c for context and A+i for the block (page §2, §3, §4)."""
    S, N, W, n_h, d_c, d_r, d_v = 64, 5, 16, 3, 8, 8, 4
    c = synth.random_case(13, 2, S, N, W, n_h, d_c, d_r, d_v, "f32")
    c["anchors"][1, :3] = torch.tensor([3, 15, 62], dtype=torch.int32)
    an = c["anchors"].numpy()
    o, _ = oracle_mod.attn_fwd(*_np(c), an, c["keep"].numpy(), S, W, BASE)
    for b in range(2):
        for n in range(N):
            a = int(an[b, n])
            ctx = list(range(max(0, a - W + 1), a))
            keys = ctx + [S + 5 * n + i for i in range(5)]
            pos = ctx + [a + i for i in range(5)]
            for h in range(n_h):
                ref = sdpa_rows(c, b, h, n, keys, pos, a, d_c)
                np.testing.assert_allclose(o[b, h, 5 * n:5 * n + 5], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_scale_is_inverse_sqrt_qk_dim(oracle_mod):
    """Scale (d_c + d_r)^(-1/2) (page §4): doubling q by 2 equals scaling the
    logits by 2, which SDPA reproduces with scale=2/sqrt(d)."""
    S, N, W, n_h, d_c, d_r, d_v = 20, 2, 6, 1, 6, 2, 3
    c = synth.random_case(14, 1, S, N, W, n_h, d_c, d_r, d_v, "f32")
    c["anchors"][0] = torch.tensor([0, 0], dtype=torch.int32)
    c2 = dict(c)
    c2["q"] = c["q"] * 2
    o, _ = oracle_mod.attn_fwd(*_np(c2), c["anchors"].numpy(), c["keep"].numpy(), S, W, BASE)
    q = c["q"][0, 0, 0:5].double()
    qpos = torch.arange(5, dtype=torch.float64)
    q = torch.cat([q[:, :d_c], rope_polar(q[:, d_c:], qpos)], -1)
    keys = torch.arange(S, S + 5)
    k = torch.cat([c["kc"][0, 0, keys].double(), rope_polar(c["kr"][0, keys].double(), qpos)], -1)
    ref = F.scaled_dot_product_attention(q[None], k[None], c["v"][0, 0, keys].double()[None],
                                         scale=2.0 / math.sqrt(d_c + d_r))[0]
    np.testing.assert_allclose(o[0, 0, 0:5], ref.numpy(), rtol=1e-12, atol=1e-12)


def _perturb(c, b, key, which, rng):
    c = {k: v.clone() for k, v in c.items()}
    if which == "kc":
        c["kc"][b, :, key] += torch.from_numpy(rng.standard_normal(c["kc"][b, :, key].shape)).float()
    elif which == "kr":
        c["kr"][b, key] += torch.from_numpy(rng.standard_normal(c["kr"][b, key].shape)).float()
    else:
        c["v"][b, :, key] += torch.from_numpy(rng.standard_normal(c["v"][b, :, key].shape)).float()
    return c


@pytest.mark.parametrize("which", ["kc", "kr", "v"])
def test_window_edges(oracle_mod, which):
    """Context A and A-W are invisible, A-W+1 and A-1 are visible, and another
    block's draft keys are invisible (page §3)."""
    S, N, W, n_h, d_c, d_r, d_v = 64, 3, 8, 2, 4, 4, 4
    c = synth.random_case(15, 1, S, N, W, n_h, d_c, d_r, d_v, "f32")
    c["anchors"][0] = torch.tensor([30, 50, 10], dtype=torch.int32)
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    base_o, _ = oracle_mod.attn_fwd(*_np(c), an, kp, S, W, BASE)
    rng = np.random.default_rng(0)
    n, a = 0, 30
    rows = slice(0, 5)
    for key, visible in [(a, False), (a - W, False), (a - W + 1, True), (a - 1, True),
                         (S + 5 * 1, False), (S + 5 * 2 + 4, False), (S + 0, True), (S + 4, True)]:
        c2 = _perturb(c, 0, key, which, rng)
        o2, _ = oracle_mod.attn_fwd(*_np(c2), an, kp, S, W, BASE)
        changed = np.abs(o2[0, :, rows] - base_o[0, :, rows]).max() > 1e-9
        assert changed == visible, (key, which)


def test_block_permutation_equivariance(oracle_mod):
    S, N, W, n_h, d_c, d_r, d_v = 50, 6, 10, 2, 4, 4, 3
    c = synth.random_case(16, 1, S, N, W, n_h, d_c, d_r, d_v, "f32", keep_frac=0.7)
    perm = np.array([3, 0, 5, 1, 4, 2])
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    o, lse = oracle_mod.attn_fwd(*_np(c), an, kp, S, W, BASE)
    rows = (perm[:, None] * 5 + np.arange(5)[None]).reshape(-1)
    keys = np.concatenate([np.arange(S), S + rows])
    c2 = dict(q=c["q"][:, :, rows], kc=c["kc"][:, :, keys], kr=c["kr"][:, keys], v=c["v"][:, :, keys])
    o2, lse2 = oracle_mod.attn_fwd(*_np(c2), an[:, perm], kp[:, perm], S, W, BASE)
    np.testing.assert_allclose(o2, o[:, :, rows], rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(lse2, lse[:, :, rows])


def test_rope_relativity(oracle_mod):
    """Shifting an anchor by delta and the context content with it leaves O
    unchanged (windows unclipped), since RoPE scores depend on position
    differences only."""
    S, N, W, n_h, d_c, d_r, d_v, delta = 80, 2, 12, 2, 4, 8, 3, 17
    c = synth.random_case(17, 1, S, N, W, n_h, d_c, d_r, d_v, "f32")
    c["anchors"][0] = torch.tensor([20, 40], dtype=torch.int32)
    c2 = {k: v.clone() for k, v in c.items()}
    c2["anchors"][0] = c["anchors"][0] + delta
    for key in ("kc", "v"):
        c2[key][:, :, delta:S] = c[key][:, :, :S - delta]
    c2["kr"][:, delta:S] = c["kr"][:, :S - delta]
    o, lse = oracle_mod.attn_fwd(*_np(c), c["anchors"].numpy(), c["keep"].numpy(), S, W, BASE)
    o2, lse2 = oracle_mod.attn_fwd(*_np(c2), c2["anchors"].numpy(), c2["keep"].numpy(), S, W, BASE)
    np.testing.assert_allclose(o2, o, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(lse2, lse, rtol=1e-10, atol=1e-10)


def test_rope_position_zero_is_identity_and_pairs_interleaved(oracle_mod):
    """A = 0, row j = 0: the query rope slice is unrotated. Swapping which two
    entries form a pair changes the result (adjacent pairs are what rotates)."""
    S, N, W, n_h, d_c, d_r, d_v = 8, 1, 4, 1, 0, 4, 2
    c = synth.random_case(18, 1, S, N, W, n_h, d_c, d_r, d_v, "f32")
    c["anchors"][0, 0] = 0
    o, _ = oracle_mod.attn_fwd(*_np(c), c["anchors"].numpy(), c["keep"].numpy(), S, W, BASE)
    # Row 0 at position 0 against keys at positions 0..4: recompute with the
    # angle of pair i equal to pos * base^(-2i/d_r) written as a 2x2 matrix.
    q = c["q"][0, 0, 0].double().numpy()
    keys = np.arange(S, S + 5)
    scores = []
    for t, key in enumerate(keys):
        k = c["kr"][0, key].double().numpy()
        kr = np.empty(4)
        for i in range(2):
            ang = t * BASE ** (-2.0 * i / 4)
            R = np.array([[math.cos(ang), -math.sin(ang)], [math.sin(ang), math.cos(ang)]])
            kr[2 * i:2 * i + 2] = R @ k[2 * i:2 * i + 2]
        scores.append(q @ kr / 2.0)
    p = np.exp(np.array(scores) - max(scores))
    p /= p.sum()
    ref = p @ c["v"][0, 0, keys].double().numpy()
    np.testing.assert_allclose(o[0, 0, 0], ref, rtol=1e-12, atol=1e-12)
