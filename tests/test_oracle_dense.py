"""Pin: the window-form C oracle equals the dense-mask brute force.

The "GLM 5.2 DSpark speculative-training design" page states the attention two
ways: per block through its key set (§3 attention mask) and as
softmax(QK^T/sqrt(d) + Lambda(M))V over a materialised boolean mask (appendix
"Attention implementation"). ``oracle/dense.py`` implements the second with
whole-matrix products and complex-number RoPE; the C oracle implements the
first with loops and explicit cos/sin. Agreement to fp64 rounding on many tiny
cases (including clipped and empty windows, W = 1, duplicates, padding blocks)
pins the mask rule, the RoPE positions and the softmax.
"""
import numpy as np
import pytest

from oracle import dense
from speculative_draft_mla_b200 import synth

CASES = [
    # (seed, B, S, N, W, n_h, d_c, d_r, d_v, keep_frac, dup)
    (1, 1, 20, 3, 4, 2, 4, 2, 3, 1.0, False),
    (2, 2, 12, 4, 16, 3, 6, 4, 5, 1.0, False),  # W > S: every window clipped at 0
    (3, 1, 2, 1, 3, 1, 2, 2, 2, 1.0, False),    # S = 2: only A = 0
    (4, 2, 30, 6, 1, 2, 4, 4, 4, 1.0, False),   # W = 1: block-only attention
    (5, 1, 40, 8, 8, 2, 8, 0, 6, 0.6, False),   # d_r = 0, padding blocks
    (6, 2, 25, 7, 5, 2, 2, 6, 3, 1.0, True),    # duplicate anchors
    (7, 1, 64, 4, 16, 4, 32, 16, 32, 1.0, False),
    (8, 1, 17, 5, 2, 1, 3, 2, 1, 0.0, False),   # every block padding
    (9, 3, 9, 2, 3, 2, 0, 4, 4, 0.5, True),     # d_c = 0
]


def _run(case):
    seed, B, S, N, W, n_h, d_c, d_r, d_v, kf, dup = case
    c = synth.random_case(seed, B, S, N, W, n_h, d_c, d_r, d_v, "f32", keep_frac=kf, allow_dup=dup)
    return c, (B, S, N, W, n_h, d_c, d_r, d_v)


@pytest.mark.parametrize("case", CASES)
def test_window_oracle_matches_dense(oracle_mod, case):
    c, (B, S, N, W, n_h, d_c, d_r, d_v) = _run(case)
    args = [c[k].double().numpy() for k in ("q", "kc", "kr", "v")]
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    o, lse = oracle_mod.attn_fwd(*args, an, kp, S, W, 10000.0)
    o2, lse2 = dense.dense_forward(*args, an, kp, S, N, W, d_c, d_r, 10000.0)
    np.testing.assert_allclose(o, o2, rtol=1e-11, atol=1e-11)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse2))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], lse2[fin], rtol=1e-12, atol=1e-12)
    # padding rows: O = 0 and LSE = -inf; kept rows: finite LSE
    rows_keep = np.repeat(kp.astype(bool), 5, axis=1)[:, None, :]
    assert np.all(np.isneginf(lse) == ~rows_keep)
    assert np.all(o[np.broadcast_to(~rows_keep, lse.shape)] == 0.0)


def test_rows_entry_matches_full(oracle_mod):
    c, (B, S, N, W, n_h, d_c, d_r, d_v) = _run(CASES[1])
    args = [c[k].double().numpy() for k in ("q", "kc", "kr", "v")]
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    o, lse = oracle_mod.attn_fwd(*args, an, kp, S, W, 10000.0)
    rows = np.array([[b, h, r] for b in range(B) for h in range(n_h) for r in range(5 * N)], np.int32)
    o2, lse2 = oracle_mod.attn_fwd_rows(*args, an, kp, S, W, 10000.0, rows)
    np.testing.assert_array_equal(o.reshape(-1, d_v), o2)
    np.testing.assert_array_equal(lse.reshape(-1), lse2)


def test_mask_matrix_counts():
    """Mask facts the appendix states: at most W-1 context nonzeros per kept
    row, exactly block_size draft nonzeros, padding rows all zero."""
    S, N, W = 300, 6, 128
    anchors = np.array([0, 5, 126, 127, 200, 298])
    keep = np.array([1, 1, 1, 1, 0, 1])
    M = dense.mask_matrix(S, N, W, anchors, keep)
    for n in range(N):
        rows = M[5 * n:5 * n + 5]
        if not keep[n]:
            assert not rows.any()
            continue
        a = anchors[n]
        assert rows[:, :S].sum(axis=1).tolist() == [min(a, W - 1)] * 5
        assert rows[:, S:].sum(axis=1).tolist() == [5] * 5
        assert rows[:, S + 5 * n:S + 5 * n + 5].all()
        assert not rows[:, a:S].any()  # context position A itself is excluded
