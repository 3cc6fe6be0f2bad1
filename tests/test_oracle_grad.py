"""Pins of the oracle's hand-derived backward.

- Central finite differences of the loss sum(dO * O) computed by the dense
  brute force (oracle/dense.py), in fp64, along random directions and along
  single coordinates, for every input tensor.
- The gather form (one key or row at a time) against the scatter form.
- Invariants that follow from softmax rows summing to one:
  per head, sum over keys of dV equals sum over kept rows of dO, and the sum
  over keys of the unrotated d K^C is zero.
"""
import numpy as np
import pytest

from oracle import dense
from speculative_draft_mla_b200 import synth

BASE = 10000.0


def _loss(args, an, kp, S, N, W, d_c, d_r, dout):
    o, _ = dense.dense_forward(*args, an, kp, S, N, W, d_c, d_r, BASE)
    return float((o * dout).sum())


CASES = [
    (21, 1, 24, 3, 6, 2, 4, 4, 3, 1.0, False),
    (22, 2, 10, 2, 16, 2, 2, 2, 2, 0.5, True),   # clipped windows, padding, duplicates
    (23, 1, 64, 4, 16, 4, 32, 16, 32, 1.0, False),
]


@pytest.mark.parametrize("case", CASES)
def test_directional_finite_differences(oracle_mod, case):
    seed, B, S, N, W, n_h, d_c, d_r, d_v, kf, dup = case
    c = synth.random_case(seed, B, S, N, W, n_h, d_c, d_r, d_v, "f32", keep_frac=kf, allow_dup=dup)
    args = [c[k].double().numpy() for k in ("q", "kc", "kr", "v")]
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    dout = c["dout"].double().numpy()
    grads = oracle_mod.attn_bwd(*args, an, kp, dout, S, W, BASE)
    rng = np.random.default_rng(seed)
    h = 1e-5
    for which in range(4):
        for _ in range(3):
            u = rng.standard_normal(args[which].shape)
            plus = list(args); plus[which] = args[which] + h * u
            minus = list(args); minus[which] = args[which] - h * u
            fd = (_loss(plus, an, kp, S, N, W, d_c, d_r, dout) - _loss(minus, an, kp, S, N, W, d_c, d_r, dout)) / (2 * h)
            an_ = float((grads[which] * u).sum())
            assert abs(fd - an_) <= 1e-6 * max(1.0, abs(an_)), (which, fd, an_)


def test_coordinate_finite_differences(oracle_mod):
    seed, B, S, N, W, n_h, d_c, d_r, d_v = 24, 1, 12, 2, 5, 2, 2, 4, 2
    c = synth.random_case(seed, B, S, N, W, n_h, d_c, d_r, d_v, "f32")
    c["anchors"][0] = c["anchors"].new_tensor([6, 2])
    args = [c[k].double().numpy() for k in ("q", "kc", "kr", "v")]
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    dout = c["dout"].double().numpy()
    grads = oracle_mod.attn_bwd(*args, an, kp, dout, S, W, BASE)
    h = 1e-6
    for which in range(4):
        flat = args[which].reshape(-1)
        for idx in range(flat.size):
            plus = [a.copy() for a in args]; plus[which].reshape(-1)[idx] += h
            minus = [a.copy() for a in args]; minus[which].reshape(-1)[idx] -= h
            fd = (_loss(plus, an, kp, S, N, W, d_c, d_r, dout) - _loss(minus, an, kp, S, N, W, d_c, d_r, dout)) / (2 * h)
            g = grads[which].reshape(-1)[idx]
            assert abs(fd - g) <= 1e-6 * max(1.0, abs(g)), (which, idx, fd, g)


def test_gather_equals_scatter(oracle_mod):
    seed, B, S, N, W, n_h, d_c, d_r, d_v = 25, 2, 40, 6, 12, 3, 6, 4, 5
    c = synth.random_case(seed, B, S, N, W, n_h, d_c, d_r, d_v, "f32", keep_frac=0.8, allow_dup=True)
    args = [c[k].double().numpy() for k in ("q", "kc", "kr", "v")]
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    dout = c["dout"].double().numpy()
    dq, dkc, dkr, dv = oracle_mod.attn_bwd(*args, an, kp, dout, S, W, BASE)
    L = S + 5 * N
    rows = np.array([[b, h, r] for b in range(B) for h in range(n_h) for r in range(5 * N)])
    g = oracle_mod.attn_bwd_items(*args, an, kp, dout, S, W, BASE, "dq", rows)
    np.testing.assert_allclose(g, dq.reshape(-1, d_c + d_r), rtol=1e-12, atol=1e-12)
    keys = np.array([[b, h, k] for b in range(B) for h in range(n_h) for k in range(L)])
    g = oracle_mod.attn_bwd_items(*args, an, kp, dout, S, W, BASE, "dkv", keys)
    np.testing.assert_allclose(g[:, :d_c], dkc.reshape(-1, d_c), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[:, d_c:], dv.reshape(-1, d_v), rtol=1e-12, atol=1e-12)
    keys = np.array([[b, k] for b in range(B) for k in range(L)])
    g = oracle_mod.attn_bwd_items(*args, an, kp, dout, S, W, BASE, "dkr", keys)
    np.testing.assert_allclose(g, dkr.reshape(-1, d_r), rtol=1e-12, atol=1e-12)


def test_softmax_sum_invariants(oracle_mod):
    seed, B, S, N, W, n_h, d_c, d_r, d_v = 26, 2, 60, 7, 16, 3, 6, 4, 5
    c = synth.random_case(seed, B, S, N, W, n_h, d_c, d_r, d_v, "f32", keep_frac=0.7)
    args = [c[k].double().numpy() for k in ("q", "kc", "kr", "v")]
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    dout = c["dout"].double().numpy()
    dq, dkc, dkr, dv = oracle_mod.attn_bwd(*args, an, kp, dout, S, W, BASE)
    kept_rows = np.repeat(kp.astype(bool), 5, axis=1)[:, None, :, None]
    np.testing.assert_allclose(dv.sum(axis=2), (dout * kept_rows).sum(axis=2), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(dkc.sum(axis=2), 0.0, atol=1e-11)
    # padding rows and the draft keys of padding blocks get zero gradients
    pad_rows = ~np.broadcast_to(kept_rows, dq.shape[:3] + (1,))[..., 0]
    assert np.all(dq[pad_rows] == 0)
    for b in range(B):
        for n in range(N):
            if not kp[b, n]:
                ks = slice(S + 5 * n, S + 5 * n + 5)
                assert np.all(dkc[b, :, ks] == 0) and np.all(dv[b, :, ks] == 0) and np.all(dkr[b, ks] == 0)
