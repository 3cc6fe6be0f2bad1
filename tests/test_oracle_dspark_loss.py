"""Pins of the DSpark loss oracle (page §6) against library routines, special
cases and finite differences; no GPU."""
import numpy as np
import torch
import torch.nn.functional as F

from oracle import dspark_loss as dl


def _case(seed, R=4, V=11, scale=2.0):
    rng = np.random.default_rng(seed)
    L = rng.normal(0, scale, (R, V))
    T = rng.normal(0, scale, (R, V))
    y = rng.integers(0, V, R)
    c = rng.normal(0, 1.5, R)
    m = np.array([1, 0, 1, 1][:R] + [1] * max(0, R - 4), np.uint8)
    return L, T, y, c, m


def test_terms_match_torch():
    L, T, y, c, m = _case(1)
    out = dl.loss_fwd_bwd(L, T, y, c, m)
    ce = F.cross_entropy(torch.tensor(L), torch.tensor(y), reduction="none").numpy()
    assert np.allclose(out["ce_r"], ce, rtol=0, atol=1e-12)
    bce = F.binary_cross_entropy_with_logits(torch.tensor(c), torch.tensor(out["a_r"]), reduction="none").numpy()
    assert np.allclose(out["bce_r"], bce, rtol=0, atol=1e-12)
    sel = m == 1
    want = (ce[sel].mean() + 0.9 * out["l1_r"][sel].mean() + bce[sel].mean())
    assert abs(out["loss"] - want) < 1e-12


def test_l1_special_cases():
    V = 9
    L = np.random.default_rng(2).normal(size=(1, V))
    z = dl.loss_fwd_bwd(L, L.copy(), [0], [0.0], [1])
    assert abs(z["l1_r"][0]) < 1e-15 and abs(z["a_r"][0] - 1.0) < 1e-15  # identical distributions
    P = np.full((1, V), -60.0)
    Q = P.copy()
    P[0, 1] = 60.0
    Q[0, 4] = 60.0
    d = dl.loss_fwd_bwd(P, Q, [1], [0.0], [1])
    assert abs(d["l1_r"][0] - 2.0) < 1e-12 and abs(d["a_r"][0]) < 1e-12   # disjoint: L1 = 2, target 0
    for seed in range(5):
        L, T, y, c, m = _case(seed, V=30)
        l1 = dl.loss_fwd_bwd(L, T, y, c, m)["l1_r"]
        assert (l1 >= 0).all() and (l1 <= 2).all()


def test_gradients_finite_differences():
    """Central differences of the loss with the confidence targets held at
    their values (the page stops the gradient through a)."""
    L, T, y, c, m = _case(3, R=3, V=7)
    base = dl.loss_fwd_bwd(L, T, y, c, m)
    a = base["a_r"]
    h = 1e-6
    for r in range(3):
        for i in range(7):
            Lp, Lm = L.copy(), L.copy()
            Lp[r, i] += h
            Lm[r, i] -= h
            fd = (dl.loss_fwd_bwd(Lp, T, y, c, m, a_override=a)["loss"] -
                  dl.loss_fwd_bwd(Lm, T, y, c, m, a_override=a)["loss"]) / (2 * h)
            assert abs(fd - base["grad_logits"][r, i]) < 1e-7, (r, i)
        cp, cm = c.copy(), c.copy()
        cp[r] += h
        cm[r] -= h
        fd = (dl.loss_fwd_bwd(L, T, y, cp, m, a_override=a)["loss"] -
              dl.loss_fwd_bwd(L, T, y, cm, m, a_override=a)["loss"]) / (2 * h)
        assert abs(fd - base["grad_conf"][r]) < 1e-7, r


def test_mask_invariants():
    L, T, y, c, m = _case(4, R=6, V=13)
    out = dl.loss_fwd_bwd(L, T, y, c, m)
    sel = np.nonzero(m)[0]
    sub = dl.loss_fwd_bwd(L[sel], T[sel], y[sel], c[sel], m[sel])
    assert abs(out["loss"] - sub["loss"]) < 1e-12
    assert (out["grad_logits"][m == 0] == 0).all() and (out["grad_conf"][m == 0] == 0).all()
    assert np.allclose(out["grad_logits"][sel], sub["grad_logits"], atol=1e-15)
    zero = dl.loss_fwd_bwd(L, T, y, c, np.zeros(6, np.uint8))
    assert zero["loss"] == 0 and not zero["grad_logits"].any() and not zero["grad_conf"].any()
    # each counted row's logit gradient sums to zero (softmax Jacobian rows)
    assert np.allclose(out["grad_logits"].sum(axis=1), 0, atol=1e-14)
