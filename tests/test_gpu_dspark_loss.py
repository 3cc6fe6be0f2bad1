"""DSpark loss over the draft steps (page §6) through the C ABI against the
fp64 oracle.

Tolerances: the kernel works in fp32 on the bf16 logits (the oracle in fp64 on
the same values): the scalar means agree to 1e-4 relative. The logit gradient
is rounded to bf16: per element |g - ref| <= 1e-2 |ref| + 2e-3 max|ref|,
except where the sign of p - q is not decided within fp32 (|log p - log q| <
1e-4 in fp64): there both signs are correct and the element is not compared.
"""
import numpy as np
import pytest
import torch

from oracle import dspark_loss as odl
from speculative_draft_mla_b200 import build as dbuild
from speculative_draft_mla_b200 import capi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dbuild.build()
    return capi.load()


def _inputs(seed, R, V, scale=3.0, device="cuda"):
    g = torch.Generator(device=device).manual_seed(seed)
    L = (torch.randn(R, V, generator=g, device=device) * scale).to(torch.bfloat16)
    T = (torch.randn(R, V, generator=g, device=device) * scale).to(torch.bfloat16)
    y = torch.randint(0, V, (R,), generator=g, device=device, dtype=torch.int32)
    c = torch.randn(R, generator=g, device=device) * 1.5
    m = (torch.rand(R, generator=g, device=device) < 0.8).to(torch.uint8)
    return L, T, y, c, m


def _ambiguous(L, T):
    Lr, Tr = L.double().cpu().numpy(), T.double().cpu().numpy()
    ll = Lr - np.log(np.exp(Lr - Lr.max(1, keepdims=True)).sum(1, keepdims=True)) - Lr.max(1, keepdims=True)
    lt = Tr - np.log(np.exp(Tr - Tr.max(1, keepdims=True)).sum(1, keepdims=True)) - Tr.max(1, keepdims=True)
    return np.abs(ll - lt) < 1e-4


def _check_grad(g, ref, amb):
    g = g.float().cpu().numpy().astype(np.float64)
    scale = np.abs(ref).max()
    bad = (np.abs(g - ref) > 1e-2 * np.abs(ref) + 2e-3 * scale) & ~amb
    assert not bad.any(), (np.argwhere(bad)[:5], g[bad][:5], ref[bad][:5])


@pytest.mark.parametrize("R,V", [(7, 64), (13, 1000), (40, 4096), (1, 8), (20, 154880)])
def test_loss_matches_oracle(R, V):
    L, T, y, c, m = _inputs(R * 1000 + V, R, V)
    y[0] = -1  # a label outside [0, V): no CE term
    m[0] = 1
    out, g, gc, _ = capi.dspark_loss(L, T, y, c, m)
    ref = odl.loss_fwd_bwd(L.double().cpu().numpy(), T.double().cpu().numpy(), y.cpu().numpy(),
                           c.double().cpu().numpy(), m.cpu().numpy())
    got = out.cpu().numpy()
    for i, k in enumerate(("loss", "ce", "l1", "conf")):
        assert abs(got[i] - ref[k]) <= 1e-4 * abs(ref[k]) + 1e-6, (k, got[i], ref[k])
    _check_grad(g, ref["grad_logits"], _ambiguous(L, T))
    assert np.allclose(gc.cpu().numpy(), ref["grad_conf"], rtol=1e-4, atol=1e-7)


def test_no_counted_steps_and_loss_only():
    L, T, y, c, m = _inputs(5, 9, 512)
    out, g, gc, _ = capi.dspark_loss(L, T, y, c, torch.zeros_like(m))
    assert not out.any() and not g.float().any() and not gc.any()
    out2, g2, gc2, _ = capi.dspark_loss(L, T, y, c, m, with_grad=False)
    out3, _, _, _ = capi.dspark_loss(L, T, y, c, m)
    assert g2 is None and gc2 is None and torch.equal(out2, out3)
    out4, _, _, _ = capi.dspark_loss(L[:0], T[:0], y[:0], c[:0], m[:0])  # R = 0
    assert not out4.any()


def test_full_workload_sampled_rows():
    """The benchmark's loss workload (R = 5120 draft steps, V = 154880): sampled
    rows' per-step values (from the workspace) and gradients against the
    oracle on those rows alone, the totals against the per-step values."""
    R, V = 5120, 154880
    L, T, y, c, m = _inputs(77, R, V)
    out, g, gc, ws = capi.dspark_loss(L, T, y, c, m)
    M = int(m.sum())
    stats = ws[256:256 + 16 * R].view(torch.float32).view(R, 4).cpu().numpy()
    mm = m.cpu().numpy().astype(bool)
    tot = stats[mm, :3].astype(np.float64).sum(0) / M
    got = out.cpu().numpy()
    assert np.allclose(got[1:], tot, rtol=1e-5) and abs(got[0] - (tot[0] + 0.9 * tot[1] + tot[2])) < 1e-4 * got[0]
    rows = [0, 1, 2, 1000, 2047, 2048, 4095, 5119] + list(np.random.default_rng(1).integers(0, R, 8))
    sel = torch.tensor(rows, device="cuda")
    Ls, Ts = L[sel], T[sel]
    ref = odl.loss_fwd_bwd(Ls.double().cpu().numpy(), Ts.double().cpu().numpy(), y[sel].cpu().numpy(),
                           c[sel].double().cpu().numpy(), np.ones(len(rows), np.uint8))
    for i, r in enumerate(rows):
        for k, name in enumerate(("ce_r", "l1_r", "bce_r", "a_r")):
            assert abs(stats[r, k] - ref[name][i]) <= 1e-4 * abs(ref[name][i]) + 1e-5, (r, name)
    # gradients: the oracle normalises by the sampled rows' count, the kernel by M
    scale = np.array([(M / len(rows)) if mm[r] else 0.0 for r in rows])
    gg = g[sel].float().cpu().numpy().astype(np.float64) * M
    want = ref["grad_logits"] * len(rows) * (scale[:, None] > 0)
    _check_grad(torch.from_numpy(gg / M), want / M, _ambiguous(Ls, Ts))
