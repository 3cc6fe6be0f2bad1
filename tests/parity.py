"""Helpers for GPU-vs-oracle parity tests (imported by the test modules).

Tolerances (stated for the spec workloads, fp64 reference):
  fp32 outputs: max |gpu - ref| <= 1e-5.
  bf16 outputs: per element |gpu - ref| <= 2e-2 + 1e-2 * |ref|, and
                normwise max|gpu - ref| / max|ref| <= 1e-2.
The GPU result is compared after its own rounding to the output dtype. LSE is
fp32 in both cases and is held to the bound of the problem's dtype.
"""
import numpy as np
import torch

from speculative_draft_mla_b200 import capi

F32_ATOL = 1e-5
BF16_ATOL, BF16_RTOL, BF16_NORM = 2e-2, 1e-2, 1e-2


def to_dev(c, device="cuda"):
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in c.items()}


def run_gpu(c, S, W, base=10000.0, bwd=True, workspace=None):
    """Forward (and backward) through the C ABI; returns CPU tensors."""
    d = to_dev(c)
    o, lse, ws = capi.attn_fwd(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], S, W, base,
                               workspace=workspace)
    out = dict(o=o, lse=lse)
    if bwd:
        dq, dkc, dkr, dv = capi.attn_bwd(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], o, lse,
                                         d["dout"], S, W, base, workspace=ws,
                                         flags=capi.FLAG_REUSE_DESCRIPTOR)
        out.update(dq=dq, dkc=dkc, dkr=dkr, dv=dv)
    capi.get_error(ws)
    torch.cuda.synchronize()
    return {k: v.cpu() for k, v in out.items()}


def assert_close(gpu, ref, dtype, what=""):
    g = gpu.double().numpy() if torch.is_tensor(gpu) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    ninf_g, ninf_r = np.isneginf(g), np.isneginf(r)
    assert np.array_equal(ninf_g, ninf_r), "%s: -inf pattern differs" % what
    fin = ~ninf_r
    g, r = g[fin], r[fin]
    assert np.all(np.isfinite(g)), "%s: non-finite values" % what
    if g.size == 0:
        return
    err = np.abs(g - r)
    if dtype == torch.float32:
        assert err.max() <= F32_ATOL, "%s: max abs err %.3g > %g" % (what, err.max(), F32_ATOL)
    else:
        bound = BF16_ATOL + BF16_RTOL * np.abs(r)
        worst = np.argmax(err - bound)
        assert np.all(err <= bound), "%s: err %.4g > bound %.4g at %d (ref %.4g)" % (
            what, err[worst], bound[worst], worst, r[worst])
        scale = max(np.abs(r).max(), 1e-30)
        assert err.max() / scale <= BF16_NORM, "%s: normwise %.3g" % (what, err.max() / scale)


def oracle_full(oracle_mod, c, S, W, base=10000.0, bwd=True):
    args = [c[k].double().numpy() for k in ("q", "kc", "kr", "v")]
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    o, lse = oracle_mod.attn_fwd(*args, an, kp, S, W, base)
    out = dict(o=o, lse=lse)
    if bwd:
        dq, dkc, dkr, dv = oracle_mod.attn_bwd(*args, an, kp, c["dout"].double().numpy(), S, W, base)
        out.update(dq=dq, dkc=dkc, dkr=dkr, dv=dv)
    return out


def compare_full(gpu, ref, dtype, keys=("o", "lse", "dq", "dkc", "dkr", "dv")):
    for k in keys:
        if k in ref:
            assert_close(gpu[k], ref[k], dtype, k)
