"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small workloads are compared element by element on every output; the tiny
fp32 workload and the 2048-context bf16 workload are compared in full. The
three large workloads run at full size in the launch configuration the
benchmark times and are checked on sampled rows and keys that the oracle
computes one by one, plus properties that hold at any size.
"""
import numpy as np
import pytest
import torch

from parity import assert_close, compare_full, oracle_full, run_gpu, to_dev
from speculative_draft_mla_b200 import build as dbuild
from speculative_draft_mla_b200 import capi, synth

pytestmark = pytest.mark.gpu
BASE = 10000.0


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dbuild.build()
    return capi.load()


def test_tiny_f32_workload_full(oracle_mod):
    wl = synth.WORKLOADS[1]
    c = synth.make_inputs(wl)
    gpu = run_gpu(c, wl.S, wl.W)
    compare_full(gpu, oracle_full(oracle_mod, c, wl.S, wl.W), torch.float32)


# (name, seed, B, S, N, W, n_h, d_c, d_r, d_v, keep_frac, dup)
EDGE = [
    ("window_wider_than_context", 31, 2, 12, 3, 16, 2, 16, 8, 16, 1.0, False),
    ("window_one", 32, 1, 50, 6, 1, 2, 16, 8, 16, 1.0, False),
    ("ragged_tiles", 33, 2, 77, 9, 20, 3, 24, 16, 40, 1.0, False),
    ("duplicate_anchors", 34, 1, 40, 12, 8, 2, 16, 8, 16, 1.0, True),
    ("padding_blocks", 35, 2, 64, 10, 16, 2, 16, 8, 16, 0.5, False),
    ("all_padding", 36, 1, 30, 4, 8, 2, 16, 8, 16, 0.0, False),
    ("no_rope", 37, 1, 40, 5, 9, 2, 32, 0, 16, 1.0, False),
    ("rope_only", 38, 1, 40, 5, 9, 2, 0, 16, 24, 1.0, False),
    ("minimal_context", 39, 1, 2, 2, 4, 1, 8, 8, 8, 1.0, True),
    ("page_dims_small", 40, 1, 300, 20, 128, 2, 192, 64, 256, 1.0, False),
    ("page_dims_dense", 41, 1, 200, 60, 128, 2, 192, 64, 256, 0.9, True),
    ("page_dims_ragged", 42, 2, 133, 7, 128, 1, 192, 64, 256, 1.0, False),
    # three batch rows and 20 heads: the key-major kernels split the heads into
    # groups, so batch-row and head-group indexing is exercised at page dims
    ("page_dims_b3_heads20", 43, 3, 400, 40, 128, 20, 192, 64, 256, 0.85, True),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", EDGE, ids=[e[0] for e in EDGE])
def test_edge_cases_full(oracle_mod, case, dtype):
    name, seed, B, S, N, W, n_h, d_c, d_r, d_v, kf, dup = case
    c = synth.random_case(seed, B, S, N, W, n_h, d_c, d_r, d_v, dtype, keep_frac=kf, allow_dup=dup)
    if S >= 3:
        c["anchors"][0, 0] = 0          # empty context window
        c["anchors"][-1, -1] = S - 2    # last valid anchor
    gpu = run_gpu(c, S, W)
    compare_full(gpu, oracle_full(oracle_mod, c, S, W), synth.torch_dtype(dtype))


@pytest.mark.parametrize("qscale", [3.0, 4.0, 6.0])
def test_large_scores_page_dims(oracle_mod, qscale):
    """Scores with a spread of several units: the running max jumps between
    key tiles, which exercises the online-softmax rescaling of the tensor-core
    forward. Only the forward is compared here: for the backward, an fp64
    emulation of the bf16 pipeline alone (rope key rounded after rotation, O
    rounded before D = rowsum(dO * O), outputs rounded) already exceeds the
    bf16 bound on dK at Q x 3, so the backward is held to the bound on the
    N(0, 1) workloads of the other tests. Beyond Q x 6 the same emulation
    exceeds the bound on O (rotated q and k rope slices are bf16 MMA operands)."""
    c = synth.random_case(45, 1, 400, 30, 128, 2, 192, 64, 256, "bf16")
    c["q"] = (c["q"].float() * qscale).to(torch.bfloat16)
    c["anchors"][0, 0] = 0
    gpu = run_gpu(c, 400, 128, bwd=False)
    compare_full(gpu, oracle_full(oracle_mod, c, 400, 128, bwd=False), torch.bfloat16)


@pytest.mark.parametrize("qscale", [1.5, 2.0])
def test_large_scores_backward_page_dims(oracle_mod, qscale):
    """Where the backward's bf16 bound is claimed to hold beyond N(0, 1)
    queries: every output, gradients included, at Q x 1.5 and Q x 2 (score
    spread 1.5-2x the workloads'). An fp64 emulation of the bf16 roundings
    alone (rope key rounded after rotation, O rounded before D, outputs
    rounded) stays inside the bound on dK^C here (worst excess -0.018 at x1.5,
    -0.009 at x2) and leaves it at x3 (+0.003), which is why the test above
    compares only the forward at x3 and beyond."""
    c = synth.random_case(45, 1, 400, 30, 128, 2, 192, 64, 256, "bf16")
    c["q"] = (c["q"].float() * qscale).to(torch.bfloat16)
    c["anchors"][0, 0] = 0
    gpu = run_gpu(c, 400, 128)
    compare_full(gpu, oracle_full(oracle_mod, c, 400, 128), torch.bfloat16)


def test_no_blocks():
    """N = 0: nothing to attend; the backward still writes zero key gradients."""
    c = synth.random_case(50, 2, 40, 0, 8, 2, 16, 8, 16, "bf16")
    gpu = run_gpu(c, 40, 8)
    assert gpu["o"].numel() == 0 and gpu["dq"].numel() == 0
    for k in ("dkc", "dkr", "dv"):
        assert torch.count_nonzero(gpu[k]) == 0


def test_out_of_range_anchor_is_reported():
    """A kept anchor outside [0, S-2] is reported and its block treated as padding."""
    c = synth.random_case(51, 1, 32, 4, 8, 2, 16, 8, 16, "f32")
    c["anchors"][0, 1] = 31  # S - 1: not a valid anchor
    d = to_dev(c)
    o, lse, ws = capi.attn_fwd(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], 32, 8, BASE)
    with pytest.raises(capi.DsparkError) as e:
        capi.get_error(ws)
    assert e.value.status == 4
    assert torch.count_nonzero(o[0, :, 5:10]) == 0 and torch.isneginf(lse[0, :, 5:10]).all()
    capi.get_error(ws)  # the word was cleared


def test_s2048_workload_full(oracle_mod):
    wl = synth.WORKLOADS[2]
    c = synth.make_inputs(wl)
    gpu = run_gpu(c, wl.S, wl.W)
    compare_full(gpu, oracle_full(oracle_mod, c, wl.S, wl.W), torch.bfloat16)


def test_deterministic():
    """O, LSE, dK^C, dK^R and dV are bitwise reproducible (every element is
    written once, by one thread, in a fixed order). dQ is the sum of one
    contribution per key tile that meets the row's window, added in fp32 in
    whatever order the tiles finish, so two runs may differ by the rounding of
    that sum: at most one bf16 unit in the last place."""
    wl = synth.WORKLOADS[2]
    c = synth.make_inputs(wl)
    a = run_gpu(c, wl.S, wl.W)
    b = run_gpu(c, wl.S, wl.W)
    for k in a:
        if k == "dq":
            x, y = a[k].float(), b[k].float()
            # one bf16 unit of the larger value, plus the fp32 rounding of a sum
            # of O(1) terms where the value itself is near zero
            ulp = torch.maximum(x.abs(), y.abs()) * 2.0 ** -7 + 1e-6
            assert ((x - y).abs() <= ulp).all(), k
        else:
            assert torch.equal(a[k], b[k]), k


def _slice(c, b, h):
    return dict(q=c["q"][b:b + 1, h:h + 1], kc=c["kc"][b:b + 1, h:h + 1], kr=c["kr"][b:b + 1],
                v=c["v"][b:b + 1, h:h + 1], dout=c["dout"][b:b + 1, h:h + 1],
                anchors=c["anchors"][b:b + 1], keep=c["keep"][b:b + 1])


def _np(s):
    return [s[k].double().numpy() for k in ("q", "kc", "kr", "v")]


def _uncovered(an_b, kp_b, S, W):
    """Context positions inside no kept block's window [max(0, A-W+1), A)."""
    cov = np.zeros(S + 1, np.int64)
    a = an_b[kp_b == 1]
    np.add.at(cov, np.maximum(0, a - W + 1), 1)
    np.add.at(cov, a, -1)
    return np.nonzero(np.cumsum(cov)[:S] == 0)[0]


def _sample_keys(rng, an_b, kp_b, S, W, N):
    """Key positions of one batch row to compare: window edges of a sampled
    block, the edge of the lowest window, an uncovered position, the ends of
    the context, random context positions, draft keys of kept blocks and the
    draft keys of a padding block (their gradients must be zero)."""
    kept = np.nonzero(kp_b == 1)[0]
    keys = [0, S - 2, S - 1]
    far = kept[an_b[kept] >= W]
    if far.size:
        a = int(an_b[int(rng.choice(far))])
        keys += [a - 1, a - W + 1, a - W]
    low = int(kept[np.argmin(an_b[kept])])
    if an_b[low] > 0:
        keys.append(int(an_b[low]) - 1)
    unc = _uncovered(an_b, kp_b, S, W)
    if unc.size:
        keys.append(int(rng.choice(unc)))
    keys += [int(x) for x in rng.integers(0, S, 5)]
    for n in rng.choice(kept, 3, replace=False):
        keys.append(S + 5 * int(n) + int(rng.integers(5)))
    keys.append(S + 5 * int(kept[-1]) + 4)
    pads = np.nonzero(kp_b == 0)[0]
    if pads.size:
        n = int(rng.choice(pads))
        keys += [S + 5 * n, S + 5 * n + 4]
    return sorted(set(keys))


# one head of each group of 16 (the key-major kernels split the 64 heads into
# groups), the first and last head of the first group
_KEY_HEADS = (0, 15, 16, 47, 63)


@pytest.mark.parametrize("wid", [3, 4, 5])
def test_full_size_sampled(oracle_mod, wid):
    wl = synth.WORKLOADS[wid]
    c = synth.make_inputs(wl)
    gpu = run_gpu(c, wl.S, wl.W)
    rng = np.random.default_rng(wid)
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    S, W = wl.S, wl.W
    # properties at full size: padding rows are zero / -inf, all finite elsewhere
    pad = np.repeat(kp == 0, 5, axis=1)
    for b in range(wl.B):
        rows = np.nonzero(pad[b])[0]
        if rows.size:
            assert torch.count_nonzero(gpu["o"][b][:, rows]) == 0
            assert torch.isneginf(gpu["lse"][b][:, rows]).all()
            assert torch.count_nonzero(gpu["dq"][b][:, rows]) == 0
    for k in ("o", "dq", "dkc", "dkr", "dv"):
        assert torch.isfinite(gpu[k].float()).all(), k
    # sampled rows: random ones, at least four per batch row (heads in each
    # group), plus the block with the smallest anchor
    picks = []
    for b in range(wl.B):
        for h in rng.choice(_KEY_HEADS, 4, replace=False):
            picks.append((b, int(h), int(rng.integers(5 * wl.N))))
    for _ in range(8):
        picks.append((int(rng.integers(wl.B)), int(rng.integers(wl.n_h)), int(rng.integers(5 * wl.N))))
    b0 = 0
    n_small = int(np.argmin(np.where(kp[b0] == 1, an[b0], 1 << 30)))
    picks += [(b0, 0, 5 * n_small + j) for j in range(5)]
    for b, h, r in picks:
        s = _slice(c, b, h)
        o_ref, lse_ref = oracle_mod.attn_fwd_rows(*_np(s), s["anchors"].numpy(), s["keep"].numpy(), S, W, BASE,
                                                  np.array([[0, 0, r]]))
        assert_close(gpu["o"][b, h, r][None], o_ref, torch.bfloat16, "o[%d,%d,%d]" % (b, h, r))
        assert_close(gpu["lse"][b, h, r][None], lse_ref, torch.bfloat16, "lse")
        dq_ref = oracle_mod.attn_bwd_items(*_np(s), s["anchors"].numpy(), s["keep"].numpy(),
                                           s["dout"].double().numpy(), S, W, BASE, "dq", np.array([[0, 0, r]]))
        assert_close(gpu["dq"][b, h, r][None], dq_ref, torch.bfloat16, "dq[%d,%d,%d]" % (b, h, r))
    # key gradients of every batch row: dK^C and dV at each sampled key for one
    # head of every head group, dK^R (the sum over all heads) at every sampled key
    for b in range(wl.B):
        keys = _sample_keys(rng, an[b], kp[b], S, W, wl.N)
        assert len(keys) >= 16, keys
        items = np.array([[0, 0, k] for k in keys])
        for h in _KEY_HEADS:
            s = _slice(c, b, h)
            ref = oracle_mod.attn_bwd_items(*_np(s), s["anchors"].numpy(), s["keep"].numpy(),
                                            s["dout"].double().numpy(), S, W, BASE, "dkv", items)
            assert_close(gpu["dkc"][b, h, keys], ref[:, :wl.d_c], torch.bfloat16, "dkc[b=%d,h=%d]" % (b, h))
            assert_close(gpu["dv"][b, h, keys], ref[:, wl.d_c:], torch.bfloat16, "dv[b=%d,h=%d]" % (b, h))
        dkr_items = np.array([[0, k] for k in keys])
        tot = np.zeros((len(keys), wl.d_r))
        kr_b = c["kr"][b:b + 1].double().numpy()
        for h in range(wl.n_h):
            s = _slice(c, b, h)
            tot += oracle_mod.attn_bwd_items(s["q"].double().numpy(), s["kc"].double().numpy(), kr_b,
                                             s["v"].double().numpy(), s["anchors"].numpy(), s["keep"].numpy(),
                                             s["dout"].double().numpy(), S, W, BASE, "dkr", dkr_items)
        assert_close(gpu["dkr"][b, keys], tot, torch.bfloat16, "dkr[b=%d]" % b)
        pads = np.nonzero(kp[b] == 0)[0]
        if pads.size:  # draft keys of padding blocks: zero gradients for every head
            pk = (wl.S + 5 * pads[:, None] + np.arange(5)[None]).ravel()
            for k in ("dkc", "dv"):
                assert torch.count_nonzero(gpu[k][b][:, pk]) == 0, k
            assert torch.count_nonzero(gpu["dkr"][b][pk]) == 0
