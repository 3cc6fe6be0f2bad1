"""Seeded synthetic inputs for the DSpark draft attention workloads.

This module only draws random inputs; it holds none of the attention
arithmetic. The test suite feeds the same draws to the CUDA path and to the
fp64 oracle, and the benchmark times the CUDA path on them.

Recipe (one torch CPU generator per workload, seeded 1000 + id, drawn in this
order): loss_mask, anchors, keep, Q, K^C, K^R, V, dO. Tensor values are N(0, 1)
in fp32, then cast to the workload dtype (round to nearest even for bf16).

Workloads follow the synthetic shapes of the DSpark design page (block 5,
W = 128, 64 heads, head dims 192 nope + 64 rope / 256 value):

  id  name                dtype  B  S      N     W    n_h  d_c/d_r/d_v
  1   tiny_f32            f32    1  64     4     16   4    32/16/32
  2   s2048_n128          bf16   1  2048   128   128  64   192/64/256
  3   s8192_n512_b2       bf16   2  8192   512   128  64   192/64/256
  4   s32768_n1024        bf16   1  32768  1024  128  64   192/64/256
  5   s4096_n512_b4_pad   bf16   4  4096   512   128  64   192/64/256

loss_mask: 1 all ones; 2 Bernoulli(0.9); 3 all ones; 4 all ones; 5 Bernoulli(0.8).
For 2, 3 and 5 the last position is then set to 0, as the data loader of the
design page does on read.
Anchors (block order is a random permutation):
  1   uniform without replacement from [0, S-2];
  2,3,5  uniform without replacement among A with loss_mask[A] = loss_mask[A+1] = 1;
  4   A = 0, 15 more from [1, 126] (windows clipped at 0), 1008 from [127, S-2].
keep: all 1, except workload 5 where a seeded 10% of the blocks (N // 10 per
batch row) get keep = 0. If fewer candidates than N exist, the missing blocks
are padding (anchor 0, keep 0).
"""
from dataclasses import dataclass

import torch

BLOCK = 5


@dataclass(frozen=True)
class Workload:
    id: int
    name: str
    dtype: str  # "f32" or "bf16"
    B: int
    S: int
    N: int
    W: int
    n_h: int
    d_c: int
    d_r: int
    d_v: int
    loss_mask: tuple = ("ones",)
    last_zero: bool = False
    anchors: str = "valid"
    drop_frac: float = 0.0
    rope_base: float = 10000.0

    @property
    def L(self):
        return self.S + BLOCK * self.N

    @property
    def rows(self):
        """Query-head rows B * 5N * n_h (padding rows included)."""
        return self.B * BLOCK * self.N * self.n_h

    def with_(self, **kw):
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    1: Workload(1, "tiny_f32", "f32", 1, 64, 4, 16, 4, 32, 16, 32, ("ones",), False, "range"),
    2: Workload(2, "s2048_n128", "bf16", 1, 2048, 128, 128, 64, 192, 64, 256, ("bernoulli", 0.9), True, "valid"),
    3: Workload(3, "s8192_n512_b2", "bf16", 2, 8192, 512, 128, 64, 192, 64, 256, ("ones",), True, "valid"),
    4: Workload(4, "s32768_n1024", "bf16", 1, 32768, 1024, 128, 64, 192, 64, 256, ("ones",), False, "forced_low"),
    5: Workload(5, "s4096_n512_b4_pad", "bf16", 4, 4096, 512, 128, 64, 192, 64, 256, ("bernoulli", 0.8), True,
                "valid", 0.1),
}


def torch_dtype(name):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _draw_loss_mask(wl, g):
    kind = wl.loss_mask[0]
    if kind == "ones":
        lm = torch.ones(wl.B, wl.S, dtype=torch.uint8)
    else:
        lm = (torch.rand(wl.B, wl.S, generator=g) < wl.loss_mask[1]).to(torch.uint8)
    if wl.last_zero:
        lm[:, -1] = 0
    return lm


def _draw_anchors(wl, lm, g):
    anchors = torch.zeros(wl.B, wl.N, dtype=torch.int32)
    keep = torch.zeros(wl.B, wl.N, dtype=torch.uint8)
    for b in range(wl.B):
        if wl.anchors == "range":
            pool = torch.arange(0, wl.S - 1)
        elif wl.anchors == "valid":
            m = lm[b].bool()
            pool = torch.nonzero(m[:-1] & m[1:]).flatten()
        elif wl.anchors == "forced_low":
            low = torch.arange(1, 127)[torch.randperm(126, generator=g)[:15]]
            high_pool = torch.arange(127, wl.S - 1)
            high = high_pool[torch.randperm(high_pool.numel(), generator=g)[:wl.N - 16]]
            pool = torch.cat([torch.zeros(1, dtype=torch.long), low, high])
            pool = pool[torch.randperm(pool.numel(), generator=g)]
            anchors[b] = pool.to(torch.int32)
            keep[b] = 1
            continue
        else:
            raise ValueError(wl.anchors)
        take = min(wl.N, pool.numel())
        sel = pool[torch.randperm(pool.numel(), generator=g)[:take]]
        anchors[b, :take] = sel.to(torch.int32)
        keep[b, :take] = 1
    return anchors, keep


def _draw_keep(wl, keep, g):
    if wl.drop_frac > 0:
        drop = int(wl.N * wl.drop_frac)
        for b in range(wl.B):
            idx = torch.randperm(wl.N, generator=g)[:drop]
            keep[b, idx] = 0
    return keep


def make_inputs(wl, with_grad=True, dtype=None):
    """All inputs of one workload as CPU tensors (dict).

    Keys: loss_mask [B,S] u8, anchors [B,N] i32, keep [B,N] u8,
    q [B,n_h,5N,d_c+d_r], kc [B,n_h,L,d_c], kr [B,L,d_r], v [B,n_h,L,d_v],
    and dout [B,n_h,5N,d_v] when with_grad.
    """
    if isinstance(wl, int):
        wl = WORKLOADS[wl]
    g = torch.Generator().manual_seed(1000 + wl.id)
    dt = torch_dtype(dtype or wl.dtype)
    lm = _draw_loss_mask(wl, g)
    anchors, keep = _draw_anchors(wl, lm, g)
    keep = _draw_keep(wl, keep, g)
    R = BLOCK * wl.N
    out = dict(loss_mask=lm, anchors=anchors, keep=keep)
    out["q"] = torch.randn(wl.B, wl.n_h, R, wl.d_c + wl.d_r, generator=g).to(dt)
    out["kc"] = torch.randn(wl.B, wl.n_h, wl.L, wl.d_c, generator=g).to(dt)
    out["kr"] = torch.randn(wl.B, wl.L, wl.d_r, generator=g).to(dt)
    out["v"] = torch.randn(wl.B, wl.n_h, wl.L, wl.d_v, generator=g).to(dt)
    if with_grad:
        out["dout"] = torch.randn(wl.B, wl.n_h, R, wl.d_v, generator=g).to(dt)
    return out


def random_case(seed, B, S, N, W, n_h, d_c, d_r, d_v, dtype="f32", keep_frac=1.0, anchor_hi=None,
                allow_dup=False):
    """A small random case for edge-case tests: anchors uniform in [0, anchor_hi]
    (default S-2), optionally with duplicates, and keep ~ Bernoulli(keep_frac)."""
    g = torch.Generator().manual_seed(seed)
    hi = S - 2 if anchor_hi is None else anchor_hi
    if allow_dup or N > hi + 1:
        anchors = torch.randint(0, hi + 1, (B, N), generator=g, dtype=torch.int64)
    else:
        anchors = torch.stack([torch.randperm(hi + 1, generator=g)[:N] for _ in range(B)])
    keep = (torch.rand(B, N, generator=g) < keep_frac).to(torch.uint8)
    dt = torch_dtype(dtype)
    R = BLOCK * N
    L = S + BLOCK * N
    return dict(
        anchors=anchors.to(torch.int32), keep=keep,
        q=torch.randn(B, n_h, R, d_c + d_r, generator=g).to(dt),
        kc=torch.randn(B, n_h, L, d_c, generator=g).to(dt),
        kr=torch.randn(B, L, d_r, generator=g).to(dt),
        v=torch.randn(B, n_h, L, d_v, generator=g).to(dt),
        dout=torch.randn(B, n_h, R, d_v, generator=g).to(dt),
    )
