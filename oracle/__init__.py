"""fp64 CPU oracle for the DSpark draft MLA attention.

TEST INFRASTRUCTURE ONLY. Only the test suite, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg may import this package. The product library
(``speculative_draft_mla_b200``) neither imports it nor shares code with it.

``dspark_oracle.c`` holds the window-form definition (plain C, fp64) and is
compiled on first use (or by ``build()``) into ``_dspark_oracle.so`` next to it.
``dense.py`` holds the dense-mask brute force for tiny sizes.

Parity status: every function here is pinned by tests under ``tests/``
(dense-mask brute force, textbook special cases, invariants, finite
differences); see ``tests/test_oracle_*.py``.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dspark_oracle.c")
_LIB = os.path.join(_HERE, "_dspark_oracle.so")
_lib = None


def build(force=False):
    """Compile the C oracle with gcc (OpenMP over independent units)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        bp = ctypes.POINTER(ctypes.c_uint8)
        dims = [ctypes.c_int] * 8 + [ctypes.c_double]
        lib.oracle_attn_fwd.argtypes = dims + [dp, dp, dp, dp, ip, bp, dp, dp]
        lib.oracle_attn_bwd.argtypes = dims + [dp, dp, dp, dp, ip, bp, dp, dp, dp, dp, dp]
        lib.oracle_attn_fwd_rows.argtypes = dims + [dp, dp, dp, dp, ip, bp, ctypes.c_int, ip, ip, ip, dp, dp]
        lib.oracle_attn_bwd_items.argtypes = dims + [dp, dp, dp, dp, ip, bp, dp, ctypes.c_int, ctypes.c_int,
                                                     ip, ip, ip, dp]
        lib.oracle_anchor_candidates.argtypes = [ctypes.c_int, bp, ip]
        for f in (lib.oracle_attn_fwd, lib.oracle_attn_bwd, lib.oracle_attn_fwd_rows,
                  lib.oracle_attn_bwd_items, lib.oracle_anchor_candidates):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _d(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _i(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _u8(a):
    a = np.ascontiguousarray(a, dtype=np.uint8)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


class OracleError(RuntimeError):
    pass


def _check(rc):
    if rc != 0:
        raise OracleError({-1: "bad size", -2: "kept anchor outside [0, S-2]", -3: "allocation failed"}.get(rc, rc))


def _dims(q, kc, kr, v, anchors, S, W, base):
    B, n_h, R, dqk = q.shape
    N = R // 5
    d_c = kc.shape[-1]
    d_r = kr.shape[-1]
    d_v = v.shape[-1]
    assert R == 5 * N and dqk == d_c + d_r
    assert kc.shape == (B, n_h, S + 5 * N, d_c) and kr.shape == (B, S + 5 * N, d_r)
    assert v.shape == (B, n_h, S + 5 * N, d_v) and np.shape(anchors) == (B, N)
    return B, n_h, N, d_c, d_r, d_v


def attn_fwd(q, kc, kr, v, anchors, keep, S, W, base):
    """O [B,n_h,5N,d_v] and LSE [B,n_h,5N] in fp64 (window form)."""
    B, n_h, N, d_c, d_r, d_v = _dims(q, kc, kr, v, anchors, S, W, base)
    lib = _load()
    q, qp = _d(q); kc, kcp = _d(kc); kr, krp = _d(kr); v, vp = _d(v)
    an, ap = _i(anchors); kp_, kpp = _u8(keep)
    o = np.empty((B, n_h, 5 * N, d_v)); lse = np.empty((B, n_h, 5 * N))
    _check(lib.oracle_attn_fwd(B, n_h, S, N, W, d_c, d_r, d_v, base, qp, kcp, krp, vp, ap, kpp,
                               _d(o)[1], _d(lse)[1]))
    return o, lse


def attn_bwd(q, kc, kr, v, anchors, keep, dout, S, W, base):
    """(dq, dkc, dkr, dv) in fp64 for the loss sum(dout * O)."""
    B, n_h, N, d_c, d_r, d_v = _dims(q, kc, kr, v, anchors, S, W, base)
    lib = _load()
    q, qp = _d(q); kc, kcp = _d(kc); kr, krp = _d(kr); v, vp = _d(v)
    an, ap = _i(anchors); kp_, kpp = _u8(keep); do, dop = _d(dout)
    dq = np.empty_like(q); dkc = np.empty_like(kc); dkr = np.empty_like(kr); dv = np.empty_like(v)
    _check(lib.oracle_attn_bwd(B, n_h, S, N, W, d_c, d_r, d_v, base, qp, kcp, krp, vp, ap, kpp, dop,
                               _d(dq)[1], _d(dkc)[1], _d(dkr)[1], _d(dv)[1]))
    return dq, dkc, dkr, dv


def attn_fwd_rows(q, kc, kr, v, anchors, keep, S, W, base, rows):
    """O and LSE of selected rows; rows is an int array [count, 3] of (b, h, r)."""
    B, n_h, N, d_c, d_r, d_v = _dims(q, kc, kr, v, anchors, S, W, base)
    lib = _load()
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    cnt = rows.shape[0]
    q, qp = _d(q); kc, kcp = _d(kc); kr, krp = _d(kr); v, vp = _d(v)
    an, ap = _i(anchors); kp_, kpp = _u8(keep)
    rb, rbp = _i(rows[:, 0]); rh, rhp = _i(rows[:, 1]); rr, rrp = _i(rows[:, 2])
    o = np.empty((cnt, d_v)); lse = np.empty(cnt)
    _check(lib.oracle_attn_fwd_rows(B, n_h, S, N, W, d_c, d_r, d_v, base, qp, kcp, krp, vp, ap, kpp,
                                    cnt, rbp, rhp, rrp, _d(o)[1], _d(lse)[1]))
    return o, lse


def attn_bwd_items(q, kc, kr, v, anchors, keep, dout, S, W, base, kind, items):
    """Gradients of selected items (gather form).

    kind 'dq':  items (b, h, r)   -> [count, d_c + d_r]
    kind 'dkv': items (b, h, key) -> [count, d_c + d_v]  (dkc then dv)
    kind 'dkr': items (b, key)    -> [count, d_r]        (summed over heads)
    """
    B, n_h, N, d_c, d_r, d_v = _dims(q, kc, kr, v, anchors, S, W, base)
    lib = _load()
    items = np.ascontiguousarray(items, dtype=np.int32)
    cnt = items.shape[0]
    k = {"dq": 0, "dkv": 1, "dkr": 2}[kind]
    if k == 2:
        ib, ih, ix = items[:, 0], np.zeros(cnt, np.int32), items[:, 1]
    else:
        ib, ih, ix = items[:, 0], items[:, 1], items[:, 2]
    width = (d_c + d_r, d_c + d_v, d_r)[k]
    q, qp = _d(q); kc, kcp = _d(kc); kr, krp = _d(kr); v, vp = _d(v)
    an, ap = _i(anchors); kp_, kpp = _u8(keep); do, dop = _d(dout)
    ib, ibp = _i(ib); ih, ihp = _i(ih); ix, ixp = _i(ix)
    out = np.empty((cnt, width))
    _check(lib.oracle_attn_bwd_items(B, n_h, S, N, W, d_c, d_r, d_v, base, qp, kcp, krp, vp, ap, kpp, dop,
                                     k, cnt, ibp, ihp, ixp, _d(out)[1]))
    return out


def anchor_candidates(loss_mask):
    """Valid anchors of page §2 for one sequence, loss_mask[S-1] read as 0."""
    lm, lmp = _u8(loss_mask)
    S = lm.shape[0]
    out = np.empty(max(S, 1), np.int32)
    cnt = _load().oracle_anchor_candidates(S, lmp, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    return out[:cnt].copy()
