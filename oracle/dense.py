"""Dense-mask brute force for the DSpark draft MLA attention (fp64, NumPy).

TEST INFRASTRUCTURE ONLY: used by the test suite to pin the C oracle. Nothing
in the product imports it.

This is the second, independent formulation the "GLM 5.2 DSpark
speculative-training design" page gives for the same attention (appendix
"Attention implementation", eager/sdpa backend): the boolean mask
M in {0,1}^{5N x (S+5N)} of §3 is materialised densely, and

    O = softmax(Q K^T / sqrt(d) + Lambda(M)) V,   Lambda = 0 where M = 1, -inf where M = 0,

is evaluated with whole-matrix products. Rows whose mask is all zero (padding
blocks, block_keep_mask = 0) give O = 0 and LSE = -inf.

RoPE is written here in complex form: the interleaved pair (x_{2i}, x_{2i+1}) is
the complex number x_{2i} + i x_{2i+1}, multiplied by exp(i * pos * theta_i),
theta_i = base^(-2i/d_r) (page §4 "RoPE", interleaved adjacent pairs). The C
oracle writes the same rotation with explicit cos/sin terms, so the two do not
share a formula transcription.

Small sizes only: the score tensor is n_h x 5N x (S+5N).
"""
import numpy as np

BLOCK = 5  # block_size of page §2


def mask_matrix(S, N, W, anchors, keep):
    """Boolean M [5N, S+5N] of page §3 for one batch element."""
    M = np.zeros((BLOCK * N, S + BLOCK * N), dtype=bool)
    kv = np.arange(S + BLOCK * N)
    for n in range(N):
        if not keep[n]:
            continue  # padding block: its 5 rows see nothing
        a = int(anchors[n])
        ctx = (kv < S) & (kv >= a - W + 1) & (kv < a)  # window A-W+1 <= kv < A
        own = (kv >= S + BLOCK * n) & (kv < S + BLOCK * n + BLOCK)  # own block, bidirectional
        M[BLOCK * n:BLOCK * n + BLOCK, :] = ctx | own
    return M


def position_ids(S, N, anchors):
    """RoPE positions along the KV axis (page §2): 0..S-1, then A_n..A_n+4."""
    pos = np.concatenate([np.arange(S), (np.asarray(anchors)[:, None] + np.arange(BLOCK)[None, :]).reshape(-1)])
    return pos.astype(np.float64)


def rope_complex(x, pos, base):
    """Rotate the last axis of x (even width) by pos (broadcast over leading axes)."""
    d_r = x.shape[-1]
    if d_r == 0:
        return x.copy()
    theta = base ** (-2.0 * np.arange(d_r // 2) / d_r)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * pos[..., None] * theta)
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def dense_forward(q, kc, kr, v, anchors, keep, S, N, W, d_c, d_r, base):
    """Returns (O [B,n_h,5N,d_v], LSE [B,n_h,5N]) in fp64."""
    q = np.asarray(q, np.float64)
    kc = np.asarray(kc, np.float64)
    kr = np.asarray(kr, np.float64)
    v = np.asarray(v, np.float64)
    B, n_h, R, dqk = q.shape
    assert R == BLOCK * N and dqk == d_c + d_r
    d_v = v.shape[-1]
    O = np.zeros((B, n_h, R, d_v))
    LSE = np.full((B, n_h, R), -np.inf)
    scale = 1.0 / np.sqrt(d_c + d_r)
    for b in range(B):
        M = mask_matrix(S, N, W, anchors[b], keep[b])
        pos = position_ids(S, N, anchors[b])
        qpos = pos[S:]  # queries are the draft positions, aligned with the right of KV
        q_rot = np.concatenate([q[b, :, :, :d_c], rope_complex(q[b, :, :, d_c:], qpos, base)], axis=-1)
        k_rope = rope_complex(kr[b], pos, base)  # [L, d_r], one per position
        k_rot = np.concatenate([kc[b], np.broadcast_to(k_rope, (n_h,) + k_rope.shape)], axis=-1)
        scores = np.einsum("hqd,hkd->hqk", q_rot, k_rot) * scale
        scores = np.where(M[None], scores, -np.inf)
        live = M.any(axis=1)
        m = np.where(live[None, :], scores.max(axis=-1), 0.0)
        e = np.exp(scores - m[..., None])
        l = e.sum(axis=-1)
        with np.errstate(divide="ignore", invalid="ignore"):
            P = np.where(live[None, :, None], e / l[..., None], 0.0)
            LSE[b] = np.where(live[None, :], m + np.log(l), -np.inf)
        O[b] = np.einsum("hqk,hkd->hqd", P, v[b])
    return O, LSE
