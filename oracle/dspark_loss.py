"""Oracle of the DSpark training loss over the draft steps and its gradient.

TEST INFRASTRUCTURE ONLY (see the package docstring): NumPy in fp64, written
from the page "GLM 5.2 DSpark speculative-training design", §6 (training
objective). For draft step r (one row: batch row, block, offset k) with
student logits L (the draft's §5 logits), teacher logits T (the frozen lm_head
on z_{A+k}), label y, confidence logit c (§5 confidence head) and eval_mask m:

  CE_r  = logsumexp(L) - L[y]                                  (coefficient 1)
  L1_r  = || softmax(L) - softmax(T) ||_1                      (coefficient 0.9)
  a_r   = clip(1 - L1_r / 2, 0, 1), with the gradient stopped  (§6 "Confidence")
  BCE_r = BCE-with-logits(c, a_r) = max(c, 0) - c a_r + log(1 + exp(-|c|))
                                                               (coefficient 1)
  loss  = (1 * sum_r m_r CE_r + 0.9 * sum_r m_r L1_r + 1 * sum_r m_r BCE_r) / M,
  M     = sum_r m_r (each term summed over the counted steps, then averaged).

Gradients (teacher logits are constants; a_r is a stop-gradient target):
  d loss / d L_i = (m_r / M) (alpha_ce (p_i - [i = y]) + alpha_l1 p_i (s_i - sum_j s_j p_j)),
      p = softmax(L), q = softmax(T), s = sign(p - q) (sign 0 -> 0),
  d loss / d c   = (m_r / M) alpha_conf (sigmoid(c) - a_r).
Readings: M = 0 gives loss 0 and zero gradients; a label outside [0, V) adds
no CE term (and no CE gradient).

Parity status: pinned by tests/test_oracle_dspark_loss.py (torch's
cross_entropy and binary_cross_entropy_with_logits, L1 special cases and
bounds, central finite differences of the loss with the confidence target
held fixed, masking invariants).
"""
import numpy as np

CE_ALPHA, L1_ALPHA, CONF_ALPHA = 1.0, 0.9, 1.0  # §6 coefficients


def _logsumexp(x):
    m = np.max(x)
    return m + np.log(np.sum(np.exp(x - m)))


def loss_fwd_bwd(L, T, labels, conf, eval_mask, ce_alpha=CE_ALPHA, l1_alpha=L1_ALPHA, conf_alpha=CONF_ALPHA,
                 a_override=None):
    """L, T [R, V]; labels [R] int; conf [R]; eval_mask [R] (0/1).
    a_override: optional [R] confidence targets used instead of a_r (for the
    stop-gradient check). Returns a dict: loss, ce, l1, conf (the three means),
    per-row ce_r, l1_r, bce_r, a_r, grad_logits [R, V], grad_conf [R]."""
    L = np.asarray(L, np.float64)
    T = np.asarray(T, np.float64)
    conf = np.asarray(conf, np.float64)
    m = np.asarray(eval_mask).astype(np.float64)
    R, V = L.shape
    M = m.sum()
    ce_r, l1_r, bce_r, a_r = (np.zeros(R) for _ in range(4))
    grad = np.zeros((R, V))
    grad_c = np.zeros(R)
    for r in range(R):
        y = int(labels[r])
        lse_l = _logsumexp(L[r])
        p = np.exp(L[r] - lse_l)
        q = np.exp(T[r] - _logsumexp(T[r]))
        valid = 0 <= y < V
        ce_r[r] = lse_l - L[r, y] if valid else 0.0
        d = p - q
        l1_r[r] = np.abs(d).sum()
        s = np.sign(d)
        sbar = (s * p).sum()
        a = min(max(1.0 - 0.5 * l1_r[r], 0.0), 1.0) if a_override is None else float(a_override[r])
        a_r[r] = a
        c = conf[r]
        bce_r[r] = max(c, 0.0) - c * a + np.log1p(np.exp(-abs(c)))
        w = m[r] / M if M > 0 else 0.0
        g = l1_alpha * p * (s - sbar)
        if valid:
            g = g + ce_alpha * p
            g[y] -= ce_alpha
        grad[r] = w * g
        grad_c[r] = w * conf_alpha * (1.0 / (1.0 + np.exp(-c)) - a)
    if M > 0:
        ce, l1, cf = (m * ce_r).sum() / M, (m * l1_r).sum() / M, (m * bce_r).sum() / M
    else:
        ce = l1 = cf = 0.0
    return dict(loss=ce_alpha * ce + l1_alpha * l1 + conf_alpha * cf, ce=ce, l1=l1, conf=cf, ce_r=ce_r, l1_r=l1_r,
                bce_r=bce_r, a_r=a_r, grad_logits=grad, grad_conf=grad_c)
