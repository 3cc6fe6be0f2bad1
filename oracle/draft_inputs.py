"""Oracle of the draft-input step: anchor sampling and the draft block's ids,
positions, labels, Markov-head predecessors and eval_mask.

TEST INFRASTRUCTURE ONLY (see the package docstring): plain Python / NumPy,
slow and obviously correct, written from the page "GLM 5.2 DSpark
speculative-training design", §2 (anchor sampling, draft block), §5 (Markov
head predecessors) and §6 (labels, eval_mask).

Random numbers. The page only says the N anchors are drawn at random from the
valid positions. The GPU sampler draws them by priority sampling with a
counter-based generator, and this oracle implements the same generator from
its published definition: SplitMix64 (Steele, Lea and Flood, OOPSLA 2014),
whose k-th output (k = 0, 1, ...) for seed s is mix(s + (k + 1) * gamma).
Candidate A of batch row b gets the key output_{A}(seed + b); the N candidates
with the smallest (key, A) are kept. Independent continuous keys make every
N-subset equally likely, i.e. a uniform draw without replacement.

Parity status: pinned by tests/test_oracle_draft_inputs.py (the generator's
published first outputs, the page's candidate rule on hand-made masks, a
hand-worked golden fixture for the builder, invariants and a uniformity test).
"""
import numpy as np

MASK_ID = 154821  # the page's MASK token id (§2 "Draft block")
BLOCK = 5         # block_size (§2)
_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def splitmix64_mix(z):
    """SplitMix64's output function (its finaliser) on a 64-bit state."""
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def splitmix64_output(seed, k):
    """k-th output (k >= 0) of SplitMix64 started from state `seed`."""
    return splitmix64_mix((seed + (k + 1) * _GAMMA) & _M64)


def candidates(loss_mask_row):
    """Valid anchors of §2 for one sequence: A in [0, S-2] with
    loss_mask[A] = loss_mask[A+1] = 1, loss_mask[S-1] read as 0 (§6)."""
    lm = [int(x) != 0 for x in loss_mask_row]
    S = len(lm)
    if S:
        lm[S - 1] = False
    return [a for a in range(0, S - 1) if lm[a] and lm[a + 1]]


def sample_anchors(loss_mask, N, seed):
    """Anchors [B, N] int32 (ascending) and keep [B, N] uint8: for each batch
    row b, the min(N, #candidates) candidates with the smallest
    (output_A(seed + b), A), in ascending order of A, then padding blocks
    (anchor 0, keep 0) as §3 prescribes when there are fewer than N."""
    loss_mask = np.asarray(loss_mask)
    B = loss_mask.shape[0]
    anchors = np.zeros((B, N), np.int32)
    keep = np.zeros((B, N), np.uint8)
    for b in range(B):
        cand = candidates(loss_mask[b])
        keyed = sorted((splitmix64_output((seed + b) & _M64, a), a) for a in cand)
        chosen = sorted(a for _, a in keyed[:N])
        anchors[b, :len(chosen)] = chosen
        keep[b, :len(chosen)] = 1
    return anchors, keep


def build_draft_inputs(input_ids, loss_mask, anchors, keep, mask_id=MASK_ID):
    """Per block n with anchor A, offsets j = 0..4 (row 5n + j):
      draft_ids  = x_A at j = 0, MASK at j = 1..4                      (§2)
      position   = A + j (the block's RoPE positions on the KV axis)   (§2)
      label      = y_j = x_{A+j+1}, -1 where A+j+1 >= S                (§6)
      prev       = x_{A+j} (anchor, then the gold tokens), MASK where
                   A+j >= S                                           (§5)
      eval_mask  = prefix product over j of [A+j+1 < S and
                   loss_mask[A+j+1] = 1 (loss_mask[S-1] read as 0) and
                   keep = 1]                                           (§6)
    Positions outside [0, S) (also for an anchor outside the page's range)
    read as MASK (ids, prev) and -1 (labels), and end the eval_mask prefix.
    Returns a dict of [B, 5N] arrays (int32, eval_mask uint8)."""
    x = np.asarray(input_ids)
    lm = np.array(loss_mask, dtype=np.uint8, copy=True)
    B, S = x.shape
    if S:
        lm[:, S - 1] = 0
    N = anchors.shape[1]
    out = {k: np.zeros((B, BLOCK * N), np.int32) for k in ("draft_ids", "position_ids", "labels", "prev_ids")}
    out["eval_mask"] = np.zeros((B, BLOCK * N), np.uint8)

    def inside(p):
        return 0 <= p < S

    for b in range(B):
        for n in range(N):
            A = int(anchors[b, n])
            on = bool(keep[b, n])
            for j in range(BLOCK):
                r = BLOCK * n + j
                out["draft_ids"][b, r] = int(x[b, A]) if j == 0 and inside(A) else mask_id
                out["position_ids"][b, r] = A + j
                out["labels"][b, r] = int(x[b, A + j + 1]) if inside(A + j + 1) else -1
                out["prev_ids"][b, r] = int(x[b, A + j]) if inside(A + j) else mask_id
                step = inside(A + j + 1) and lm[b, A + j + 1] == 1 and keep[b, n] == 1
                on = on and step
                out["eval_mask"][b, r] = 1 if on else 0
    return out
