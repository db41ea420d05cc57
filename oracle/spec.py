"""CPU oracle of the MTP draft / verify step -- TEST INFRASTRUCTURE (see __init__.py).

Speculative decoding with a multi-token-prediction head, as the bs178.com
llamAmpere post describes it ("Why it is this fast", part four): a small draft
head proposes the next tokens (depth 3), the main model checks them in one
pass, and each drafted token is kept with probability min(1, p/q), p the main
model's probability of the token and q the draft head's; the draft head's
vocabulary projection covers only the 65,536 tokens of a vocabulary map, while
the main model still chooses from the whole vocabulary.  The post says the
output distribution equals that of plain generation but does not spell out
the step after a rejection; the plain reading that makes that statement true
(the standard speculative-sampling step) is used: at the first rejected
position j the emitted token is drawn from max(0, p_j - q_j) normalised, and
if every draft is kept one more token is drawn from the main model's next
distribution.

Definitions (fp64 throughout):

    dist(l, T)[v]  = exp((l[v] - max l) / T) / sum_w exp((l[w] - max l) / T)    (T > 0)
    sample(w, u)   = the smallest i with sum_{k <= i} w[k] > u * sum_k w[k]   (u in [0, 1))
    draft:  q = dist(z, T) over the mapped rows; row i = sample(q, u); token map[i]
    verify: for j = 0 .. n-1, with d = map[row_j], p = dist(l_j, T) over the
            whole vocabulary, q_j = dist(z_j, T) placed at the mapped tokens
            (0 elsewhere):
              keep d iff u_acc[j] * q_j[d] < p[d]        (probability min(1, p/q))
              else emit sample(max(0, p - q_j), u_res[j]) and stop
            all kept: emit sample(dist(l_n, T), u_bonus)
    T = 0 (greedy): dist is the one-hot of the first maximum; d is kept iff it
    is that maximum, and the emitted correction / bonus is the maximum.

The random numbers are inputs: u = [u_acc (n), u_res (n), u_bonus], each in
[0, 1).  Logits of -inf (masked tokens) have probability 0.
"""
from __future__ import annotations

import numpy as np


def dist(logits: np.ndarray, T: float) -> np.ndarray:
    """Softmax at temperature T > 0, fp64; -inf entries get 0."""
    l = np.asarray(logits, dtype=np.float64)
    m = np.max(l)
    w = np.exp((l - m) / T)
    return w / w.sum()


def sample(weights: np.ndarray, u: float) -> int:
    """Inverse-CDF draw: the smallest i whose running sum exceeds u * total."""
    c = np.cumsum(np.asarray(weights, dtype=np.float64))
    i = int(np.searchsorted(c, u * c[-1], side="right"))
    return min(i, c.size - 1)


def draft(z: np.ndarray, vmap: np.ndarray, T: float, u: float) -> tuple[int, int, float]:
    """One draft token from the mapped logits z: (token, mapped row, q of it)."""
    if T == 0:
        i = int(np.argmax(z))
        return int(vmap[i]), i, 1.0
    q = dist(z, T)
    i = sample(q, u)
    return int(vmap[i]), i, float(q[i])


def verify(target: np.ndarray, drafts: np.ndarray, vmap: np.ndarray, rows: np.ndarray, u: np.ndarray,
           T: float) -> tuple[int, list[int]]:
    """target: [n+1][V] main-model logits of the n drafted positions and the
    next one; drafts: [n][n_map] draft logits; rows: [n] the drafted mapped
    rows; u: [2n+1].  Returns (number of drafts kept, emitted tokens), the
    emitted tokens being the kept drafts and then one correction or bonus."""
    target = np.asarray(target, dtype=np.float64)
    n, V = len(rows), target.shape[1]
    vmap = np.asarray(vmap, dtype=np.int64)
    out: list[int] = []
    for j in range(n):
        d = int(vmap[rows[j]])
        if T == 0:
            best = int(np.argmax(target[j]))
            if d == best:
                out.append(d)
                continue
            out.append(best)
            return j, out
        p = dist(target[j], T)
        q = np.zeros(V)
        q[vmap] = dist(drafts[j], T)
        if u[j] * q[d] < p[d]:
            out.append(d)
            continue
        r = np.maximum(p - q, 0.0)
        out.append(sample(r if r.sum() > 0 else p, u[n + j]))
        return j, out
    out.append(int(np.argmax(target[n])) if T == 0 else sample(dist(target[n], T), u[2 * n]))
    return n, out


def inverse_map(vmap: np.ndarray, V: int) -> np.ndarray:
    """int32 [V]: the mapped row of each token, -1 for tokens outside the map."""
    inv = np.full(V, -1, dtype=np.int32)
    inv[np.asarray(vmap, dtype=np.int64)] = np.arange(len(vmap), dtype=np.int32)
    return inv
