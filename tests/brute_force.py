"""Scalar pure-Python brute force of one decode step, for tiny caches only.

Written from the definitions, independently of ``oracle/``: explicit loops,
``math.exp``, no NumPy arithmetic.  It is one of the pins of the oracle.
Definitions: attention of the current query over the filled slots and the
new token; score of a slot = its probability averaged over the query heads of
the group (``score="alpha_l1v"``: that average times the sum of the absolute
values of the slot's value vector, the summary page's §2B form);
candidates = slot index >= sink and position older than the last ``window``
positions; lowest score wins, lowest index on ties; a free slot (position
-1) is filled first and then nothing is evicted.
"""
import math


def brute_row(K, V, pos, q, k_new, v_new, sink, window, score="mean_prob"):
    """K, V: lists of N lists of D floats; pos: list of N ints; q: G lists.

    Returns (out [G][D], evicted, slot, t)."""
    N = len(K)
    D = len(k_new)
    G = len(q)
    scale = 1.0 / math.sqrt(D)

    t = 0
    for j in range(N):
        if pos[j] >= 0 and pos[j] + 1 > t:
            t = pos[j] + 1

    probs = []      # probs[i][j] for cached slots (0.0 if empty)
    out = []
    for i in range(G):
        logits = {}
        for j in range(N):
            if pos[j] >= 0:
                acc = 0.0
                for d in range(D):
                    acc += q[i][d] * K[j][d]
                logits[j] = acc * scale
        acc = 0.0
        for d in range(D):
            acc += q[i][d] * k_new[d]
        s_new = acc * scale
        m = s_new
        for j in logits:
            if logits[j] > m:
                m = logits[j]
        w = {j: math.exp(logits[j] - m) for j in logits}
        w_new = math.exp(s_new - m)
        total = w_new
        for j in w:
            total += w[j]
        row_p = [0.0] * N
        for j in w:
            row_p[j] = w[j] / total
        probs.append(row_p)
        o = [0.0] * D
        for d in range(D):
            acc = (w_new / total) * v_new[d]
            for j in w:
                acc += row_p[j] * V[j][d]
            o[d] = acc
        out.append(o)

    for j in range(N):
        if pos[j] < 0:
            return out, -1, j, t

    best = None
    best_score = None
    for j in range(N):
        if j < sink:
            continue
        if pos[j] >= t - window:
            continue
        sc = 0.0
        for i in range(G):
            sc += probs[i][j]
        sc /= G
        if score == "alpha_l1v":
            l1 = 0.0
            for d in range(D):
                l1 += abs(V[j][d])
            sc *= l1
        if best is None or sc < best_score:
            best, best_score = j, sc
    if best is None:
        raise ValueError("no candidate")
    return out, best, best, t
