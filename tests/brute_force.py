"""Pure-Python brute force of the layer's definitions, for tiny inputs.

An independent restatement (Python floats and ``math`` only, explicit loops,
no NumPy) used to pin the NumPy oracle: a dropped term, a wrong sign, a wrong
bias row or a transposed operand in either implementation shows up as a
mismatch.  Sources as in ``oracle/hca.py``.
"""

import math


def compress_entry(cand, logits, bias, tokens, bias_rows):
    """One compressed entry: per channel j, softmax over the given tokens of
    logits[r][j] + bias[bias_row][j], then the weighted sum of cand[r][j]."""
    c = len(cand[0])
    out = []
    for j in range(c):
        zs = [logits[r][j] + bias[br][j] for r, br in zip(tokens, bias_rows)]
        zmax = max(zs)
        es = [math.exp(z - zmax) for z in zs]
        tot = sum(es)
        out.append(sum(e / tot * cand[r][j] for e, r in zip(es, tokens)))
    return out


def csa_compress(cand, logits, bias, m):
    T = len(cand)
    out = []
    for i in range(T // m):
        tokens, rows = [], []
        for r in range(i * m - m, i * m + m):      # previous block, then current block
            if 0 <= r < T:
                tokens.append(r)
                rows.append(r - (i * m - m))
        out.append(compress_entry(cand, logits, bias, tokens, rows))
    return out


def hca_compress(cand, logits, bias, m_hca):
    T = len(cand)
    out = []
    for i in range(T // m_hca):
        tokens = list(range(i * m_hca, i * m_hca + m_hca))
        out.append(compress_entry(cand, logits, bias, tokens, list(range(m_hca))))
    return out


def index_score(q_heads, w, key):
    tot = 0.0
    for j in range(len(q_heads)):
        dot = 0.0
        for d in range(len(key)):
            dot += q_heads[j][d] * key[d]
        tot += w[j] * (dot if dot > 0.0 else 0.0)
    return tot


def topk(scores, k):
    return sorted(range(len(scores)), key=lambda s: (-scores[s], s))[:k]


def visible(t, rate, n_entries):
    return [s for s in range(n_entries) if (s + 1) * rate - 1 <= t]


def attend(q_heads, rows, scale):
    out = []
    for qh in q_heads:
        logits = [scale * sum(a * b for a, b in zip(qh, r)) for r in rows]
        mx = max(logits)
        es = [math.exp(x - mx) for x in logits]
        tot = sum(es)
        out.append([sum(es[u] / tot * rows[u][d] for u in range(len(rows))) for d in range(len(qh))])
    return out


def attend_with_sink_row(q_heads, rows, scale, sink):
    """The sink as one more row: logit sink[h] for head h and an all-zero value, in
    an ordinary softmax over U + 1 rows (loops only)."""
    out = []
    for h, qh in enumerate(q_heads):
        logits = [scale * sum(a * b for a, b in zip(qh, r)) for r in rows] + [sink[h]]
        values = [list(r) for r in rows] + [[0.0] * len(qh)]
        mx = max(logits)
        es = [math.exp(x - mx) for x in logits]
        tot = sum(es)
        out.append([sum(es[u] / tot * values[u][d] for u in range(len(values))) for d in range(len(qh))])
    return out
