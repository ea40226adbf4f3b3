"""Pure-Python brute force (math module, explicit loops) for tiny cases.

Written independently of the oracle: no numpy arithmetic, no shared helpers.
Used only to pin the oracle on inputs small enough for loops.
"""

import math


def softmax_attention(q, keys, values, scale):
    """q: list[D]; keys, values: list[L][D]. Textbook softmax attention."""
    scores = []
    for k in keys:
        s = 0.0
        for qi, ki in zip(q, k):
            s += qi * ki
        scores.append(s * scale)
    top = max(scores)
    ws = [math.exp(s - top) for s in scores]
    tot = math.fsum(ws)
    out = [0.0] * len(values[0])
    for w, v in zip(ws, values):
        for d in range(len(v)):
            out[d] += (w / tot) * v[d]
    return out


def dual_decode(q1, q2raw, a, kc, vc, table, seqlens, block_size, Hq, Hkv):
    """Nested lists in, nested lists out: (o1, o2) [B][Hq][D]."""
    G = Hq // Hkv
    B = len(q1)
    D = len(q1[0][0])
    scale = 1.0 / math.sqrt(D)
    o1, o2 = [], []
    for b in range(B):
        r1, r2 = [], []
        for h in range(Hq):
            g = h // G
            keys, vals = [], []
            for j in range(seqlens[b]):
                page = table[b][j // block_size]
                keys.append(list(kc[page][g][j % block_size]))
                vals.append(list(vc[page][g][j % block_size]))
            q2 = [q2raw[b][h][d] + a[h][d] * q1[b][h][d] for d in range(D)]
            r1.append(softmax_attention(q1[b][h], keys, vals, scale))
            r2.append(softmax_attention(q2, keys, vals, scale))
        o1.append(r1)
        o2.append(r2)
    return o1, o2


def matmul_nt(x, w):
    """x [M][K], w [N][K] -> x w^T as nested lists."""
    return [[math.fsum(xi * wi for xi, wi in zip(row, wrow)) for wrow in w] for row in x]


def causal_prefill(q_rows, keys, values, ctx, scale):
    """q_rows: list[n][D] queries of positions ctx .. ctx+n-1; keys, values:
    list[ctx+n][D] in position order. Row i attends to keys 0..ctx+i."""
    out = []
    for i, q in enumerate(q_rows):
        stop = ctx + i + 1
        out.append(softmax_attention(q, keys[:stop], values[:stop], scale))
    return out
