"""A second, deliberately naive implementation of the CSA2 decode step in
pure Python (loops, math.exp), for tiny inputs only.

It shares no code with the oracle.  Its job is to catch a dropped term, a
wrong sign or index, or a transposed operand in the oracle.  Selection here
works by repeated maximum extraction, not by sorting.
"""
import math


def score(q, w, key):
    total = 0
    for h in range(len(q)):
        dot = 0
        for d in range(len(key)):
            dot += int(q[h][d]) * int(key[d])
        if dot > 0:
            total += int(w[h]) * dot
    return total


def select(scores_by_pos, k):
    """scores_by_pos: dict position -> score.  Repeatedly take the highest
    score, breaking ties by the lowest position."""
    left = dict(scores_by_pos)
    chosen = []
    while left and len(chosen) < k:
        best = None
        for p, s in left.items():
            if best is None or s > left[best] or (s == left[best] and p < best):
                best = p
        chosen.append(best)
        del left[best]
    return sorted(chosen)


E2M1 = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}


def e4m3(b):
    s = -1.0 if b & 0x80 else 1.0
    e = (b >> 3) & 15
    m = b & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1 + m / 8.0) * 2.0 ** (e - 7)


def dequant_row(code_bytes, scale_bytes, dim):
    out = []
    for j in range(dim):
        byte = code_bytes[j // 2]
        nib = (byte & 15) if j % 2 == 0 else (byte >> 4)
        v = E2M1[nib & 7] * (-1.0 if nib & 8 else 1.0)
        out.append(v * e4m3(scale_bytes[j // 32]))
    return out


def attend(q, rows, scale):
    out = []
    for qh in q:
        logits = [scale * sum(qh[d] * r[d] for d in range(len(r))) for r in rows]
        m = max(logits)
        ws = [math.exp(x - m) for x in logits]
        tot = sum(ws)
        out.append([sum(ws[i] * rows[i][d] for i in range(len(rows))) / tot for d in range(len(q[0]))])
    return out


def decode_step(modes, layers, pos, pool, topk, window):
    """Returns per layer (sel, attn_set, out) for the plan ``modes``."""
    res = []
    pool_set = sel = None
    for mode, L in zip(modes, layers):
        if mode == 0:
            sc = {p: score(L["q"], L["w"], L["keys"][p]) for p in range(pos + 1)}
            pool_set = select(sc, pool)
            sel = select({p: sc[p] for p in pool_set}, topk)
        elif mode == 1:
            sc = {p: score(L["q"], L["w"], L["keys"][p]) for p in pool_set}
            sel = select(sc, topk)
        wstart = max(0, pos - window + 1)
        S = sorted(set(sel) | set(range(wstart, pos + 1)))
        D = len(L["q_attn"][0])
        ring = L.get("local_ring")
        rows = []
        for p in S:
            if ring is not None and p >= wstart:   # the layer's local cache: slot p mod ring length
                rows.append([float(x) for x in ring[p % len(ring)]])
            else:
                rows.append(dequant_row(L["codes"][p], L["scales"][p], D))
        res.append((list(sel), S, attend(L["q_attn"], rows, 1.0 / math.sqrt(D))))
    return res
