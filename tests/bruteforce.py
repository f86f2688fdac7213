"""Scalar-loop brute force of GVA decode for tiny inputs (T <= 8).

Written independently of the oracle: plain Python floats, math.cos/sin/exp,
no numpy matmul, content keys built element by element from K_h = V_g(h) M_h
(onedev.kr review, "How it works").  Used only to pin the oracle.
"""
import math


def rope_pairs(x, pos, base):
    d = len(x)
    half = d // 2
    y = list(x)
    for i in range(half):
        theta = base ** (-(2.0 * i) / d)
        a = pos * theta
        c, s = math.cos(a), math.sin(a)
        y[i] = x[i] * c - x[i + half] * s
        y[i + half] = x[i] * s + x[i + half] * c
    return y


def gva_decode_loops(q, M, q_pos, V, KR, offs, lens, d_n, d_r, base):
    """q[b][h][k], M[h][i][k], V[slot][g][i], KR[slot][r]; nested lists or arrays."""
    B = len(q)
    H = len(q[0])
    G = len(V[0])
    d_h = len(V[0][0])
    hpg = H // G
    scale = 1.0 / math.sqrt(d_n + d_r)
    out = [[[0.0] * d_h for _ in range(H)] for _ in range(B)]
    lse = [[-math.inf] * H for _ in range(B)]
    for b in range(B):
        for h in range(H):
            g = h // hpg
            L = int(lens[b])
            if L == 0:
                continue
            qr = rope_pairs([float(q[b][h][d_n + r]) for r in range(d_r)], float(q_pos[b]), base)
            scores = []
            for j in range(L):
                row = int(offs[b]) + j
                s = 0.0
                for k in range(d_n):
                    key = 0.0
                    for i in range(d_h):
                        key += float(V[row][g][i]) * float(M[h][i][k])
                    s += float(q[b][h][k]) * key
                for r in range(d_r):
                    s += qr[r] * float(KR[row][r])
                scores.append(s * scale)
            mx = max(scores)
            w = [math.exp(s - mx) for s in scores]
            z = sum(w)
            for i in range(d_h):
                acc = 0.0
                for j in range(L):
                    acc += w[j] / z * float(V[int(offs[b]) + j][g][i])
                out[b][h][i] = acc
            lse[b][h] = mx + math.log(z)
    return out, lse
