"""Direct triple-loop MLA decode in plain Python floats, for tiny shapes.

Written separately from the oracle (no shared code, no numpy in the
arithmetic) so that the oracle can be checked against it: every sum is a
``math.fsum`` over explicit index loops, straight from the definitions in
"MLA deep compression" (operatorworld.com): latent c = W^DKV h, per-head key
[W^UK_i c || k^R], value W^UV_i c, query [W^Q_i h || RoPE(W^QR_i h)], score =
sum of the content and RoPE dot products, softmax, weighted sum of values.
"""
import math


def _matvec(M, x):
    return [math.fsum(M[r][c] * x[c] for c in range(len(x))) for r in range(len(M))]


def _rotate_pairs(x, pos, base):
    d = len(x)
    y = list(x)
    for k in range(d // 2):
        ang = pos * base ** (-(2.0 * k) / d)
        a, b = x[2 * k], x[2 * k + 1]
        y[2 * k] = a * math.cos(ang) - b * math.sin(ang)
        y[2 * k + 1] = a * math.sin(ang) + b * math.cos(ang)
    return y


def _tolist(a):
    return a.tolist() if hasattr(a, "tolist") else a


def brute_decode(inp, w):
    """Returns {(b, r, i): (o list[d_v], lse float)} for every query row and head."""
    seqlens = [int(x) for x in _tolist(inp["seqlens"])]
    bt = _tolist(inp["block_table"])
    W_Q, W_QR = _tolist(inp["W_Q"]), _tolist(inp["W_QR"])
    W_UK, W_UV = _tolist(inp["W_UK"]), _tolist(inp["W_UV"])
    h_q = _tolist(inp["h_q"])
    qpos = _tolist(inp["qpos"])
    if "cache" in inp:
        cache = _tolist(inp["cache"])

        def row(b, j):
            return cache[bt[b][j // w.page_size] * w.page_size + j % w.page_size]
    else:
        W_DKV, W_KR, h_ctx = _tolist(inp["W_DKV"]), _tolist(inp["W_KR"]), _tolist(inp["h_ctx"])

        def row(b, j):
            h = h_ctx[b][j]
            return _matvec(W_DKV, h) + _rotate_pairs(_matvec(W_KR, h), j, w.rope_base)

    out = {}
    for b in range(w.B):
        L = seqlens[b]
        rows = [row(b, j) for j in range(L)]
        for r in range(w.s_q):
            pos = qpos[b][r]
            h = h_q[b][r]
            for i in range(w.n_h):
                q = _matvec(W_Q[i], h) + _rotate_pairs(_matvec(W_QR[i], h), pos, w.rope_base)
                scores, values = [], []
                for j in range(L):
                    if j > L - w.s_q + r:
                        continue
                    c, kr = rows[j][:w.d_c], rows[j][w.d_c:]
                    k = _matvec(W_UK[i], c) + list(kr)
                    scores.append(w.softmax_scale * math.fsum(q[t] * k[t] for t in range(len(q))))
                    values.append(_matvec(W_UV[i], c))
                mx = max(scores)
                e = [math.exp(s - mx) for s in scores]
                z = math.fsum(e)
                o = [math.fsum(e[j] / z * values[j][v] for j in range(len(e))) for v in range(w.d_v)]
                out[(b, r, i)] = (o, mx + math.log(z))
    return out
