"""Brute-force STCA forward in scalar Python, for tiny inputs only.

An independent restatement of the equations used to pin the oracle: it uses
the naive attention form (per-head K and V projections of every token, Eqs.
(4)-(6) of the "Make It Long, Keep It Fast" digest §2.1), explicit scalar loops,
math.exp, and nested lists.  It shares no code with oracle/.
"""
import math


def _col(A, j):
    return [row[j] for row in A]


def _vecmat(x, A):
    """x (n) times A (n x m) -> (m)."""
    n, m = len(A), len(A[0])
    assert len(x) == n
    out = []
    for j in range(m):
        acc = 0.0
        for k in range(n):
            acc += x[k] * A[k][j]
        out.append(acc)
    return out


def _sigmoid(z):
    if z >= 0:
        return 1.0 / (1.0 + math.exp(-z))
    e = math.exp(z)
    return e / (1.0 + e)


def _ffn(x, Wu, Wg, Wd):
    a = _vecmat(x, Wu)
    g = _vecmat(x, Wg)
    hidden = [a[k] * (g[k] * _sigmoid(g[k])) for k in range(len(a))]
    return _vecmat(hidden, Wd)


def _ln(y, gamma, beta, eps=1e-5):
    n = len(y)
    mu = sum(y) / n
    var = sum((v - mu) * (v - mu) for v in y) / n
    s = math.sqrt(var + eps)
    return [(y[k] - mu) / s * gamma[k] + beta[k] for k in range(n)]


def _tolist(a):
    return [[float(v) for v in row] for row in a]


def forward_request(X, xt, W, h):
    """Z (T_r x M x d nested lists) for one request, brute force."""
    X = _tolist(X)
    xt = _tolist(xt)
    M = len(W["Wu"])
    d = len(X[0])
    dh = d // h
    L = len(X)
    mats = ("Wu", "Wg", "Wd", "Wq", "Wk", "Wv", "Wo", "Wc", "qWu", "qWg", "qWd")
    Wl = {k: [None if a is None else _tolist(a) for a in W[k]]
          for k in mats if W.get(k) is not None}
    qffn = (lambda i: (Wl["qWu"][i], Wl["qWg"][i], Wl["qWd"][i])) if "qWu" in Wl else \
        (lambda i: (Wl["Wu"][i], Wl["Wg"][i], Wl["Wd"][i]))
    if W.get("q_ln_g") is not None:
        qg = [float(v) for v in W["q_ln_g"]]
        qb = [float(v) for v in W["q_ln_b"]]
    else:
        qg = [float(v) for v in W["ln_g"][0]]
        qb = [float(v) for v in W["ln_b"][0]]
    enc = []
    for i in range(M):
        g = [float(v) for v in W["ln_g"][i]]
        b = [float(v) for v in W["ln_b"][i]]
        enc.append([_ln(_ffn(x, Wl["Wu"][i], Wl["Wg"][i], Wl["Wd"][i]), g, b) for x in X])
    Z = []
    for x_t in xt:
        q = _ln(_ffn(x_t, *qffn(0)), qg, qb)
        outs = []
        for i in range(M):
            Wq, Wk, Wv, Wo = Wl["Wq"][i], Wl["Wk"][i], Wl["Wv"][i], Wl["Wo"][i]
            concat = []
            for j in range(h):
                cols = range(j * dh, (j + 1) * dh)
                qh = [sum(q[k] * Wq[k][c] for k in range(d)) for c in cols]
                keys = [[sum(x[k] * Wk[k][c] for k in range(d)) for c in cols] for x in enc[i]]
                vals = [[sum(x[k] * Wv[k][c] for k in range(d)) for c in cols] for x in enc[i]]
                s = [sum(qh[c] * keys[l][c] for c in range(dh)) / math.sqrt(dh) for l in range(L)]
                mx = max(s)
                e = [math.exp(v - mx) for v in s]
                tot = sum(e)
                alpha = [v / tot for v in e]
                concat += [sum(alpha[l] * vals[l][c] for l in range(L)) for c in range(dh)]
            o = _vecmat(concat, Wo)
            outs.append(o)
            if i + 1 < M:
                cat = [v for oo in outs for v in oo] + list(x_t)
                q = _ffn(_vecmat(cat, Wl["Wc"][i + 1]), *qffn(i + 1))
        Z.append(outs)
    return Z


def prediction_head(outs, xt, W):
    """z of Eq. (9) for one target: outs = [o(1), ..., o(M)] (lists of d),
    xt (d); the head's FFN weights zWu, zWg, zWd and W_Z ((M+1) d x d)."""
    cat = []
    for o in outs:
        cat += [float(v) for v in o]
    cat += [float(v) for v in xt]
    y = _vecmat(cat, _tolist(W["Wz"]))
    return _ffn(y, _tolist(W["zWu"]), _tolist(W["zWg"]), _tolist(W["zWd"]))
