"""Plain fp64 CPU oracle of the backward pass of the pieces of the STCA forward
-- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
legs may import or run this module.  The product path (the CUDA library and its
Python binding) never calls it and shares no code with it.

Sources: "Make It Long, Keep It Fast" digest §2.1, Eqs. (1)-(2) (the history
encoding X~ = LN(SwiGLUFFN(X))), Eq. (3) (the query init), Eq. (13) (the
reordered single-query attention, alpha = softmax(u X~^T), c = alpha X~, with
the projections W_Q, W_K, W_V and W_O of Eq. (6)), Eq. (7) (the W_C fusion) and
Eq. (9) (the prediction head); the STCA blog §2.5 (request-
level batching trains with the history encoded once for all of a request's
targets, so the gradient of X~ sums over every target and head).

Readings (the pages give the forward only):
  B1  The backward is the exact derivative of the forward as this oracle's
      forward module defines it (readings O1-O3 for the encoder: no biases,
      LN with affine (gamma, beta), eps 1e-5, biased variance).
  B2  The loss is synthetic: <output, G> for a given tensor G, so the gradient
      that enters each piece is G itself.  The pages train with BCE on the
      prediction head, which needs labels.
  B3  Attention: a query row is u with its scale already in it (the forward's
      u_j = (q W_Q^j) W_K^j^T / sqrt(d_h)); its output is the merged
      c = softmax(u X~^T) X~ before W_V and W_O.  The backward gives dU and dX~
      for one request's rows against its own keys.

Everything is float64 from the (bf16- or fp32-valued) inputs; matrix products
use numpy's matmul as a library primitive.
"""
from __future__ import annotations

import numpy as np

from .stca_oracle import LN_EPS, sigmoid, softmax


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def encode_history_backward(X, W, i, dXt, eps=LN_EPS):
    """Gradients of <LN(((X W_u) * SiLU(X W_g)) W_d), dXt> (Eqs. (1)-(2), layer i).

    Returns dX (N x d), dWu, dWg (d x rd), dWd (rd x d), dgamma, dbeta (d)."""
    x = _f64(X)
    Wu, Wg, Wd = _f64(W["Wu"][i]), _f64(W["Wg"][i]), _f64(W["Wd"][i])
    gamma = _f64(W["ln_g"][i])
    dxt = _f64(dXt)
    a = x @ Wu                                   # up projection
    g = x @ Wg                                   # gate pre-activation
    sg = sigmoid(g)
    s = g * sg                                   # SiLU(g)
    H = a * s
    y = H @ Wd
    mu = y.mean(axis=-1, keepdims=True)
    var = ((y - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    yh = (y - mu) * rstd                         # normalised, before the affine
    dgamma = (dxt * yh).sum(axis=0)
    dbeta = dxt.sum(axis=0)
    dyh = dxt * gamma
    # LayerNorm: dy = rstd (dyh - mean(dyh) - yh mean(dyh * yh)) over the d features
    dy = rstd * (dyh - dyh.mean(axis=-1, keepdims=True) - yh * (dyh * yh).mean(axis=-1, keepdims=True))
    dWd = H.T @ dy
    dH = dy @ Wd.T
    da = dH * s
    # d SiLU(g) / dg = sigmoid(g) (1 + g (1 - sigmoid(g)))
    dg = dH * a * sg * (1.0 + g * (1.0 - sg))
    dWu = x.T @ da
    dWg = x.T @ dg
    dX = da @ Wu.T + dg @ Wg.T
    return {"dX": dX, "dWu": dWu, "dWg": dWg, "dWd": dWd, "dgamma": dgamma, "dbeta": dbeta}


def attention_rows_backward(U, Xt, dC):
    """Gradients of <softmax(U X~^T) X~, dC> for one request (Eq. (13), reading B3).

    U: (R, d) query rows, Xt: (L, d) keys (the encoded history), dC: (R, d).
    With P = softmax(U X~^T) and C = P X~:
      dP = dC X~^T,  dS = P (dP - rowsum(P dP)),  dU = dS X~,  dX~ = P^T dC + dS^T U."""
    U, Xt, dC = _f64(U), _f64(Xt), _f64(dC)
    P = softmax(U @ Xt.T)
    dP = dC @ Xt.T
    dS = P * (dP - (P * dP).sum(axis=-1, keepdims=True))
    return dS @ Xt, P.T @ dC + dS.T @ U


def attention_backward_batch(U, Xt, offsets, target_offsets, h, dC):
    """attention_rows_backward over a jagged batch: request r's rows are the
    T_r h rows of U starting at target_offsets[r] * h, its keys rows
    offsets[r] .. offsets[r+1]-1 of X~.  Returns dU (T h x d) and dX~ (N x d)."""
    U, Xt, dC = _f64(U), _f64(Xt), _f64(dC)
    dU = np.zeros_like(U)
    dX = np.zeros_like(Xt)
    for r in range(len(offsets) - 1):
        q0, q1 = int(target_offsets[r]) * h, int(target_offsets[r + 1]) * h
        k0, k1 = int(offsets[r]), int(offsets[r + 1])
        if q1 == q0:
            continue
        du, dx = attention_rows_backward(U[q0:q1], Xt[k0:k1], dC[q0:q1])
        dU[q0:q1] = du
        dX[k0:k1] = dx
    return dU, dX


def output_backward(C, Wv, Wo, h, dZ):
    """Gradients of <o, dZ> with o = [c_1 W_V^1 || ... || c_h W_V^h] W_O (Eqs. (6), (13)).

    C: (T, h, d) merged rows c_j (row t h + j of the attention output), W_V, W_O:
    (d, d), head j on columns [j d_h, (j+1) d_h) of W_V (reading O7).  Returns
    dC (T, h, d), dWv, dWo (d, d)."""
    C, Wv, Wo, dZ = _f64(C), _f64(Wv), _f64(Wo), _f64(dZ)
    T, hh, d = C.shape
    dh = d // h
    Oh = np.concatenate([C[:, j, :] @ Wv[:, j * dh:(j + 1) * dh] for j in range(h)], axis=-1)
    dOh = dZ @ Wo.T
    dWo = Oh.T @ dZ
    dC = np.stack([dOh[:, j * dh:(j + 1) * dh] @ Wv[:, j * dh:(j + 1) * dh].T for j in range(h)], axis=1)
    dWv = np.concatenate([C[:, j, :].T @ dOh[:, j * dh:(j + 1) * dh] for j in range(h)], axis=-1)
    return dC, dWv, dWo


def query_backward(Q, Wq, Wk, h, dU):
    """Gradients of <U, dU> with u_j = (q W_Q^j) W_K^j^T / sqrt(d_h) (Eq. (13)).

    Q: (T, d) query vectors q, dU: (T, h, d).  Returns dQ (T, d), dWq, dWk (d, d)."""
    Q, Wq, Wk, dU = _f64(Q), _f64(Wq), _f64(Wk), _f64(dU)
    T, d = Q.shape
    dh = d // h
    s = 1.0 / np.sqrt(dh)
    P = Q @ Wq                                             # (T, d): heads' q W_Q^j side by side
    dP = np.concatenate([s * dU[:, j, :] @ Wk[:, j * dh:(j + 1) * dh] for j in range(h)], axis=-1)
    dWk = np.concatenate([s * dU[:, j, :].T @ P[:, j * dh:(j + 1) * dh] for j in range(h)], axis=-1)
    return dP @ Wq.T, Q.T @ dP, dWk


def ffn_backward(x, Wu, Wg, Wd, dy):
    """Gradients of <((x W_u) * SiLU(x W_g)) W_d, dy>: the SwiGLU FFN with no
    LayerNorm (Eq. (1) as Eqs. (7) and (9) use it).  Returns dx, dWu, dWg, dWd."""
    x, Wu, Wg, Wd, dy = _f64(x), _f64(Wu), _f64(Wg), _f64(Wd), _f64(dy)
    a = x @ Wu
    g = x @ Wg
    sg = sigmoid(g)
    H = a * (g * sg)
    dH = dy @ Wd.T
    da = dH * (g * sg)
    dg = dH * a * sg * (1.0 + g * (1.0 - sg))
    return da @ Wu.T + dg @ Wg.T, x.T @ da, x.T @ dg, H.T @ dy


def fusion_backward(outs, xt, Wc, Wu, Wg, Wd, dy):
    """Gradients of <SwiGLUFFN([o^(1) || ... || o^(i) || x_t] W_C), dy>.

    Eq. (7) (W_C of layer i+1 and that layer's query FFN) and Eq. (9) (W_Z
    and the head's FFN) have this form, x_t the last block (reading O8).
    Returns (douts: list of (T, d), dxt, dWc, dWu, dWg, dWd)."""
    outs = [_f64(o) for o in outs]
    cat = np.concatenate(outs + [_f64(xt)], axis=-1)
    a = cat @ _f64(Wc)
    da, dWu, dWg, dWd = ffn_backward(a, Wu, Wg, Wd, dy)
    dcat = da @ _f64(Wc).T
    d = outs[0].shape[1] if outs else _f64(xt).shape[1]
    douts = [dcat[:, k * d:(k + 1) * d] for k in range(len(outs))]
    return douts, dcat[:, len(outs) * d:], cat.T @ da, dWu, dWg, dWd


def query_init_backward(xt, W, dq):
    """Gradients of <q^(1), dq> with q^(1) = LN(SwiGLUFFN^(1)(x_t)) (Eq. (3),
    reading O5: the query FFN and query LayerNorm weights, which default to
    layer 1's).  Returns the encode_history_backward dict (dX is dx_t)."""
    q = {"Wu": [W["qWu"][0] if W.get("qWu") is not None else W["Wu"][0]],
         "Wg": [W["qWg"][0] if W.get("qWg") is not None else W["Wg"][0]],
         "Wd": [W["qWd"][0] if W.get("qWd") is not None else W["Wd"][0]],
         "ln_g": [W["q_ln_g"] if W.get("q_ln_g") is not None else W["ln_g"][0]]}
    return encode_history_backward(xt, q, 0, dq)
