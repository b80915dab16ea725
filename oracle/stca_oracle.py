"""Plain fp64 CPU oracle of the STCA forward pass -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
legs may import or run this module.  The product path (the CUDA library and its
Python binding) never calls it and shares no code with it.

Sources (the pages this follows):
  [digest]  "Make It Long, Keep It Fast: End-to-End 10k-Sequence Modeling at
            Billion Scale on Douyin" (paper digest), §2.1, Eqs. (1)-(8), (12), (13).
  [blog]    "字节跳动-STCA：抖音 10k 长序列端到端建模的架构、系统与外推三件套"
            (STCA blog), §2.2 (encoding, attention), §2.3 (fusion), §2.4 (reordering),
            §2.5 (request-level batching).

Everything is computed in float64 from the (already bf16- or fp32-valued)
inputs, with no intermediate rounding.  Matrix products use numpy's matmul as
a library primitive; there is no blocking, fusion or reordering beyond what the
equations state.

Readings taken where the pages are silent or garbled:
  O1  Eq. (1) prints W_o twice and gives it shape d x rd.  The blog's prose
      (§2.2) names W_u, W_v in R^{d x rd}, W_o in R^{rd x d} with the gate
      x W_v (.) sigmoid(x W_v).  We use FFN(x) = ((x W_u) (.) SiLU(x W_g)) W_d,
      W_u, W_g: d x rd, W_d: rd x d, SiLU(z) = z * sigmoid(z).
  O2  No biases anywhere (the blog says they are omitted).
  O3  LayerNorm: per-layer affine (gamma, beta), eps = 1e-5, biased variance
      over the d features.
  O4  The M history encodings are independent: X~(i) = LN(FFN^(i)(X)) always
      reads the raw X (Eq. (2)); they are not chained.
  O5  Eq. (3) uses layer 1's FFN and LayerNorm for the query; Eq. (7) uses
      layer (i+1)'s FFN with no LayerNorm.  Separate query-side FFN weights may
      be given; by default they alias the history FFN.
  O6  Scores are divided by sqrt(d_h), d_h = d / h, in both forms (Eqs. (4), (13)).
  O7  Head j uses columns [j d_h, (j+1) d_h) of W_Q, W_K, W_V (each d x d);
      heads are concatenated in order before W_O (Eq. (6)).
  O8  The Eq. (7) concatenation is [o^(1) || ... || o^(i) || x_t] with the raw
      target embedding x_t last.
  O9  No residual connections (none are written).
  O10 A request with an empty history is rejected (softmax over no keys is
      undefined); a request with no targets produces no rows.
  O11 The output per target is Z_H = [o^(1); ...; o^(M)] (Eq. (8)), M x d.
  O12 The prediction-head token z of Eq. (9) is a separate output, computed
      from Z_H and x_t; its SwiGLU FFN has weights of its own (zW_u, zW_g,
      zW_d), not shared with the history or query FFNs.
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence

import numpy as np

LN_EPS = 1e-5


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def sigmoid(z):
    """Logistic function 1 / (1 + exp(-z)), evaluated without overflow."""
    z = _f64(z)
    out = np.empty_like(z)
    pos = z >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-z[pos]))
    ez = np.exp(z[~pos])
    out[~pos] = ez / (1.0 + ez)
    return out


def silu(z):
    """SiLU / Swish gate z * sigmoid(z) ([blog] §2.2, the gate of SwiGLUFFN)."""
    z = _f64(z)
    return z * sigmoid(z)


def swiglu_ffn(x, Wu, Wg, Wd):
    """SwiGLUFFN(x) = ((x W_u) (.) SiLU(x W_g)) W_d -- [digest] Eq. (1), reading O1.

    x: (..., d); W_u, W_g: (d, rd); W_d: (rd, d).  Row-wise, no biases (O2).
    """
    x = _f64(x)
    return ((x @ _f64(Wu)) * silu(x @ _f64(Wg))) @ _f64(Wd)


def layer_norm(y, gamma, beta, eps=LN_EPS):
    """LayerNorm over the last axis with affine (gamma, beta) -- reading O3."""
    y = _f64(y)
    mu = y.mean(axis=-1, keepdims=True)
    var = ((y - mu) ** 2).mean(axis=-1, keepdims=True)
    return (y - mu) / np.sqrt(var + eps) * _f64(gamma) + _f64(beta)


def softmax(s):
    """Exact softmax over the last axis (max-subtracted) -- [blog] §2.2 stresses
    that the attention distribution is exact, not approximated."""
    s = _f64(s)
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# per-layer pieces
# --------------------------------------------------------------------------

def encode_history(X, W, i):
    """X~(i) = LN(SwiGLUFFN^(i)(X)) -- [digest] Eq. (2); independent per layer (O4)."""
    return layer_norm(swiglu_ffn(X, W["Wu"][i], W["Wg"][i], W["Wd"][i]),
                      W["ln_g"][i], W["ln_b"][i])


def _query_ffn(W, i):
    if W.get("qWu") is not None:
        return W["qWu"][i], W["qWg"][i], W["qWd"][i]
    return W["Wu"][i], W["Wg"][i], W["Wd"][i]


def query_init(xt, W):
    """q^(1) = LN(SwiGLUFFN^(1)(x_t)) -- [digest] Eq. (3), reading O5."""
    g = W["q_ln_g"] if W.get("q_ln_g") is not None else W["ln_g"][0]
    b = W["q_ln_b"] if W.get("q_ln_b") is not None else W["ln_b"][0]
    return layer_norm(swiglu_ffn(xt, *_query_ffn(W, 0)), g, b)


def head_cols(d, h, j):
    """Columns of head j in W_Q / W_K / W_V (reading O7)."""
    dh = d // h
    return slice(j * dh, (j + 1) * dh)


def attention_naive(q, Xt, Wq, Wk, Wv, Wo, h):
    """Multi-head single-query cross attention in the standard form.

    For each head j: alpha = softmax((q W_Q^j)(X~ W_K^j)^T / sqrt(d_h)),
    o^j = alpha (X~ W_V^j); o = [o^1 || ... || o^h] W_O.
    [digest] Eqs. (4), (5), (6) and (12).  q: (T, d) -- each row is one target's
    single query, attending to all L rows of Xt: (L, d).  Returns (T, d).
    """
    q, Xt = _f64(q), _f64(Xt)
    d = q.shape[-1]
    dh = d // h
    heads = []
    for j in range(h):
        c = head_cols(d, h, j)
        K = Xt @ _f64(Wk)[:, c]                      # (L, d_h)
        V = Xt @ _f64(Wv)[:, c]                      # (L, d_h)
        alpha = softmax((q @ _f64(Wq)[:, c]) @ K.T / math.sqrt(dh))   # (T, L)
        heads.append(alpha @ V)                      # (T, d_h)
    return np.concatenate(heads, axis=-1) @ _f64(Wo)


def attention_reordered(q, Xt, Wq, Wk, Wv, Wo, h, return_alpha=False):
    """The same attention in the reordered form of [digest] Eq. (13) / [blog] §2.4.

    u^j = (q W_Q^j) W_K^j^T (1 x d), alpha^j = softmax(u^j X~^T / sqrt(d_h)),
    o^j = (alpha^j X~) W_V^j; then the Eq. (6) concat and W_O.
    No L x d_h intermediate is formed.
    """
    q, Xt = _f64(q), _f64(Xt)
    d = q.shape[-1]
    dh = d // h
    heads, alphas = [], []
    for j in range(h):
        c = head_cols(d, h, j)
        u = (q @ _f64(Wq)[:, c]) @ _f64(Wk)[:, c].T  # (T, d)
        alpha = softmax(u @ Xt.T / math.sqrt(dh))    # (T, L)
        ctx = alpha @ Xt                             # (T, d): alpha X~
        heads.append(ctx @ _f64(Wv)[:, c])           # (T, d_h)
        alphas.append(alpha)
    o = np.concatenate(heads, axis=-1) @ _f64(Wo)
    if return_alpha:
        return o, alphas
    return o


def query_fusion(outs: Sequence[np.ndarray], xt, W, i_next):
    """q^(i+1) = SwiGLUFFN^(i+1)([o^(1) || ... || o^(i) || x_t] W_C^(i+1)).

    [digest] Eq. (7); the raw x_t is always the last block (O8), no LayerNorm (O5).
    `i_next` is the 0-based index of layer i+1.
    """
    cat = np.concatenate([_f64(o) for o in outs] + [_f64(xt)], axis=-1)
    return swiglu_ffn(cat @ _f64(W["Wc"][i_next]), *_query_ffn(W, i_next))


def prediction_head(outs: Sequence[np.ndarray], xt, W):
    """z = SwiGLUFFN([o^(1) || ... || o^(M) || x_t] W_Z), W_Z of (M+1)d x d.

    [digest] §2.1 Eq. (9) (the prediction head).  The head's SwiGLU FFN has
    weights of its own, zW_u, zW_g (d x rd) and zW_d (rd x d) (reading O12);
    as in Eq. (7), no LayerNorm (O5) and the raw x_t as the last block (O8).
    """
    cat = np.concatenate([_f64(o) for o in outs] + [_f64(xt)], axis=-1)
    return swiglu_ffn(cat @ _f64(W["Wz"]), _f64(W["zWu"]), _f64(W["zWg"]), _f64(W["zWd"]))


def head_from_outputs(Z, targets, W):
    """z (T, d) of Eq. (9) for every target, from Z (T, M, d) of Eq. (8)."""
    Z = _f64(Z)
    return prediction_head([Z[:, i, :] for i in range(Z.shape[1])], targets, W)


# --------------------------------------------------------------------------
# whole forward
# --------------------------------------------------------------------------

def forward_request(X_r, xt_r, W, h, attention: Optional[Callable] = None):
    """Z for one request: all T_r targets against the shared history X_r.

    The history encodings are computed once and reused by every target
    (request-level batching, [digest] §2.2 / [blog] §2.5).  Returns (T_r, M, d):
    row k is Z_H of target k, [digest] Eq. (8).
    """
    attention = attention or attention_reordered
    X_r, xt_r = _f64(X_r), _f64(xt_r)
    M = len(W["Wu"])
    T_r, d = xt_r.shape
    if X_r.shape[0] == 0:
        raise ValueError("empty history: softmax over no keys is undefined (reading O10)")
    if T_r == 0:
        return np.zeros((0, M, d))
    Xts = [encode_history(X_r, W, i) for i in range(M)]
    q = query_init(xt_r, W)
    outs = []
    for i in range(M):
        outs.append(attention(q, Xts[i], W["Wq"][i], W["Wk"][i], W["Wv"][i], W["Wo"][i], h))
        if i + 1 < M:
            q = query_fusion(outs, xt_r, W, i + 1)
    return np.stack(outs, axis=1)


def forward(X, offsets, targets, target_offsets, W, h, requests=None,
            attention: Optional[Callable] = None):
    """Z (T, M, d) in target order for the jagged batch, or for `requests` only.

    With `requests` given, only those requests' rows are computed; the result
    is then a dict {r: (T_r, M, d)}.
    """
    offsets = np.asarray(offsets, dtype=np.int64)
    target_offsets = np.asarray(target_offsets, dtype=np.int64)
    R = offsets.shape[0] - 1
    M, d = len(W["Wu"]), X.shape[1]
    rs = range(R) if requests is None else requests
    out = {}
    for r in rs:
        lo, hi = int(offsets[r]), int(offsets[r + 1])
        tlo, thi = int(target_offsets[r]), int(target_offsets[r + 1])
        out[r] = forward_request(X[lo:hi], targets[tlo:thi], W, h, attention)
    if requests is not None:
        return out
    T = int(target_offsets[-1])
    Z = np.zeros((T, M, d))
    for r in range(R):
        Z[int(target_offsets[r]):int(target_offsets[r + 1])] = out[r]
    return Z


def forward_workload(wl, requests=None, attention=None):
    """forward() on a gen.Workload."""
    return forward(wl.X, wl.offsets, wl.targets, wl.target_offsets, wl.weights, wl.h,
                   requests=requests, attention=attention)


# --------------------------------------------------------------------------
# algorithmic counts (used by the bench's roofline and pinned by a test)
# --------------------------------------------------------------------------

def attention_length_flops(L, d, h, form):
    """Length-dependent FLOPs of one target's single-query attention, all heads.

    naive (Eq. (12)): per head, projecting all L tokens to K and V
    (2 x 2 L d d_h) plus the scores and the alpha V sum (2 x 2 L d_h).
    reordered (Eq. (13)): per head, the scores u X~^T and the sum alpha X~,
    each over d columns (2 x 2 L d).
    """
    dh = d // h
    if form == "naive":
        return h * (4 * L * d * dh + 4 * L * dh)
    if form == "reordered":
        return h * (4 * L * d)
    raise ValueError(form)


def reordering_saving_factor(d, h):
    """Per-token, per-head cost of forming (X W_K, X W_V) over the cost of the
    weighted reduction alpha X that replaces it -- the blog's §2.4 accounting
    (about 4 L d d_h against 2 L d, a saving of about 2 d_h)."""
    dh = d // h
    return (4 * d * dh) / (2 * d)
