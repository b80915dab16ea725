"""Pins of the backward oracle (oracle/stca_backward.py) against things other
than itself: central finite differences of the fp64 forward (the oracle's own
forward module, pinned elsewhere), PyTorch float64 autograd through library
routines (F.layer_norm, F.silu, torch.softmax), and the invariances of
LayerNorm and softmax.  Planted mistakes must fail at least one pin."""
import numpy as np
import pytest

from oracle import stca_backward as B
from oracle import stca_oracle as O


def _small_weights(rng, d, rd):
    return {"Wu": [rng.standard_normal((d, rd)) / np.sqrt(d)], "Wg": [rng.standard_normal((d, rd)) / np.sqrt(d)],
            "Wd": [rng.standard_normal((rd, d)) / np.sqrt(rd)],
            "ln_g": [rng.uniform(0.5, 1.5, d)], "ln_b": [rng.uniform(-0.5, 0.5, d)]}


def pin_encoder_finite_differences():
    rng = np.random.default_rng(1)
    N, d, rd = 5, 6, 8
    X = rng.standard_normal((N, d))
    W = _small_weights(rng, d, rd)
    G = rng.standard_normal((N, d))
    loss = lambda X_, W_: float((O.encode_history(X_, W_, 0) * G).sum())  # noqa: E731
    g = B.encode_history_backward(X, W, 0, G)
    eps = 1e-6
    for name, arr in [("dX", None), ("dWu", "Wu"), ("dWg", "Wg"), ("dWd", "Wd"),
                      ("dgamma", "ln_g"), ("dbeta", "ln_b")]:
        base = X if arr is None else W[arr][0]
        V = rng.standard_normal(base.shape)
        def shifted(sgn):
            if arr is None:
                return loss(X + sgn * eps * V, W)
            W2 = {k: [v[0].copy()] for k, v in W.items()}
            W2[arr][0] = W2[arr][0] + sgn * eps * V
            return loss(X, W2)
        fd = (shifted(1) - shifted(-1)) / (2 * eps)
        an = float((g[name] * V).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)


def pin_attention_finite_differences():
    rng = np.random.default_rng(2)
    R, L, d = 4, 7, 5
    U = rng.standard_normal((R, d))
    Xt = rng.standard_normal((L, d))
    G = rng.standard_normal((R, d))
    loss = lambda U_, X_: float(((O.softmax(U_ @ X_.T) @ X_) * G).sum())  # noqa: E731
    dU, dX = B.attention_rows_backward(U, Xt, G)
    eps = 1e-6
    for an_grad, which in [(dU, "U"), (dX, "X")]:
        V = rng.standard_normal(an_grad.shape)
        if which == "U":
            fd = (loss(U + eps * V, Xt) - loss(U - eps * V, Xt)) / (2 * eps)
        else:
            fd = (loss(U, Xt + eps * V) - loss(U, Xt - eps * V)) / (2 * eps)
        an = float((an_grad * V).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (which, fd, an)


def pin_torch_autograd():
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F
    rng = np.random.default_rng(3)
    N, d, rd = 9, 8, 16
    X = rng.standard_normal((N, d))
    W = _small_weights(rng, d, rd)
    G = rng.standard_normal((N, d))
    t = {k: torch.tensor(v[0], dtype=torch.float64, requires_grad=True) for k, v in W.items()}
    tx = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    y = ((tx @ t["Wu"]) * F.silu(tx @ t["Wg"])) @ t["Wd"]
    out = F.layer_norm(y, (d,), t["ln_g"], t["ln_b"], eps=1e-5)
    (out * torch.tensor(G)).sum().backward()
    g = B.encode_history_backward(X, W, 0, G)
    for name, ref in [("dX", tx.grad), ("dWu", t["Wu"].grad), ("dWg", t["Wg"].grad),
                      ("dWd", t["Wd"].grad), ("dgamma", t["ln_g"].grad), ("dbeta", t["ln_b"].grad)]:
        np.testing.assert_allclose(g[name], ref.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)
    R, L = 6, 11
    U = torch.tensor(rng.standard_normal((R, d)), requires_grad=True)
    Xt = torch.tensor(rng.standard_normal((L, d)), requires_grad=True)
    Gc = rng.standard_normal((R, d))
    ((torch.softmax(U @ Xt.T, dim=-1) @ Xt) * torch.tensor(Gc)).sum().backward()
    dU, dX = B.attention_rows_backward(U.detach().numpy(), Xt.detach().numpy(), Gc)
    np.testing.assert_allclose(dU, U.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dX, Xt.grad.numpy(), rtol=1e-10, atol=1e-12)


def pin_invariances():
    rng = np.random.default_rng(4)
    N, d, rd = 6, 8, 12
    X = rng.standard_normal((N, d))
    W = _small_weights(rng, d, rd)
    G = rng.standard_normal((N, d))
    g = B.encode_history_backward(X, W, 0, G)
    # LN(y + c 1) = LN(y): the gradient reaching y sums to zero in every row, so
    # dW_d = H^T dy has zero row sums
    assert np.allclose(g["dWd"].sum(axis=1), 0.0, atol=1e-10)
    # adding one vector v to every key shifts each row's scores by u.v (softmax
    # unchanged) and each output c by v: d<C, G>/dv = sum of the key gradients
    R, L = 3, 9
    U = rng.standard_normal((R, d))
    Xt = rng.standard_normal((L, d))
    Gc = rng.standard_normal((R, d))
    dU, dX = B.attention_rows_backward(U, Xt, Gc)
    np.testing.assert_allclose(dX.sum(axis=0), Gc.sum(axis=0), rtol=1e-10, atol=1e-10)
    # scaling every key by (1 + t) scales the scores: along U the derivative is
    # <dU, U> = d/dt <C(U (1 + t)), G> at t = 0, by the chain rule on the scores
    eps = 1e-6
    f = lambda t: float(((O.softmax(U * (1 + t) @ Xt.T) @ Xt) * Gc).sum())  # noqa: E731
    assert abs((f(eps) - f(-eps)) / (2 * eps) - float((dU * U).sum())) < 1e-6


def pin_output_query_finite_differences():
    rng = np.random.default_rng(7)
    T, h, d = 3, 2, 6
    dh = d // h
    C = rng.standard_normal((T, h, d))
    Wv, Wo, Wq, Wk = (rng.standard_normal((d, d)) for _ in range(4))
    Q = rng.standard_normal((T, d))
    dZ = rng.standard_normal((T, d))
    dUg = rng.standard_normal((T, h, d))

    def out(C_, Wv_, Wo_):
        return np.concatenate([C_[:, j] @ Wv_[:, j * dh:(j + 1) * dh] for j in range(h)], -1) @ Wo_

    def uq(Q_, Wq_, Wk_):
        return np.stack([(Q_ @ Wq_[:, j * dh:(j + 1) * dh]) @ Wk_[:, j * dh:(j + 1) * dh].T / np.sqrt(dh)
                         for j in range(h)], axis=1)
    dC, dWv, dWo = B.output_backward(C, Wv, Wo, h, dZ)
    dQ, dWq, dWk = B.query_backward(Q, Wq, Wk, h, dUg)
    eps = 1e-6
    for grad, f, args, i in [(dC, out, [C, Wv, Wo], 0), (dWv, out, [C, Wv, Wo], 1),
                             (dWo, out, [C, Wv, Wo], 2), (dQ, uq, [Q, Wq, Wk], 0),
                             (dWq, uq, [Q, Wq, Wk], 1), (dWk, uq, [Q, Wq, Wk], 2)]:
        G = dZ if f is out else dUg
        V = rng.standard_normal(grad.shape)
        a1 = list(args); a1[i] = a1[i] + eps * V
        a2 = list(args); a2[i] = a2[i] - eps * V
        fd = float(((f(*a1) - f(*a2)) * G).sum()) / (2 * eps)
        assert abs(fd - float((grad * V).sum())) <= 1e-6 * max(1.0, abs(fd)), (f.__name__, i)


def pin_layer_chain():
    """The three pieces composed give the gradient of the forward oracle's
    reordered attention layer (queries, keys and all four projections)."""
    rng = np.random.default_rng(8)
    T, L, h, d = 2, 5, 2, 4
    dh = d // h
    q = rng.standard_normal((T, d))
    Xt = rng.standard_normal((L, d))
    Ws = [rng.standard_normal((d, d)) / np.sqrt(d) for _ in range(4)]
    dZ = rng.standard_normal((T, d))
    Wq, Wk, Wv, Wo = Ws
    U = np.stack([(q @ Wq[:, j * dh:(j + 1) * dh]) @ Wk[:, j * dh:(j + 1) * dh].T / np.sqrt(dh)
                  for j in range(h)], axis=1)                       # (T, h, d), row t h + j
    C = np.stack([O.softmax(U[:, j] @ Xt.T) @ Xt for j in range(h)], axis=1)
    dC, dWv, dWo = B.output_backward(C, Wv, Wo, h, dZ)
    dU, dXt = B.attention_rows_backward(U.reshape(T * h, d), Xt, dC.reshape(T * h, d))
    dq, dWq, dWk = B.query_backward(q, Wq, Wk, h, dU.reshape(T, h, d))
    args = [q, Xt, Wq, Wk, Wv, Wo]
    grads = [dq, dXt, dWq, dWk, dWv, dWo]
    loss = lambda a: float((O.attention_reordered(a[0], a[1], a[2], a[3], a[4], a[5], h) * dZ).sum())  # noqa: E731
    eps = 1e-6
    for i, g in enumerate(grads):
        V = rng.standard_normal(g.shape)
        a1 = list(args); a1[i] = a1[i] + eps * V
        a2 = list(args); a2[i] = a2[i] - eps * V
        fd = (loss(a1) - loss(a2)) / (2 * eps)
        assert abs(fd - float((g * V).sum())) <= 1e-6 * max(1.0, abs(fd)), i


def test_attention_layer_chain_matches_forward_oracle():
    pin_layer_chain()


def _fd_check(loss, args, grads, rng, tag):
    eps = 1e-6
    for i, g in enumerate(grads):
        if g is None:
            continue
        V = rng.standard_normal(np.shape(g))
        a1 = list(args); a1[i] = a1[i] + eps * V
        a2 = list(args); a2[i] = a2[i] - eps * V
        fd = (loss(a1) - loss(a2)) / (2 * eps)
        assert abs(fd - float((np.asarray(g) * V).sum())) <= 1e-6 * max(1.0, abs(fd)), (tag, i)


def _tiny_weights(rng, d, h, M, r):
    from gen import make_workload
    wl = make_workload(lengths=[5], targets=[2], d=d, h=h, M=M, r=r, dtype="f32", seed=int(rng.integers(1 << 30)),
                       random_ln=True, distinct_query_ffn=True)
    return {k: (None if v is None else ([None if a is None else np.asarray(a, np.float64) for a in v]
                                        if isinstance(v, list) else np.asarray(v, np.float64)))
            for k, v in wl.weights.items()}


def pin_fusion_head_query_init():
    """Eq. (7) fusion, Eq. (9) head and Eq. (3) query init against finite
    differences of the forward oracle's query_fusion, prediction_head, query_init."""
    rng = np.random.default_rng(9)
    T, d, h, M, r = 3, 4, 2, 3, 2
    W = _tiny_weights(rng, d, h, M, r)
    outs = [rng.standard_normal((T, d)) for _ in range(M)]
    xt = rng.standard_normal((T, d))
    dy = rng.standard_normal((T, d))
    # fusion into layer 3 (index 2): q^(3) from o^(1), o^(2), x_t
    i = 2
    douts, dxt, dWc, dWu, dWg, dWd = B.fusion_backward(outs[:i], xt, W["Wc"][i], W["qWu"][i], W["qWg"][i],
                                                       W["qWd"][i], dy)

    def fusion_loss(a):
        Wd_ = dict(W)
        Wd_["Wc"] = list(W["Wc"]); Wd_["Wc"][i] = a[3]
        Wd_["qWu"] = list(W["qWu"]); Wd_["qWu"][i] = a[4]
        return float((O.query_fusion([a[0], a[1]], a[2], Wd_, i) * dy).sum())
    _fd_check(fusion_loss, [outs[0], outs[1], xt, W["Wc"][i], W["qWu"][i]],
              [douts[0], douts[1], dxt, dWc, dWu], rng, "fusion")
    # the prediction head over all M outputs
    douts, dxt, dWz, dzu, dzg, dzd = B.fusion_backward(outs, xt, W["Wz"], W["zWu"], W["zWg"], W["zWd"], dy)

    def head_loss(a):
        Wd_ = dict(W, Wz=a[4], zWg=a[5], zWd=a[6])
        return float((O.prediction_head(a[:3], a[3], Wd_) * dy).sum())
    _fd_check(head_loss, outs + [xt, W["Wz"], W["zWg"], W["zWd"]], douts + [dxt, dWz, dzg, dzd], rng, "head")
    # the query init
    g = B.query_init_backward(xt, W, dy)

    def init_loss(a):
        Wd_ = dict(W, q_ln_g=a[1])
        Wd_["qWd"] = list(W["qWd"]); Wd_["qWd"][0] = a[2]
        return float((O.query_init(a[0], Wd_) * dy).sum())
    _fd_check(init_loss, [xt, W["q_ln_g"], W["qWd"][0]], [g["dX"], g["dgamma"], g["dWd"]], rng, "init")


def request_backward(X, xt, W, h, GZ, Gz):
    """Gradient of <Z, GZ> + <z, Gz> for one request, Z of Eq. (8) and z of
    Eq. (9), by chaining the backward pieces from the head down to layer 1.
    Returns dX, dxt and a few weight gradients."""
    M = len(W["Wu"])
    T, d = xt.shape
    dh = d // h
    Xts = [O.encode_history(X, W, i) for i in range(M)]
    qs, Us, Cs, outs = [O.query_init(xt, W)], [], [], []
    for i in range(M):
        q = qs[-1]
        U = np.stack([(q @ W["Wq"][i][:, j * dh:(j + 1) * dh]) @ W["Wk"][i][:, j * dh:(j + 1) * dh].T / np.sqrt(dh)
                      for j in range(h)], axis=1)
        C = np.stack([O.softmax(U[:, j] @ Xts[i].T) @ Xts[i] for j in range(h)], axis=1)
        Us.append(U); Cs.append(C)
        outs.append(O.attention_reordered(q, Xts[i], W["Wq"][i], W["Wk"][i], W["Wv"][i], W["Wo"][i], h))
        if i + 1 < M:
            qs.append(O.query_fusion(outs, xt, W, i + 1))
    douts, dxt, dWz, _, _, _ = B.fusion_backward(outs, xt, W["Wz"], W["zWu"], W["zWg"], W["zWd"], Gz)
    dO = [GZ[:, i] + douts[i] for i in range(M)]
    dX = np.zeros_like(X)
    grads = {"dWz": dWz}
    for i in reversed(range(M)):
        dC, dWv, _ = B.output_backward(Cs[i], W["Wv"][i], W["Wo"][i], h, dO[i])
        dU, dXt = B.attention_rows_backward(Us[i].reshape(T * h, d), Xts[i], dC.reshape(T * h, d))
        dX += B.encode_history_backward(X, W, i, dXt)["dX"]
        dq, dWq, _ = B.query_backward(qs[i], W["Wq"][i], W["Wk"][i], h, dU.reshape(T, h, d))
        grads[f"dWv{i}"], grads[f"dWq{i}"] = dWv, dWq
        if i > 0:
            dprev, dx_i, dWc, _, _, _ = B.fusion_backward(outs[:i], xt, W["Wc"][i], W["qWu"][i], W["qWg"][i],
                                                          W["qWd"][i], dq)
            for k in range(i):
                dO[k] = dO[k] + dprev[k]
            dxt = dxt + dx_i
            grads[f"dWc{i}"] = dWc
        else:
            dxt = dxt + B.query_init_backward(xt, W, dq)["dX"]
    grads["dX"], grads["dxt"] = dX, dxt
    return grads


def pin_request_chain():
    """Every backward piece chained over a whole request (M = 2, with the head)
    against finite differences of the forward oracle's forward_request and
    prediction head."""
    rng = np.random.default_rng(10)
    L, T, d, h, M, r = 5, 2, 4, 2, 2, 2
    W = _tiny_weights(rng, d, h, M, r)
    X = rng.standard_normal((L, d))
    xt = rng.standard_normal((T, d))
    GZ = rng.standard_normal((T, M, d))
    Gz = rng.standard_normal((T, d))
    g = request_backward(X, xt, W, h, GZ, Gz)

    def loss(a):
        Wd_ = dict(W, Wz=a[2])
        for key, idx, pos in (("Wv", 0, 3), ("Wq", 1, 4), ("Wc", 1, 5)):
            Wd_[key] = list(W[key]); Wd_[key][idx] = a[pos]
        Z = O.forward_request(a[0], a[1], Wd_, h)
        z = O.head_from_outputs(Z, a[1], Wd_)
        return float((Z * GZ).sum() + (z * Gz).sum())
    _fd_check(loss, [X, xt, W["Wz"], W["Wv"][0], W["Wq"][1], W["Wc"][1]],
              [g["dX"], g["dxt"], g["dWz"], g["dWv0"], g["dWq1"], g["dWc1"]], rng, "request")


def test_fusion_head_query_init_finite_differences():
    pin_fusion_head_query_init()


def test_request_chain_matches_forward_oracle():
    pin_request_chain()


def test_output_and_query_backward_finite_differences():
    pin_output_query_finite_differences()


def test_encoder_backward_finite_differences():
    pin_encoder_finite_differences()


def test_attention_backward_finite_differences():
    pin_attention_finite_differences()


def test_backward_torch_autograd():
    pin_torch_autograd()


def test_backward_invariances():
    pin_invariances()


def test_attention_batch_matches_per_request():
    rng = np.random.default_rng(5)
    off = np.array([0, 5, 5 + 1, 5 + 1 + 9])
    toff = np.array([0, 2, 2, 3])
    h, d = 2, 4
    U = rng.standard_normal((3 * h, d))
    Xt = rng.standard_normal((15, d))
    dC = rng.standard_normal((3 * h, d))
    dU, dX = B.attention_backward_batch(U, Xt, off, toff, h, dC)
    du0, dx0 = B.attention_rows_backward(U[:4], Xt[:5], dC[:4])
    np.testing.assert_allclose(dU[:4], du0)
    np.testing.assert_allclose(dX[:5], dx0)
    assert np.all(dX[5:6] == 0)                 # request 1 has no targets: no gradient
    du2, dx2 = B.attention_rows_backward(U[4:], Xt[6:], dC[4:])
    np.testing.assert_allclose(dX[6:], dx2)


# ------------------------------------------------------------------ mutations

def _enc_no_mean_term(X, W, i, dXt, eps=1e-5):
    x = np.asarray(X, float)
    Wu, Wg, Wd = (np.asarray(W[k][i], float) for k in ("Wu", "Wg", "Wd"))
    a, g = x @ Wu, x @ Wg
    sg = O.sigmoid(g); s = g * sg; H = a * s; y = H @ Wd
    mu = y.mean(-1, keepdims=True); rstd = 1 / np.sqrt(((y - mu) ** 2).mean(-1, keepdims=True) + eps)
    yh = (y - mu) * rstd
    dyh = dXt * np.asarray(W["ln_g"][i])
    dy = rstd * (dyh - yh * (dyh * yh).mean(-1, keepdims=True))      # mean(dyh) dropped
    dH = dy @ Wd.T; da = dH * s; dg = dH * a * sg * (1 + g * (1 - sg))
    return {"dX": da @ Wu.T + dg @ Wg.T, "dWu": x.T @ da, "dWg": x.T @ dg, "dWd": H.T @ dy,
            "dgamma": (dXt * yh).sum(0), "dbeta": np.asarray(dXt).sum(0)}


def _enc_sigmoid_derivative(X, W, i, dXt, eps=1e-5):
    x = np.asarray(X, float)
    Wu, Wg, Wd = (np.asarray(W[k][i], float) for k in ("Wu", "Wg", "Wd"))
    a, g = x @ Wu, x @ Wg
    sg = O.sigmoid(g); s = g * sg; H = a * s; y = H @ Wd
    mu = y.mean(-1, keepdims=True); rstd = 1 / np.sqrt(((y - mu) ** 2).mean(-1, keepdims=True) + eps)
    yh = (y - mu) * rstd
    dyh = dXt * np.asarray(W["ln_g"][i])
    dy = rstd * (dyh - dyh.mean(-1, keepdims=True) - yh * (dyh * yh).mean(-1, keepdims=True))
    dH = dy @ Wd.T; da = dH * s
    dg = dH * a * sg                                     # d SiLU / dg taken as sigmoid(g)
    return {"dX": da @ Wu.T + dg @ Wg.T, "dWu": x.T @ da, "dWg": x.T @ dg, "dWd": H.T @ dy,
            "dgamma": (dXt * yh).sum(0), "dbeta": np.asarray(dXt).sum(0)}


_output_backward = B.output_backward
_query_backward = B.query_backward
_fusion_backward = B.fusion_backward


def _fusion_xt_first(outs, xt, Wc, Wu, Wg, Wd, dy):
    cat = np.concatenate([np.asarray(xt, np.float64)] + [np.asarray(o, np.float64) for o in outs], axis=-1)
    a = cat @ np.asarray(Wc, np.float64)
    da, dWu, dWg, dWd = B.ffn_backward(a, Wu, Wg, Wd, dy)
    dcat = da @ np.asarray(Wc, np.float64).T
    d = np.asarray(xt).shape[1]
    return ([dcat[:, (k + 1) * d:(k + 2) * d] for k in range(len(outs))], dcat[:, :d], cat.T @ da,
            dWu, dWg, dWd)


def _ffn_silu_term_dropped(x, Wu, Wg, Wd, dy):
    x, Wu, Wg, Wd, dy = (np.asarray(t, np.float64) for t in (x, Wu, Wg, Wd, dy))
    a, g = x @ Wu, x @ Wg
    sg = O.sigmoid(g)
    dH = dy @ Wd.T
    da, dg = dH * g * sg, dH * a * sg            # the g (1 - sigmoid(g)) term dropped
    return da @ Wu.T + dg @ Wg.T, x.T @ da, x.T @ dg, (a * g * sg).T @ dy


def _out_wrong_transpose(C, Wv, Wo, h, dZ):
    dC, dWv, dWo = _output_backward(C, Wv, Wo, h, dZ)
    return dC, dWv, dWo.T                                   # dW_O transposed


def _query_no_scale(Q, Wq, Wk, h, dU):
    dQ, dWq, dWk = _query_backward(Q, Wq, Wk, h, dU)
    d = np.asarray(Q).shape[1]
    return dQ * np.sqrt(d // h), dWq * np.sqrt(d // h), dWk * np.sqrt(d // h)   # 1/sqrt(d_h) dropped


def _attn_sign(U, Xt, dC):
    U, Xt, dC = (np.asarray(a, float) for a in (U, Xt, dC))
    P = O.softmax(U @ Xt.T); dP = dC @ Xt.T
    dS = P * (dP + (P * dP).sum(-1, keepdims=True))        # wrong sign
    return dS @ Xt, P.T @ dC + dS.T @ U


def _attn_no_value_term(U, Xt, dC):
    U, Xt, dC = (np.asarray(a, float) for a in (U, Xt, dC))
    P = O.softmax(U @ Xt.T); dP = dC @ Xt.T
    dS = P * (dP - (P * dP).sum(-1, keepdims=True))
    return dS @ Xt, dS.T @ U                                 # P^T dC dropped


def _attn_transposed(U, Xt, dC):
    U, Xt, dC = (np.asarray(a, float) for a in (U, Xt, dC))
    P = O.softmax(U @ Xt.T); dP = dC @ Xt.T
    dS = P * (dP - (P * dP).sum(-1, keepdims=True))
    return dS @ Xt, P.T @ dC + dS.T @ dC                     # U replaced by dC


MUTANTS = {
    "ln_mean_term_dropped": ("encode_history_backward", _enc_no_mean_term),
    "silu_derivative_wrong": ("encode_history_backward", _enc_sigmoid_derivative),
    "softmax_sign": ("attention_rows_backward", _attn_sign),
    "value_path_dropped": ("attention_rows_backward", _attn_no_value_term),
    "query_replaced": ("attention_rows_backward", _attn_transposed),
    "wo_gradient_transposed": ("output_backward", _out_wrong_transpose),
    "query_scale_dropped": ("query_backward", _query_no_scale),
    "fusion_xt_first": ("fusion_backward", _fusion_xt_first),
    "ffn_silu_term_dropped": ("ffn_backward", _ffn_silu_term_dropped),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(B, attr, fn)
    failed = 0
    for pin in (pin_encoder_finite_differences, pin_attention_finite_differences, pin_torch_autograd,
                pin_invariances, pin_output_query_finite_differences, pin_layer_chain,
                pin_fusion_head_query_init, pin_request_chain):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed, f"mutant {name} passes every pin"
