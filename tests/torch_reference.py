"""The STCA forward assembled from PyTorch library routines in float64 on the CPU.

Used only to pin the oracle: torch.nn.functional.layer_norm, silu and
scaled_dot_product_attention (standard form, one query per target and head,
default 1/sqrt(d_h) scale) stand in for the LayerNorm, the SwiGLU gate and
Eqs. (4)-(5) of the "Make It Long, Keep It Fast" digest §2.1.  Shares no code
with oracle/.
"""
import torch
import torch.nn.functional as F


def _t(a):
    return torch.as_tensor(a, dtype=torch.float64)


def forward_request(X, xt, W, h, eps=1e-5):
    X, xt = _t(X), _t(xt)
    M = len(W["Wu"])
    T, d = xt.shape
    dh = d // h

    def ffn(x, i, query):
        if query and W.get("qWu") is not None:
            wu, wg, wd = W["qWu"][i], W["qWg"][i], W["qWd"][i]
        else:
            wu, wg, wd = W["Wu"][i], W["Wg"][i], W["Wd"][i]
        return ((x @ _t(wu)) * F.silu(x @ _t(wg))) @ _t(wd)

    enc = [F.layer_norm(ffn(X, i, False), (d,), _t(W["ln_g"][i]), _t(W["ln_b"][i]), eps)
           for i in range(M)]
    qg = W["q_ln_g"] if W.get("q_ln_g") is not None else W["ln_g"][0]
    qb = W["q_ln_b"] if W.get("q_ln_b") is not None else W["ln_b"][0]
    q = F.layer_norm(ffn(xt, 0, True), (d,), _t(qg), _t(qb), eps)
    outs = []
    for i in range(M):
        Q = (q @ _t(W["Wq"][i])).view(T, h, dh).transpose(0, 1).unsqueeze(2)   # (h, T, 1, dh)
        K = (enc[i] @ _t(W["Wk"][i])).view(-1, h, dh).transpose(0, 1)          # (h, L, dh)
        V = (enc[i] @ _t(W["Wv"][i])).view(-1, h, dh).transpose(0, 1)
        K = K.unsqueeze(1).expand(h, T, K.shape[1], dh)
        V = V.unsqueeze(1).expand(h, T, V.shape[1], dh)
        o = F.scaled_dot_product_attention(Q, K, V)                             # (h, T, 1, dh)
        o = o.squeeze(2).transpose(0, 1).reshape(T, d) @ _t(W["Wo"][i])
        outs.append(o)
        if i + 1 < M:
            q = ffn(torch.cat(outs + [xt], dim=-1) @ _t(W["Wc"][i + 1]), i + 1, True)
    return torch.stack(outs, dim=1).numpy()


def prediction_head(Z, xt, W):
    """z of Eq. (9) for every target: Z (T, M, d), xt (T, d); F.silu for the gate."""
    Z, xt = _t(Z), _t(xt)
    T, M, d = Z.shape
    cat = torch.cat([Z.reshape(T, M * d), xt], dim=-1)
    y = cat @ _t(W["Wz"])
    return (((y @ _t(W["zWu"])) * F.silu(y @ _t(W["zWg"]))) @ _t(W["zWd"])).numpy()
