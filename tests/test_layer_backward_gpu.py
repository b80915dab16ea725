"""Backward pass of the projections around the merged attention (Eqs. (6) and
(13)) through the C ABI, against the fp64 backward oracle: the output side
(W_V, W_O), the query side (W_Q, W_K), and one whole attention layer composed
on the device (output -> attention -> query) against the oracle's chain.

Error metric: max |g - o| / max |o| over each gradient tensor (per row for the
per-row gradients); 2e-2 for bf16 handles (TF32 products), 1e-3 for fp32."""
import numpy as np
import pytest

from gen import make_workload
from oracle import stca_backward as B
from oracle import stca_oracle as O
from tests.gpu_helpers import TOL, normwise_err, storage_weights, to_device

pytestmark = pytest.mark.gpu


def _rel(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.abs(g - o).max() / max(np.abs(o).max(), 1e-30))


def _dev(a, gpu):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(gpu)


def _wl(dtype, d, h, targets, seed):
    lengths = [40 + 13 * i for i in range(len(targets))]
    return make_workload(lengths=lengths, targets=targets, d=d, h=h, M=2, r=2, dtype=dtype, seed=seed)


@pytest.mark.parametrize("dtype,d,h,layer,targets", [("bf16", 128, 8, 1, [37, 5, 1]),
                                                     ("f32", 64, 2, 0, [3, 0, 9]),
                                                     ("bf16", 256, 16, 0, [130, 2]),
                                                     ("bf16", 64, 4, 1, [1])])
def test_output_backward_matches_oracle(gpu, dtype, d, h, layer, targets):
    import torch
    import target_attention_jagged_b200 as S
    wl = _wl(dtype, d, h, targets, 300 + d)
    rng = np.random.default_rng(d + h)
    C = rng.standard_normal((wl.T, h, d)).astype(np.float32)
    dZ = rng.standard_normal((wl.T, d)).astype(np.float32)
    with S.Stca(storage_weights(wl), d, h, 2, 2, dtype) as st:
        dC, dWv, dWo = S.stca_output_backward(st.handle, layer, _dev(C, gpu), _dev(dZ, gpu), h)
        torch.cuda.synchronize()
        got = [t.cpu().numpy() for t in (dC, dWv, dWo)]
    want = B.output_backward(C, wl.weights["Wv"][layer], wl.weights["Wo"][layer], h, dZ)
    tol = TOL[dtype]
    assert normwise_err(got[0], want[0].reshape(wl.T * h, d)) <= tol
    assert _rel(got[1], want[1]) <= tol and _rel(got[2], want[2]) <= tol


@pytest.mark.parametrize("dtype,d,h,layer,targets", [("bf16", 128, 8, 0, [37, 5, 1]),
                                                     ("f32", 64, 2, 1, [3, 0, 9]),
                                                     ("bf16", 256, 16, 1, [130, 2]),
                                                     ("f32", 128, 4, 0, [1])])
def test_query_backward_matches_oracle(gpu, dtype, d, h, layer, targets):
    import torch
    import target_attention_jagged_b200 as S
    wl = _wl(dtype, d, h, targets, 400 + d)
    rng = np.random.default_rng(d * h)
    Q = rng.standard_normal((wl.T, d)).astype(np.float32)
    dU = rng.standard_normal((wl.T * h, d)).astype(np.float32)
    with S.Stca(storage_weights(wl), d, h, 2, 2, dtype) as st:
        dQ, dWq, dWk = S.stca_query_backward(st.handle, layer, _dev(Q, gpu), _dev(dU, gpu), h)
        torch.cuda.synchronize()
        got = [t.cpu().numpy() for t in (dQ, dWq, dWk)]
    want = B.query_backward(Q, wl.weights["Wq"][layer], wl.weights["Wk"][layer], h, dU.reshape(wl.T, h, d))
    tol = TOL[dtype]
    assert normwise_err(got[0], want[0]) <= tol
    assert _rel(got[1], want[1]) <= tol and _rel(got[2], want[2]) <= tol


def test_projection_backward_empty_batch(gpu):
    import torch
    import target_attention_jagged_b200 as S
    wl = _wl("bf16", 64, 2, [1], 5)
    with S.Stca(storage_weights(wl), 64, 2, 2, 2, "bf16") as st:
        e = torch.empty((0, 64), dtype=torch.float32, device=gpu)
        dC, dWv, dWo = S.stca_output_backward(st.handle, 0, e, e, 2)
        dQ, dWq, dWk = S.stca_query_backward(st.handle, 1, e, e, 2)
        torch.cuda.synchronize()
        assert dC.shape == (0, 64) and dQ.shape == (0, 64)
        for w in (dWv, dWo, dWq, dWk):
            assert torch.count_nonzero(w).item() == 0
        with pytest.raises(S.StcaError):
            S.stca_output_backward(st.handle, 2, e, e, 2)               # no such layer


@pytest.mark.parametrize("dtype,d,h,layer", [("bf16", 128, 8, 1), ("f32", 64, 2, 0)])
def test_attention_layer_chain(gpu, dtype, d, h, layer):
    """One attention layer's backward composed on the device: dZ -> (dC, dWv,
    dWo) -> (dU, dX~) -> (dQ, dWq, dWk), against the oracle's chain on the same
    q, X~ and weights."""
    import torch
    import target_attention_jagged_b200 as S
    lengths, targets = [300, 1, 129, 64], [3, 2, 0, 5]
    wl = make_workload(lengths=lengths, targets=targets, d=d, h=h, M=2, r=2, dtype=dtype, seed=55 + d)
    rng = np.random.default_rng(7 * d)
    Q = rng.standard_normal((wl.T, d)).astype(np.float32)
    dZ = rng.standard_normal((wl.T, d)).astype(np.float32)
    W = wl.weights
    Wq, Wk, Wv, Wo = (np.asarray(W[k][layer], np.float64) for k in ("Wq", "Wk", "Wv", "Wo"))
    dh = d // h
    with S.Stca(storage_weights(wl), d, h, 2, 2, dtype) as st:
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        xt = torch.empty((wl.N, d), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device=gpu)
        S.stca_get_encoded(st.handle, layer, xt)
        torch.cuda.synchronize()
        Xt = xt.float().cpu().numpy().astype(np.float64)
        # the forward's merged rows and attention outputs, from the oracle
        U = np.stack([(Q @ Wq[:, j * dh:(j + 1) * dh]) @ Wk[:, j * dh:(j + 1) * dh].T / np.sqrt(dh)
                      for j in range(h)], axis=1)                       # (T, h, d)
        C = np.zeros_like(U)
        for r in range(len(lengths)):
            t0, t1 = int(wl.target_offsets[r]), int(wl.target_offsets[r + 1])
            k0, k1 = int(wl.offsets[r]), int(wl.offsets[r + 1])
            for j in range(h):
                if t1 > t0:
                    C[t0:t1, j] = O.softmax(U[t0:t1, j] @ Xt[k0:k1].T) @ Xt[k0:k1]
        dC, dWv, dWo = S.stca_output_backward(st.handle, layer, _dev(C, gpu), _dev(dZ, gpu), h)
        dU, dX = S.stca_attention_backward(st.handle, layer, _dev(U.reshape(wl.T * h, d), gpu),
                                           wl.target_offsets, dC, wl.N)
        dQ, dWq, dWk = S.stca_query_backward(st.handle, layer, _dev(Q, gpu), dU, h)
        torch.cuda.synchronize()
        st.status()
        got = {k: v.cpu().numpy() for k, v in dict(dWv=dWv, dWo=dWo, dX=dX, dQ=dQ, dWq=dWq, dWk=dWk).items()}
    w_dC, w_dWv, w_dWo = B.output_backward(C, Wv, Wo, h, dZ)
    w_dU, w_dX = B.attention_backward_batch(U.reshape(wl.T * h, d), Xt, wl.offsets, wl.target_offsets, h,
                                            w_dC.reshape(wl.T * h, d))
    w_dQ, w_dWq, w_dWk = B.query_backward(Q, Wq, Wk, h, w_dU.reshape(wl.T, h, d))
    tol = TOL[dtype]
    for k, want in (("dWv", w_dWv), ("dWo", w_dWo), ("dWq", w_dWq), ("dWk", w_dWk)):
        assert _rel(got[k], want) <= tol, (k, _rel(got[k], want))
    # targets of the one-key request have dQ = 0 exactly (their dU is zero): those
    # rows are held to the tensor's scale, the others per row
    live = np.abs(w_dQ).max(axis=1) > 0
    assert normwise_err(got["dQ"][live], w_dQ[live]) <= tol
    assert np.abs(got["dQ"][~live]).max(initial=0.0) <= tol * np.abs(w_dQ).max()
    keyrows = np.abs(w_dX).max(axis=1) > 0
    assert normwise_err(got["dX"][keyrows], w_dX[keyrows]) <= tol
    assert np.all(got["dX"][~keyrows] == 0)
