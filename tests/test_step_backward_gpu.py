"""Backward of the per-target step's query side through the C ABI, against the
fp64 backward oracle: the Eq. (7) fusion blocks and the Eq. (9) head
(stca_fusion_backward), the Eq. (3) query init (stca_query_init_backward), and
every backward piece chained on the device over a jagged batch against the
oracle's whole-request chain (itself pinned by finite differences of the
forward oracle).

Error metric: max |g - o| / max |o| per gradient tensor (per row for per-row
gradients); 2e-2 for bf16 handles (TF32 products), 1e-3 for fp32 handles."""
import numpy as np
import pytest

from gen import make_workload
from oracle import stca_backward as B
from oracle import stca_oracle as O
from tests.gpu_helpers import TOL, normwise_err, storage_weights, to_device
from tests.test_backward_pins import request_backward

pytestmark = pytest.mark.gpu


def _rel(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.abs(g - o).max() / max(np.abs(o).max(), 1e-30))


def _dev(a, gpu):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(gpu)


def _w64(W):
    return {k: (None if v is None else ([None if a is None else np.asarray(a, np.float64) for a in v]
                                        if isinstance(v, list) else np.asarray(v, np.float64)))
            for k, v in W.items()}


@pytest.mark.parametrize("dtype,d,M,r,block,distinct", [("bf16", 128, 3, 2, 1, False),
                                                        ("f32", 64, 3, 2, 2, True),
                                                        ("bf16", 128, 2, 4, 2, False),
                                                        ("f32", 64, 2, 2, 2, True),
                                                        ("bf16", 256, 4, 2, 3, True)])
def test_fusion_backward_matches_oracle(gpu, dtype, d, M, r, block, distinct):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[30, 17, 5], targets=[37, 0, 6], d=d, h=4, M=M, r=r, dtype=dtype,
                       seed=600 + d + block, distinct_query_ffn=distinct)
    W = _w64(wl.weights)
    rng = np.random.default_rng(d * M + block)
    Z = rng.standard_normal((wl.T, M, d)).astype(np.float32)
    dy = rng.standard_normal((wl.T, d)).astype(np.float32)
    pre_Z = rng.standard_normal((wl.T, M, d)).astype(np.float32)
    pre_x = rng.standard_normal((wl.T, d)).astype(np.float32)
    head = block == M
    with S.Stca(storage_weights(wl), d, 4, r, M, dtype) as st:
        xt = to_device(wl, wl.targets, gpu)
        g = S.stca_fusion_backward(st.handle, block, _dev(Z, gpu), xt, _dev(dy, gpu), r * d)
        acc = S.stca_fusion_backward(st.handle, block, _dev(Z, gpu), xt, _dev(dy, gpu), r * d,
                                     dZ=_dev(pre_Z, gpu), dxt=_dev(pre_x, gpu), accumulate=True)
        torch.cuda.synchronize()
        got = {k: v.cpu().numpy() for k, v in g.items()}
        got_acc = {k: acc[k].cpu().numpy() for k in ("dZ", "dxt")}
    outs = [Z[:, k].astype(np.float64) for k in range(block)]
    if head:
        want = B.fusion_backward(outs, wl.targets, W["Wz"], W["zWu"], W["zWg"], W["zWd"], dy)
    else:
        q = "q" if distinct else ""
        want = B.fusion_backward(outs, wl.targets, W["Wc"][block], W[q + "Wu"][block], W[q + "Wg"][block],
                                 W[q + "Wd"][block], dy)
    douts, dxt, dW, dWu, dWg, dWd = want
    tol = TOL[dtype]
    want_dZ = np.stack(douts, axis=1)                       # (T, block, d)
    assert normwise_err(got["dZ"][:, :block].reshape(-1, d), want_dZ.reshape(-1, d)) <= tol
    assert np.all(got["dZ"][:, block:] == 0)                # columns of later layers untouched
    assert normwise_err(got["dxt"], dxt) <= tol
    for k, w in (("dW", dW), ("dWu", dWu), ("dWg", dWg), ("dWd", dWd)):
        assert _rel(got[k], w) <= tol, (k, _rel(got[k], w))
    # accumulate: added to what was there; other columns keep their values
    # (an overwrite would miss by the size of what was there, O(1) here)
    added = (got_acc["dZ"][:, :block] - pre_Z[:, :block]).reshape(-1, d)
    assert normwise_err(added, want_dZ.reshape(-1, d)) <= tol
    assert np.all(got_acc["dZ"][:, block:] == pre_Z[:, block:])
    assert normwise_err(got_acc["dxt"] - pre_x, dxt) <= tol


@pytest.mark.parametrize("dtype,d,r,distinct", [("bf16", 128, 4, False), ("f32", 64, 2, True),
                                                ("bf16", 256, 2, True)])
def test_query_init_backward_matches_oracle(gpu, dtype, d, r, distinct):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[20, 9], targets=[150, 3], d=d, h=4, M=2, r=r, dtype=dtype, seed=700 + d,
                       random_ln=True, distinct_query_ffn=distinct)
    dq = np.random.default_rng(d + r).standard_normal((wl.T, d)).astype(np.float32)
    with S.Stca(storage_weights(wl), d, 4, r, 2, dtype) as st:
        g = S.stca_query_init_backward(st.handle, to_device(wl, wl.targets, gpu), _dev(dq, gpu), r * d)
        torch.cuda.synchronize()
        got = {k: v.cpu().numpy() for k, v in g.items()}
    want = B.query_init_backward(wl.targets, _w64(wl.weights), dq)
    tol = TOL[dtype]
    assert normwise_err(got["dxt"], want["dX"]) <= tol
    for k in ("dWu", "dWg", "dWd", "dgamma", "dbeta"):
        assert _rel(got[k], want[k]) <= tol, (k, _rel(got[k], want[k]))


def test_fusion_backward_rejects_bad_blocks(gpu):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[20], targets=[2], d=64, h=2, M=2, r=2, dtype="bf16", seed=3)
    Z = torch.zeros((2, 2, 64), dtype=torch.float32, device=gpu)
    dy = torch.zeros((2, 64), dtype=torch.float32, device=gpu)
    xt = to_device(wl, wl.targets, gpu)
    with S.Stca(storage_weights(wl), 64, 2, 2, 2, "bf16") as st:
        for block in (0, 3):
            with pytest.raises(S.StcaError):
                S.stca_fusion_backward(st.handle, block, Z, xt, dy, 128)
        S.stca_fusion_backward(st.handle, 1, Z, xt, dy, 128)
    sw = storage_weights(wl)
    for k in ("Wz", "zWu", "zWg", "zWd"):
        sw[k] = None
    with S.Stca(sw, 64, 2, 2, 2, "bf16") as st:
        with pytest.raises(S.StcaError) as e:                 # block M is the head: no head weights
            S.stca_fusion_backward(st.handle, 2, Z, xt, dy, 128)
        assert "head" in str(e.value)
        empty = torch.zeros((0, 2, 64), dtype=torch.float32, device=gpu)
        g = S.stca_fusion_backward(st.handle, 1, empty, xt[:0], dy[:0], 128)
        torch.cuda.synchronize()
        assert torch.count_nonzero(g["dW"]).item() == 0


def _forward_intermediates(X, xt, W, h):
    """q^(i), the merged rows U_i (T, h, d), C_i (T, h, d) and o^(i) for one
    request, from the forward oracle."""
    M = len(W["Wu"])
    d = xt.shape[1]
    dh = d // h
    Xts = [O.encode_history(X, W, i) for i in range(M)]
    qs, Us, Cs, outs = [O.query_init(xt, W)], [], [], []
    for i in range(M):
        q = qs[-1]
        U = np.stack([(q @ W["Wq"][i][:, j * dh:(j + 1) * dh]) @ W["Wk"][i][:, j * dh:(j + 1) * dh].T / np.sqrt(dh)
                      for j in range(h)], axis=1)
        C = np.stack([O.softmax(U[:, j] @ Xts[i].T) @ Xts[i] for j in range(h)], axis=1)
        Us.append(U)
        Cs.append(C)
        outs.append(O.attention_reordered(q, Xts[i], W["Wq"][i], W["Wk"][i], W["Wv"][i], W["Wo"][i], h))
        if i + 1 < M:
            qs.append(O.query_fusion(outs, xt, W, i + 1))
    return qs, Us, Cs, np.stack(outs, axis=1)


@pytest.mark.parametrize("dtype,d,h,r", [("f32", 64, 2, 2), ("bf16", 128, 4, 2)])
def test_request_chain_on_device(gpu, dtype, d, h, r):
    """The whole backward of Z (Eq. (8)) and z (Eq. (9)) under <Z, GZ> + <z, Gz>,
    chained on the device piece by piece from the head down to layer 1, with
    the forward's intermediates taken from the forward oracle."""
    import torch
    import target_attention_jagged_b200 as S
    M = 2
    lengths, targets = [90, 7, 33], [2, 3, 1]
    wl = make_workload(lengths=lengths, targets=targets, d=d, h=h, M=M, r=r, dtype=dtype, seed=808 + d,
                       random_ln=True, distinct_query_ffn=True)
    W = _w64(wl.weights)
    T, N = wl.T, wl.N
    rng = np.random.default_rng(d)
    GZ = rng.standard_normal((T, M, d))
    Gz = rng.standard_normal((T, d))
    qs = [np.zeros((T, d)) for _ in range(M)]
    Us = [np.zeros((T, h, d)) for _ in range(M)]
    Cs = [np.zeros((T, h, d)) for _ in range(M)]
    Z = np.zeros((T, M, d))
    want = {"dX": np.zeros((N, d)), "dxt": np.zeros((T, d))}
    for rq in range(len(lengths)):
        k0, k1 = int(wl.offsets[rq]), int(wl.offsets[rq + 1])
        t0, t1 = int(wl.target_offsets[rq]), int(wl.target_offsets[rq + 1])
        X_r, xt_r = np.asarray(wl.X[k0:k1], np.float64), np.asarray(wl.targets[t0:t1], np.float64)
        q_r, U_r, C_r, Z_r = _forward_intermediates(X_r, xt_r, W, h)
        for i in range(M):
            qs[i][t0:t1], Us[i][t0:t1], Cs[i][t0:t1] = q_r[i], U_r[i], C_r[i]
        Z[t0:t1] = Z_r
        g = request_backward(X_r, xt_r, W, h, GZ[t0:t1], Gz[t0:t1])
        want["dX"][k0:k1] = g["dX"]
        want["dxt"][t0:t1] = g["dxt"]
        for k in ("dWz", "dWv0", "dWq1", "dWc1"):
            want[k] = want.get(k, 0) + g[k]
    with S.Stca(storage_weights(wl), d, h, r, M, dtype) as st:
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        X = to_device(wl, wl.X, gpu)
        xt = to_device(wl, wl.targets, gpu)
        Zd = _dev(Z, gpu)
        dZ = _dev(GZ, gpu)
        dxt = torch.zeros((T, d), dtype=torch.float32, device=gpu)
        dX = torch.zeros((N, d), dtype=torch.float32, device=gpu)
        got = {}
        got["dWz"] = S.stca_fusion_backward(st.handle, M, Zd, xt, _dev(Gz, gpu), r * d, dZ=dZ, dxt=dxt,
                                            accumulate=True)["dW"]
        for i in reversed(range(M)):
            dO = dZ[:, i, :].contiguous()
            dC, dWv, _ = S.stca_output_backward(st.handle, i, _dev(Cs[i], gpu), dO, h)
            dU, dXt = S.stca_attention_backward(st.handle, i, _dev(Us[i].reshape(T * h, d), gpu),
                                                wl.target_offsets, dC, N)
            dX += S.stca_encode_backward(st.handle, i, X, dXt, d, r * d)["dX"]
            dq, dWq, _ = S.stca_query_backward(st.handle, i, _dev(qs[i], gpu), dU, h)
            got[f"dWv{i}"], got[f"dWq{i}"] = dWv, dWq
            if i > 0:
                got[f"dWc{i}"] = S.stca_fusion_backward(st.handle, i, Zd, xt, dq, r * d, dZ=dZ, dxt=dxt,
                                                        accumulate=True)["dW"]
            else:
                dxt += S.stca_query_init_backward(st.handle, xt, dq, r * d)["dxt"]
        torch.cuda.synchronize()
        st.status()
        got = {k: v.cpu().numpy() for k, v in got.items()}
        got["dX"], got["dxt"] = dX.cpu().numpy(), dxt.cpu().numpy()
    tol = TOL[dtype]
    assert normwise_err(got["dX"], want["dX"]) <= tol
    assert normwise_err(got["dxt"], want["dxt"]) <= tol
    for k in ("dWz", "dWv0", "dWq1", "dWc1"):
        assert _rel(got[k], want[k]) <= tol, (k, _rel(got[k], want[k]))
