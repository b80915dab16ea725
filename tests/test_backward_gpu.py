"""Backward pass of the history encoding (Eqs. (1)-(2)) and of the merged
single-query attention (Eq. (13)) through the C ABI, against the fp64 backward
oracle (oracle/stca_backward.py) on the same inputs.

Error metric: max |g - o| / max |o| over each gradient tensor (per row for dX,
dU and dX~); 2e-2 for bf16 handles (TF32 products), 1e-3 for fp32 handles."""
import numpy as np
import pytest

from gen import make_workload
from oracle import stca_backward as B
from tests.gpu_helpers import TOL, normwise_err, storage_weights, to_device

pytestmark = pytest.mark.gpu


def _rel(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.abs(g - o).max() / max(np.abs(o).max(), 1e-30))


@pytest.mark.parametrize("dtype,d,r,layer", [("bf16", 128, 4, 1), ("f32", 64, 2, 0),
                                             ("bf16", 256, 2, 0), ("bf16", 64, 4, 1)])
def test_encode_backward_matches_oracle(gpu, dtype, d, r, layer):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[1500, 777, 1], targets=[1, 1, 1], d=d, h=4, M=2, r=r, dtype=dtype,
                       seed=900 + d, random_ln=True)
    G = np.random.default_rng(d + layer).standard_normal((wl.N, d)).astype(np.float32)
    with S.Stca(storage_weights(wl), d, 4, r, 2, dtype) as st:
        X = to_device(wl, wl.X, gpu)
        g = S.stca_encode_backward(st.handle, layer, X, torch.from_numpy(G).to(gpu), d, r * d)
        torch.cuda.synchronize()
        got = {k: v.cpu().numpy() for k, v in g.items()}
    want = B.encode_history_backward(wl.X, wl.weights, layer, G)
    tol = TOL[dtype]
    assert normwise_err(got["dX"], want["dX"]) <= tol
    for k in ("dWu", "dWg", "dWd", "dgamma", "dbeta"):
        assert _rel(got[k], want[k]) <= tol, (k, _rel(got[k], want[k]))


@pytest.mark.parametrize("d,r,lengths", [(128, 4, [5000, 1200, 3]), (64, 2, [4100, 1])])
def test_encode_backward_gemm_paths(gpu, d, r, lengths):
    """bf16 handle: the library's tensor-core TF32 GEMM (default) and cuBLASLt
    (STCA_OPT_BW_GEMM = 1) against the oracle, on enough rows (N > 4096) that the
    weight gradients' long K is split over CTAs and added atomically."""
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=lengths, targets=[1] * len(lengths), d=d, h=4, M=1, r=r, dtype="bf16",
                       seed=950 + d, random_ln=True)
    G = np.random.default_rng(d).standard_normal((wl.N, d)).astype(np.float32)
    want = B.encode_history_backward(wl.X, wl.weights, 0, G)
    for gemm in (0, 1):
        with S.Stca(storage_weights(wl), d, 4, r, 1, "bf16") as st:
            st.set_option(S.STCA_OPT_BW_GEMM, gemm)
            X = to_device(wl, wl.X, gpu)
            g = S.stca_encode_backward(st.handle, 0, X, torch.from_numpy(G).to(gpu), d, r * d)
            torch.cuda.synchronize()
            st.status()
            got = {k: v.cpu().numpy() for k, v in g.items()}
        assert normwise_err(got["dX"], want["dX"]) <= TOL["bf16"], gemm
        for k in ("dWu", "dWg", "dWd", "dgamma", "dbeta"):
            assert _rel(got[k], want[k]) <= TOL["bf16"], (gemm, k, _rel(got[k], want[k]))


# path 0: the library's choice (tensor cores for bf16 and d in {64, 128}, else
# CUDA cores); path 1: the CUDA-core kernels forced (STCA_OPT_ATTN_PATH).
# The last cases give requests several 128-row query tiles (several tiles add
# to the same history rows) and a 6000-key history (its query tile's keys are
# split over several CTAs, whose dU parts add up).
@pytest.mark.parametrize("dtype,d,h,layer,lengths,targets,path", [
    ("bf16", 128, 8, 0, [700, 1, 129, 300, 64], [3, 2, 0, 5, 1], 0),
    ("bf16", 128, 8, 0, [700, 1, 129, 300, 64], [3, 2, 0, 5, 1], 1),
    ("f32", 64, 2, 1, [700, 1, 129, 300, 64], [3, 2, 0, 5, 1], 0),
    ("bf16", 256, 16, 1, [700, 1, 129, 300, 64], [3, 2, 0, 5, 1], 0),
    ("bf16", 64, 4, 1, [700, 1, 129, 300, 64], [3, 2, 0, 5, 1], 0),
    ("bf16", 128, 8, 1, [6000, 333, 1, 900], [20, 17, 1, 0], 0),
    ("bf16", 64, 8, 0, [6000, 333, 1, 900], [20, 17, 1, 0], 0),
])
def test_attention_backward_matches_oracle(gpu, dtype, d, h, layer, lengths, targets, path):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=lengths, targets=targets, d=d, h=h, M=2, r=2, dtype=dtype, seed=77 + d)
    rng = np.random.default_rng(d + h)
    rows = wl.T * h
    U = (rng.standard_normal((rows, d)) * (2.0 / np.sqrt(d))).astype(np.float32)
    dC = rng.standard_normal((rows, d)).astype(np.float32)
    with S.Stca(storage_weights(wl), d, h, 2, 2, dtype) as st:
        if path:
            st.set_option(S.STCA_OPT_ATTN_PATH, path)
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        xt = torch.empty((wl.N, d), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device=gpu)
        S.stca_get_encoded(st.handle, layer, xt)
        for _ in range(2):          # a second call reuses the workspace
            dU, dX = S.stca_attention_backward(st.handle, layer, torch.from_numpy(U).to(gpu),
                                               wl.target_offsets, torch.from_numpy(dC).to(gpu), wl.N)
            torch.cuda.synchronize()
            st.status()
        Xt = xt.float().cpu().numpy()
        got_u, got_x = dU.cpu().numpy(), dX.cpu().numpy()
    want_u, want_x = B.attention_backward_batch(U, Xt, wl.offsets, wl.target_offsets, h, dC)
    tol = TOL[dtype]
    # A request with a one-key history has dU = 0 exactly (a softmax over one key
    # does not depend on u): those rows are held to the tensor's scale, since a
    # rounding residue has no row scale to be relative to.
    live = np.abs(want_u).max(axis=1) > 0
    assert normwise_err(got_u[live], want_u[live]) <= tol, normwise_err(got_u[live], want_u[live])
    assert np.abs(got_u[~live]).max(initial=0.0) <= tol * np.abs(want_u).max()
    keyrows = np.abs(want_x).max(axis=1) > 0               # rows of requests with targets
    assert normwise_err(got_x[keyrows], want_x[keyrows]) <= tol
    assert np.all(got_x[~keyrows] == 0)


def test_backward_rejects_bad_arguments(gpu):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[20], targets=[1], d=64, h=2, M=1, r=2, dtype="bf16", seed=1)
    with S.Stca(storage_weights(wl), 64, 2, 2, 1, "bf16") as st:
        X = to_device(wl, wl.X, gpu)
        G = torch.zeros((wl.N, 64), dtype=torch.float32, device=gpu)
        with pytest.raises(S.StcaError):
            S.stca_encode_backward(st.handle, 5, X, G, 64, 128)         # no such layer
        with pytest.raises(S.StcaError) as e:                             # before any encode
            S.stca_attention_backward(st.handle, 0, torch.zeros((2, 64), device=gpu), [0, 1],
                                      torch.zeros((2, 64), device=gpu), wl.N)
        assert e.value.code == S.stca.STCA_ESTATE
