"""Parity of the prediction-head token of Eq. (9) ("Make It Long, Keep It
Fast" digest, §2.1) computed by stca_head through the C ABI, with the fp64
oracle's prediction_head.

The head reads Z (the forward's output) and the targets, so its own parity is
checked on given Z rows (seeded N(0,1) draws), across CTA tails and both
targets-per-CTA layouts; an end-to-end test chains stca_forward and stca_head
against the oracle's forward and head."""
import numpy as np
import pytest

from gen import make_config_workload, make_workload
from oracle import stca_oracle as O
from tests.gpu_helpers import TOL, normwise_err, rows_of, run_gpu, sampled_requests, \
    storage_weights, to_device

pytestmark = pytest.mark.gpu


def _head_gpu(st, wl, Z, device, rows=None):
    import torch
    xt = wl.targets if rows is None else wl.targets[rows]
    xt = to_device(wl, xt, device)
    Zd = torch.from_numpy(np.ascontiguousarray(Z, dtype=np.float32)).to(device)
    z = torch.full((Zd.shape[0], wl.d), float("nan"), dtype=torch.float32, device=device)
    st.head(xt, Zd, z)
    torch.cuda.synchronize()
    st.status()
    return z.cpu().numpy()


@pytest.mark.parametrize("dtype,d,h,M,r,T", [
    ("bf16", 128, 8, 3, 4, 1000),   # the 64-request serving shape's head, 125 CTAs
    ("f32", 64, 2, 1, 2, 13),       # ragged tail of an 8-target CTA
    ("bf16", 256, 8, 4, 2, 67),
    ("bf16", 64, 4, 2, 4, 9),
    ("f32", 128, 4, 3, 2, 1),
    ("bf16", 256, 16, 6, 2, 40),    # (M+1) d = 1792 inputs
    ("f32", 512, 8, 6, 4, 11),      # 4 targets per CTA: 8 do not fit in shared memory
])
def test_head_on_given_outputs(gpu, dtype, d, h, M, r, T):
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[5], targets=[T], d=d, h=h, M=M, r=r, dtype=dtype,
                       seed=300 + d + M + T)
    Z = np.random.default_rng([T, d, M]).standard_normal((T, M, d)).astype(np.float32)
    st = S.Stca(storage_weights(wl), d, h, r, M, dtype)
    try:
        z = _head_gpu(st, wl, Z, gpu)
    finally:
        st.close()
    want = O.head_from_outputs(Z, wl.targets, wl.weights)
    err = normwise_err(z, want)
    assert err <= TOL[dtype], f"head normwise error {err:.3e}"


@pytest.mark.parametrize("step_path", [1, 2])
def test_head_paths_bf16(gpu, step_path):
    """stca_head on a bf16 handle: the tensor-core head products (step path 2,
    the default where the handle has them) and the CUDA-core head kernel
    (step path 1), 1000 targets with a ragged last CTA."""
    import target_attention_jagged_b200 as S
    T, d, h, M, r = 1000, 128, 8, 3, 4
    wl = make_workload(lengths=[5], targets=[T], d=d, h=h, M=M, r=r, dtype="bf16", seed=350 + step_path)
    Z = np.random.default_rng([T, d]).standard_normal((T, M, d)).astype(np.float32)
    st = S.Stca(storage_weights(wl), d, h, r, M, "bf16")
    try:
        st.set_option(S.STCA_OPT_STEP_PATH, step_path)
        z = _head_gpu(st, wl, Z, gpu)
    finally:
        st.close()
    want = O.head_from_outputs(Z, wl.targets, wl.weights)
    err = normwise_err(z, want)
    assert err <= TOL["bf16"], f"head (step path {step_path}) normwise error {err:.3e}"


def test_head_after_forward_c2(gpu):
    import target_attention_jagged_b200 as S
    wl = make_config_workload("c2")
    st = S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype)
    try:
        Z = run_gpu(wl, gpu, handle=st)
        z = _head_gpu(st, wl, Z, gpu)
    finally:
        st.close()
    want = O.head_from_outputs(O.forward_workload(wl), wl.targets, wl.weights)
    err = normwise_err(z, want)
    assert err <= TOL[wl.dtype], f"forward + head normwise error {err:.3e}"


def test_head_after_forward_c3_sampled(gpu):
    import target_attention_jagged_b200 as S
    wl = make_config_workload("c3")
    st = S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype)
    try:
        Z = run_gpu(wl, gpu, handle=st)
        z = _head_gpu(st, wl, Z, gpu)
    finally:
        st.close()
    assert np.all(np.isfinite(z))
    reqs = sampled_requests(wl, 2)
    got = O.forward_workload(wl, requests=reqs)
    rows = rows_of(wl, reqs)
    want = O.head_from_outputs(np.concatenate([got[r] for r in reqs]), wl.targets[rows], wl.weights)
    err = normwise_err(z[rows], want)
    assert err <= TOL[wl.dtype], f"forward + head normwise error {err:.3e} on requests {reqs}"


def test_head_empty_and_missing_weights(gpu):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[4], targets=[2], d=64, h=2, M=2, r=2, dtype="f32", seed=5)
    st = S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype)
    try:
        e = torch.empty((0, wl.d), dtype=torch.float32, device=gpu)
        st.head(e, torch.empty((0, wl.M, wl.d), dtype=torch.float32, device=gpu), e)   # T = 0
        st.status()
    finally:
        st.close()
    w = {k: v for k, v in storage_weights(wl).items() if k not in ("Wz", "zWu", "zWg", "zWd")}
    st = S.Stca(w, wl.d, wl.h, wl.r, wl.M, wl.dtype)
    try:
        Z = torch.zeros((2, wl.M, wl.d), dtype=torch.float32, device=gpu)
        with pytest.raises(S.StcaError) as err:
            st.head(to_device(wl, wl.targets, gpu), Z)
        assert err.value.code == S.stca.STCA_EINVAL and "head weights" in str(err.value)
    finally:
        st.close()


@pytest.mark.parametrize("dtype,d,h,M,r,step_path", [
    ("bf16", 128, 8, 3, 4, 0),     # tensor-core step: the head runs in the last step launch
    ("bf16", 256, 16, 6, 2, 0),    # the widest W_Z operand the fused head takes ((M+1) d = 1792)
    ("bf16", 128, 4, 1, 2, 0),     # one layer: the query-init step is followed by the head step
    ("bf16", 128, 8, 2, 2, 1),     # CUDA-core step: the head kernel after the forward
    ("f32", 64, 2, 2, 2, 0),
])
def test_forward_head_matches_oracle(gpu, dtype, d, h, M, r, step_path):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[300, 1, 129, 2000], targets=[5, 2, 0, 17], d=d, h=h, M=M, r=r,
                       dtype=dtype, seed=41 + d + M)
    st = S.Stca(storage_weights(wl), d, h, r, M, dtype)
    try:
        if step_path:
            st.set_option(S.STCA_OPT_STEP_PATH, step_path)
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        Z, z = st.forward_head(to_device(wl, wl.targets, gpu), wl.target_offsets)
        torch.cuda.synchronize()
        st.status()
        Z, z = Z.cpu().numpy(), z.cpu().numpy()
    finally:
        st.close()
    wantZ = O.forward_workload(wl)
    wantz = O.head_from_outputs(wantZ, wl.targets, wl.weights)
    assert normwise_err(Z, wantZ) <= TOL[dtype]
    err = normwise_err(z, wantz)
    assert err <= TOL[dtype], f"forward + head normwise error {err:.3e}"
