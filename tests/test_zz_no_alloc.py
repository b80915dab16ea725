"""stca_forward_static: the forward pass for callers that cannot allocate device
memory once they serve (their memory belongs to another allocator's pool, their
budget is fixed at start-up, or they cannot afford the synchronisation that
cudaMalloc / cudaFree may bring).  Its workspace lives in a fixed device array
built into the library instead of buffers the handle grows.

Each test checks it, through the C ABI, against stca_forward -- the entry point
that allocates its own workspace -- on the same encoded batch, within the bf16
tolerance of the other GPU tests, on two calls in a row (the second call finds
the array as the first left it).  This file is collected last on purpose.
"""
import numpy as np
import pytest

from gen import make_workload
from tests.gpu_helpers import TOL, normwise_err, storage_weights, to_device

pytestmark = pytest.mark.gpu


def _compare(st, wl, X_dev, gpu):
    import torch
    import target_attention_jagged_b200 as S
    xt = to_device(wl, wl.targets, gpu)
    Zref = st.forward(xt, wl.target_offsets)
    torch.cuda.synchronize()
    ref = Zref.cpu().numpy()
    for _ in range(2):
        Z = torch.full((wl.T, wl.M, wl.d), float("nan"), dtype=torch.float32, device=gpu)
        S.stca_forward_static(st.handle, xt, wl.target_offsets, Z)
        torch.cuda.synchronize()
        st.status()
        err = normwise_err(Z.cpu().numpy(), ref)
        assert err <= TOL["bf16"], f"static forward differs from stca_forward: {err:.3e}"


@pytest.mark.parametrize("d,h", [(128, 8), (64, 4), (256, 8)])
def test_static_forward_matches_forward(gpu, d, h):
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[1500, 129, 4000, 1], targets=[3, 2, 20, 1], d=d, h=h, M=3,
                       r=2, dtype="bf16", seed=21 + d)
    other = make_workload(lengths=[1500, 129, 4000, 1], targets=[0, 7, 1, 2], d=d, h=h, M=3,
                          r=2, dtype="bf16", seed=22 + d)
    other.X, other.weights = wl.X, wl.weights          # same histories, other targets
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        X = to_device(wl, wl.X, gpu)
        st.encode(X, wl.offsets)
        _compare(st, wl, X, gpu)
        _compare(st, other, X, gpu)


def test_static_forward_rejects_oversized_batch(gpu):
    import torch
    import target_attention_jagged_b200 as S
    # 9000 targets x 16 heads x 128 x 2 bytes of query rows alone exceed the array
    wl = make_workload(lengths=[300], targets=[9000], d=128, h=16, M=1, r=1, dtype="bf16",
                       seed=23)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        Z = torch.zeros((wl.T, wl.M, wl.d), dtype=torch.float32, device=gpu)
        with pytest.raises(S.StcaError) as e:
            S.stca_forward_static(st.handle, to_device(wl, wl.targets, gpu), wl.target_offsets, Z)
        assert e.value.code == -1 and "static scratch" in str(e.value)
        assert float(Z.abs().sum()) == 0.0                   # nothing was launched
        st.status()


def test_static_forward_needs_tensor_core_handle(gpu):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[50], targets=[2], d=64, h=2, M=1, r=1, dtype="f32", seed=24)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        Z = torch.zeros((wl.T, wl.M, wl.d), dtype=torch.float32, device=gpu)
        with pytest.raises(S.StcaError):
            S.stca_forward_static(st.handle, to_device(wl, wl.targets, gpu), wl.target_offsets, Z)
