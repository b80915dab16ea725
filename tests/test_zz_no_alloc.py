"""stca_forward_static: the forward pass for callers that cannot allocate device
memory once they serve (their memory belongs to another allocator's pool, their
budget is fixed at start-up, or they cannot afford the synchronisation that
cudaMalloc / cudaFree may bring).  Its workspace lives in a fixed device array
built into the library instead of buffers the handle grows.

Each test checks it, through the C ABI, against stca_forward -- the entry point
that allocates its own workspace -- on the same encoded batch, within the bf16
tolerance of the other GPU tests, on two calls in a row (the second call finds
the array as the first left it); one test also checks it directly against the
fp64 oracle.  This file is collected last on purpose.
"""
import numpy as np
import pytest

from gen import make_workload
from oracle import stca_oracle as O
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


def test_static_forward_matches_oracle(gpu):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[300, 1, 129, 700], targets=[2, 1, 3, 0], d=128, h=8, M=2, r=2,
                       dtype="bf16", seed=25)
    want = O.forward_workload(wl)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        xt = to_device(wl, wl.targets, gpu)
        for _ in range(2):
            Z = torch.full((wl.T, wl.M, wl.d), float("nan"), dtype=torch.float32, device=gpu)
            S.stca_forward_static(st.handle, xt, wl.target_offsets, Z)
            torch.cuda.synchronize()
            st.status()
            err = normwise_err(Z.cpu().numpy(), want)
            assert err <= TOL["bf16"], f"static forward vs the oracle: {err:.3e}"


def test_static_forward_halves_ctas_to_fit(gpu):
    """At one CTA per SM this batch's split partials push the workspace past
    the 32 MiB array (about 37 MiB); with half the CTAs it fits (about 28 MiB).
    The result must not depend on the split."""
    import target_attention_jagged_b200 as S
    R, L, Tr = 64, 2000, 8
    plan = S.stca_plan_attention(np.arange(R + 1) * L, np.arange(R + 1) * Tr, 16, 2, 148)
    assert plan["partial_rows"] * (256 + 2) * 4 > 24 << 20       # the partials dominate
    wl = make_workload(lengths=[L] * R, targets=[Tr] * R, d=256, h=16, M=1, r=1, dtype="bf16",
                       seed=26)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        X = to_device(wl, wl.X, gpu)
        st.encode(X, wl.offsets)
        _compare(st, wl, X, gpu)


def test_static_forward_rejects_naive_form_and_capture(gpu):
    import torch
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[200, 64], targets=[2, 1], d=128, h=4, M=1, r=2, dtype="bf16",
                       seed=27)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        xt = to_device(wl, wl.targets, gpu)
        Z = torch.zeros((wl.T, wl.M, wl.d), dtype=torch.float32, device=gpu)
        st.set_option(S.STCA_OPT_ATTN_FORM, 1)
        with pytest.raises(S.StcaError) as e:
            S.stca_forward_static(st.handle, xt, wl.target_offsets, Z)
        assert e.value.code == -1 and "naive" in str(e.value)
        st.set_option(S.STCA_OPT_ATTN_FORM, 0)
        torch.cuda.synchronize()
        # under an active stream capture the call is refused before it enqueues anything
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            g.capture_begin()
            try:
                with pytest.raises(S.StcaError) as e:
                    S.stca_forward_static(st.handle, xt, wl.target_offsets, Z, stream=s)
            finally:
                g.capture_end()
        assert e.value.code == -1 and "captured" in str(e.value)
        torch.cuda.synchronize()
        assert float(Z.abs().sum()) == 0.0
        st.status()
