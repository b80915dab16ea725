"""The history encoder X~(i) = LN_i(SwiGLUFFN_i(X)) (Eq. (2)) against the oracle.

stca_get_encoded exposes each layer's encoding, so the tensor-core encoder and
the CUDA-core one are compared with the oracle row by row: every row of every
layer, normwise (max |g - o| / max |o| per row).
"""
import numpy as np
import pytest

from gen import make_workload
from oracle import stca_oracle as O
from tests.gpu_helpers import TOL, storage_weights, to_device

pytestmark = pytest.mark.gpu

ENCODE_SIMT, ENCODE_TC = 1, 2


def encoded_layers(wl, device, path):
    import torch
    import target_attention_jagged_b200 as S
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.set_option(S.STCA_OPT_ENCODE_PATH, path)
        st.encode(to_device(wl, wl.X, device), wl.offsets)
        outs = []
        for i in range(wl.M):
            dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
            buf = torch.full((wl.N, wl.d), float("nan"), dtype=dt, device=device)
            S.stca_get_encoded(st.handle, i, buf)
            outs.append(buf.float().cpu().numpy())
        torch.cuda.synchronize()
        st.status()
    return outs


def rowwise_err(got, want):
    num = np.abs(got.astype(np.float64) - want).max(axis=-1)
    den = np.maximum(np.abs(want).max(axis=-1), 1e-30)
    if not np.all(np.isfinite(got)):
        return float("inf")
    return float((num / den).max())


CASES = [
    # lengths, d, M, r, random_ln
    ([1000, 333, 1], 128, 3, 4, False),     # ragged last tile
    ([128] * 5, 128, 2, 2, True),           # exact tiles
    ([5000, 4000, 130], 64, 2, 2, True),    # many tiles per CTA
    ([700, 129], 256, 2, 2, True),
    ([20000], 128, 1, 8, False),            # rd = 1024
    ([77], 256, 4, 1, False),               # rd = 256, one partial tile
]


@pytest.mark.parametrize("path", [ENCODE_TC, ENCODE_SIMT])
@pytest.mark.parametrize("case", CASES)
def test_encoder_rows(gpu, case, path):
    lengths, d, M, r, rln = case
    wl = make_workload(lengths=lengths, targets=[1] * len(lengths), d=d, h=4, M=M, r=r,
                       dtype="bf16", seed=sum(lengths) + d, random_ln=rln)
    got = encoded_layers(wl, gpu, path)
    for i in range(M):
        want = O.encode_history(wl.X, wl.weights, i)
        err = rowwise_err(got[i], want)
        assert err <= TOL["bf16"], f"layer {i}: row-wise error {err:.3e}"


def test_encoder_fp32_path(gpu):
    wl = make_workload(lengths=[300, 45], targets=[1, 1], d=64, h=2, M=2, r=2, dtype="f32",
                       seed=5, random_ln=True)
    got = encoded_layers(wl, gpu, 0)
    for i in range(2):
        assert rowwise_err(got[i], O.encode_history(wl.X, wl.weights, i)) <= 1e-4


def test_tensor_core_path_rejected_when_unsupported(gpu):
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[10], targets=[1], d=96, h=4, M=1, r=1, dtype="bf16", seed=6)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.set_option(S.STCA_OPT_ENCODE_PATH, ENCODE_TC)
        with pytest.raises(S.StcaError):
            st.encode(to_device(wl, wl.X, gpu), wl.offsets)


@pytest.mark.parametrize("d,M,r", [(64, 2, 2), (128, 3, 4), (256, 3, 2)])
def test_encoder_many_tiles_per_cta(gpu, d, M, r):
    """Several 128-row tiles per persistent CTA (every weight ring wraps many
    times, the X buffers are reused): sampled rows against the oracle.  The
    encoder is row-wise, so the oracle runs on the sampled rows alone."""
    n = 148 * 128 * 3 + 77
    wl = make_workload(lengths=[n - 5000, 5000], targets=[1, 1], d=d, h=4, M=M, r=r,
                       dtype="bf16", seed=11 + d, random_ln=True)
    got = encoded_layers(wl, gpu, ENCODE_TC)
    rng = np.random.default_rng(d)
    rows = np.unique(np.concatenate([rng.integers(0, n, 400), np.arange(n - 80, n),
                                     np.arange(0, 40)]))
    for i in range(M):
        want = O.encode_history(wl.X[rows], wl.weights, i)
        err = rowwise_err(got[i][rows], want)
        assert err <= TOL["bf16"], f"d={d} layer {i}: row-wise error {err:.3e}"
