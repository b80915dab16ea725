"""The naive attention form (Eq. (12): K = X~ W_K and V = X~ W_V projected once
per layer, then single-query attention per head over d_h features), selected
with STCA_OPT_ATTN_FORM, against the fp64 oracle.  The oracle's naive and
reordered forms agree to 1e-12 (pinned on CPU), so the same expected Z serves
both forms of the library."""
import numpy as np
import pytest

from gen import make_config_workload, make_workload
from oracle import stca_oracle as O
from tests.gpu_helpers import TOL, normwise_err, rows_of, run_gpu, sampled_requests, storage_weights

pytestmark = pytest.mark.gpu

FORM_REORDERED, FORM_NAIVE, FORM_AUTO = 0, 1, 2

# lengths: one key, partial and full 128-key tiles; targets: none, one, more than
# one query slot of the packed layout (32 positions for d_h 16, 64 for d_h 32)
LENGTHS = [1, 127, 129, 300, 1000, 57]
TARGETS = [3, 0, 40, 1, 70, 33]


@pytest.mark.parametrize("d,h,M,r", [(128, 8, 2, 2), (128, 4, 3, 4), (256, 16, 2, 2),
                                     (256, 8, 2, 2), (128, 2, 2, 2)])
def test_naive_form_matches_oracle(gpu, d, h, M, r):
    wl = make_workload(lengths=LENGTHS, targets=TARGETS, d=d, h=h, M=M, r=r, dtype="bf16",
                       seed=500 + d + h)
    Z = run_gpu(wl, gpu, attn_form=FORM_NAIVE)
    want = O.forward_workload(wl, attention=O.attention_naive)
    err = normwise_err(Z, want)
    assert err <= TOL["bf16"], f"naive form d={d} h={h}: normwise error {err:.3e}"


def test_forms_agree_on_ragged_batch(gpu):
    wl = make_config_workload("c2")
    Zn = run_gpu(wl, gpu, attn_form=FORM_NAIVE)
    Zr = run_gpu(wl, gpu, attn_form=FORM_REORDERED)
    want = O.forward_workload(wl)
    assert normwise_err(Zn, want) <= TOL["bf16"]
    assert normwise_err(Zr, want) <= TOL["bf16"]


def test_naive_form_stress_sampled(gpu):
    """The 20k-key, 64-target stress batch, where the naive form has fewer FLOPs."""
    wl = make_config_workload("c5")
    Z = run_gpu(wl, gpu, attn_form=FORM_NAIVE)
    reqs = sampled_requests(wl, 1)
    got = O.forward_workload(wl, requests=reqs)
    want = np.concatenate([got[q] for q in reqs])
    err = normwise_err(Z[rows_of(wl, reqs)], want)
    assert np.all(np.isfinite(Z)) and err <= TOL["bf16"], f"c5 naive: {err:.3e} on {reqs}"


def test_auto_form_choice(gpu):
    """Auto takes the naive form where T_r h > d + T_r (many targets and heads)
    and the reordered form otherwise; both runs stay within tolerance."""
    import target_attention_jagged_b200 as S
    cases = [  # (d, h, targets per request) -> expected form
        (256, 16, 64, 1),   # T h = 1024 > d + T = 320
        (128, 8, 16, 0),    # T h = 128 < d + T = 144
    ]
    for d, h, tr, want_form in cases:
        wl = make_workload(lengths=[600, 900], targets=[tr, tr], d=d, h=h, M=2, r=2, dtype="bf16",
                           seed=7 + d)
        st = S.Stca(storage_weights(wl), d, h, 2, 2, "bf16")
        try:
            Z = run_gpu(wl, gpu, handle=st, attn_form=FORM_AUTO)
            assert st.get_option(S.STCA_OPT_LAST_FORM) == want_form, (d, h, tr)
        finally:
            st.close()
        assert normwise_err(Z, O.forward_workload(wl)) <= TOL["bf16"]


def test_naive_form_rejected_when_unsupported(gpu):
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[50], targets=[2], d=64, h=2, M=1, r=2, dtype="f32", seed=3)
    with pytest.raises(S.StcaError):
        run_gpu(wl, gpu, attn_form=FORM_NAIVE)
    Z = run_gpu(wl, gpu, attn_form=FORM_AUTO)      # auto falls back to the reordered form
    assert normwise_err(Z, O.forward_workload(wl)) <= TOL["f32"]


def test_naive_form_with_fused_head(gpu):
    """The naive form's last step also runs the Eq. (9) head (stca_forward_head)."""
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import to_device
    wl = make_workload(lengths=LENGTHS, targets=TARGETS, d=256, h=16, M=2, r=2, dtype="bf16", seed=61)
    st = S.Stca(storage_weights(wl), 256, 16, 2, 2, "bf16")
    try:
        st.set_option(S.STCA_OPT_ATTN_FORM, FORM_NAIVE)
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        Z, z = st.forward_head(to_device(wl, wl.targets, gpu), wl.target_offsets)
        torch.cuda.synchronize()
        st.status()
        assert st.get_option(S.STCA_OPT_LAST_FORM) == 1
        Z, z = Z.cpu().numpy(), z.cpu().numpy()
    finally:
        st.close()
    wantZ = O.forward_workload(wl)
    assert normwise_err(Z, wantZ) <= TOL["bf16"]
    assert normwise_err(z, O.head_from_outputs(wantZ, wl.targets, wl.weights)) <= TOL["bf16"]


def test_forward_head_without_head_weights(gpu):
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import to_device
    wl = make_workload(lengths=[40], targets=[2], d=128, h=8, M=1, r=2, dtype="bf16", seed=62)
    w = {k: v for k, v in storage_weights(wl).items() if k not in ("Wz", "zWu", "zWg", "zWd")}
    st = S.Stca(w, 128, 8, 2, 1, "bf16")
    try:
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        with pytest.raises(S.StcaError) as e:
            st.forward_head(to_device(wl, wl.targets, gpu), wl.target_offsets)
        assert e.value.code == S.stca.STCA_EINVAL
    finally:
        st.close()
