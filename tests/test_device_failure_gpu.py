"""The device-side failure path of the tensor-core attention, driven from the
host: with STCA_OPT_TEST_STOP_TILES the kernel's loader stops after a few key
tiles and the kernel leaves as it does when a bounded wait runs out -- the
other roles stop at their next wait, copies and MMAs in flight are let finish,
TMEM is freed.  Nothing is broken or left waiting without a bound.  The call
returns, stca_device_status reports STCA_EDEVICE, and after the hook is
cleared the same handle's next forward matches the oracle again."""
import numpy as np
import pytest

from gen import make_workload
from oracle import stca_oracle as O
from tests.gpu_helpers import TOL, normwise_err, storage_weights, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kernel,d,h", [(0, 128, 8), (2, 128, 8), (1, 256, 8), (0, 64, 4), (2, 64, 4)])
def test_attention_gives_up_and_recovers(gpu, kernel, d, h):
    import torch
    import target_attention_jagged_b200 as S
    # 4 requests of 20000 keys: 628 key tiles over at most 148 CTAs, so every
    # CTA of the stream-K plan holds at least 4 tiles and its loader stops
    # part-way through its run
    L = [20000, 20000, 20000, 20000]
    plan = S.stca_plan_attention(np.cumsum([0] + L), np.cumsum([0, 3, 1, 2, 5]), h, 2, 148)
    assert np.diff(plan["cta_begin"]).min() >= 1
    tiles_per_cta = -(-sum(-(-x // 128) for x in L) // plan["grid"])
    assert tiles_per_cta >= 4
    wl = make_workload(lengths=L, targets=[3, 1, 2, 5], d=d, h=h, M=1, r=2, dtype="bf16",
                       seed=500 + d + kernel)
    want = O.forward_workload(wl)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.set_option(S.STCA_OPT_ATTN_KERNEL, kernel)
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        xt = to_device(wl, wl.targets, gpu)
        st.set_option(S.STCA_OPT_TEST_STOP_TILES, 2)
        Z = torch.zeros((wl.T, wl.M, wl.d), dtype=torch.float32, device=gpu)
        st.forward(xt, wl.target_offsets, Z)            # the launches themselves succeed
        with pytest.raises(S.StcaError) as e:
            st.status()
        assert e.value.code == -5 and "attention" in str(e.value)
        st.status()                                      # the read cleared the status word
        st.set_option(S.STCA_OPT_TEST_STOP_TILES, 0)
        for _ in range(2):
            Z = torch.full((wl.T, wl.M, wl.d), float("nan"), dtype=torch.float32, device=gpu)
            st.forward(xt, wl.target_offsets, Z)
            torch.cuda.synchronize()
            st.status()
            err = normwise_err(Z.cpu().numpy(), want)
            assert err <= TOL["bf16"], f"after the failure: normwise error {err:.3e}"
