"""Handle options: every value outside its documented range is rejected with
STCA_EINVAL and leaves the option as it was; accepted values read back."""
import pytest

from gen import make_workload
from tests.gpu_helpers import storage_weights

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,good,bad", [
    ("STCA_OPT_ATTN_PATH", [0, 1, 2], [-1, 3]),
    ("STCA_OPT_ENCODE_PATH", [0, 1, 2], [-1, 3]),
    ("STCA_OPT_STEP_PATH", [0, 1, 2], [-1, 3]),
    ("STCA_OPT_ATTN_FORM", [0, 1, 2], [-1, 3]),
    ("STCA_OPT_ATTN_KERNEL", [0, 1, 2], [-1, 3]),
    ("STCA_OPT_PIPELINE", [0, 1], [-1, 2]),
    ("STCA_OPT_TEST_STOP_TILES", [0, 1, 1000], [-1]),
    ("STCA_OPT_BW_GEMM", [0, 1], [-1, 2]),
    ("STCA_OPT_SPLIT_KEYS", [0, 128, 4096], [-128, 100]),
    ("STCA_OPT_TIMING", [0, 1], [2]),
])
def test_option_ranges(gpu, name, good, bad):
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[8], targets=[1], d=64, h=2, M=1, r=1, dtype="bf16", seed=1)
    opt = getattr(S, name)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        for v in good:
            st.set_option(opt, v)
            assert st.get_option(opt) == v
        keep = st.get_option(opt)
        for v in bad:
            with pytest.raises(S.StcaError) as e:
                st.set_option(opt, v)
            assert e.value.code == -1
            assert st.get_option(opt) == keep
        with pytest.raises(S.StcaError):
            st.set_option(S.STCA_OPT_LAUNCHES, 0)      # read-only
