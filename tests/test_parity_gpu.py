"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Every test runs the library on a seeded synthetic workload and compares Z
element by element with the oracle on the same inputs (normwise per output
vector; 1e-3 for fp32, 2e-2 for bf16).  The full-size configurations are
compared on sampled requests (each request's Z depends only on its own
history and targets), the small ones in full.
"""
import numpy as np
import pytest

from gen import make_config_workload, make_workload
from oracle import stca_oracle as O
from tests.gpu_helpers import TOL, normwise_err, rows_of, run_gpu, sampled_requests

pytestmark = pytest.mark.gpu


def check_full(wl, Z, tol=None):
    want = O.forward_workload(wl)
    err = normwise_err(Z, want)
    assert err <= (tol or TOL[wl.dtype]), f"{wl.name}: normwise error {err:.3e}"
    return err


def check_sampled(wl, Z, k, seed=0):
    reqs = sampled_requests(wl, k, seed)
    got = O.forward_workload(wl, requests=reqs)
    want = np.concatenate([got[r] for r in reqs])
    err = normwise_err(Z[rows_of(wl, reqs)], want)
    assert np.all(np.isfinite(Z)), "non-finite output"
    assert err <= TOL[wl.dtype], f"{wl.name}: normwise error {err:.3e} on requests {reqs}"
    return err


# ------------------------------------------------------------ named configs

def test_c1_full(gpu):
    wl = make_config_workload("c1")
    check_full(wl, run_gpu(wl, gpu))


def test_c2_full(gpu):
    wl = make_config_workload("c2")
    check_full(wl, run_gpu(wl, gpu))


@pytest.mark.parametrize("key,k", [("c3", 3), ("c4", 6), ("c5", 1)])
def test_full_size_sampled(gpu, key, k):
    wl = make_config_workload(key)
    Z = run_gpu(wl, gpu)
    check_sampled(wl, Z, k)


# ------------------------------------------------------------ edge cases

EDGE_L = [1, 2, 127, 128, 129, 257, 1000, 1021]
EDGE_T = [1, 0, 3, 2, 1, 5, 2, 1]


ATTN_AUTO, ATTN_SIMT, ATTN_TC = 0, 1, 2


@pytest.mark.parametrize("attn", [ATTN_AUTO, ATTN_SIMT])
@pytest.mark.parametrize("dtype,d,h,M,r", [("bf16", 128, 4, 2, 2), ("f32", 64, 2, 3, 2),
                                           ("bf16", 256, 8, 2, 2), ("bf16", 64, 4, 1, 4),
                                           ("bf16", 128, 16, 3, 1)])
def test_ragged_edges(gpu, dtype, d, h, M, r, attn):
    wl = make_workload(lengths=EDGE_L, targets=EDGE_T, d=d, h=h, M=M, r=r, dtype=dtype,
                       seed=100 + d + M)
    check_full(wl, run_gpu(wl, gpu, attn_path=attn))


# The CUDA-core attention's row blocks: its launch picks the block height QB
# (4, 8 or 16 rows) from the batch's largest T_r h, so these target mixes reach
# each QB, and the 24- and 48-row requests need more than one block; the key
# counts leave partial groups of 16 (8 at d = 256) and a partial tile.
@pytest.mark.parametrize("targets", [[1, 2, 1, 2, 1], [4, 1, 3, 2, 4], [12, 1, 5, 9, 3]])
@pytest.mark.parametrize("dtype,d,h", [("f32", 32, 2), ("bf16", 32, 2), ("f32", 256, 4), ("bf16", 128, 2)])
def test_simt_row_blocks(gpu, dtype, d, h, targets):
    wl = make_workload(lengths=[1, 15, 130, 515, 1021], targets=targets, d=d, h=h, M=2, r=2,
                       dtype=dtype, seed=200 + d + sum(targets))
    check_full(wl, run_gpu(wl, gpu, attn_path=ATTN_SIMT))


@pytest.mark.parametrize("attn", [ATTN_TC, ATTN_SIMT])
def test_many_targets_per_request(gpu, attn):
    # T_r * h = 40 * 8 = 320 query rows: three 128-row tiles, the last ragged
    wl = make_workload(lengths=[700, 333], targets=[40, 17], d=128, h=8, M=2, r=2,
                       dtype="bf16", seed=7)
    check_full(wl, run_gpu(wl, gpu, attn_path=attn))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_affine_ln_and_separate_query_ffn(gpu, dtype):
    wl = make_workload(lengths=[300, 45, 1], targets=[2, 3, 1], d=128, h=4, M=3, r=2,
                       dtype=dtype, seed=8, random_ln=True, distinct_query_ffn=True)
    check_full(wl, run_gpu(wl, gpu))


def test_small_width(gpu):
    wl = make_workload(lengths=[37, 5], targets=[2, 1], d=16, h=2, M=2, r=1, dtype="f32",
                       seed=9)
    check_full(wl, run_gpu(wl, gpu))


@pytest.mark.parametrize("attn", [ATTN_TC, ATTN_SIMT])
@pytest.mark.parametrize("split", [128, 256, 4096])
def test_split_sizes_agree(gpu, split, attn):
    wl = make_workload(lengths=[1500, 129, 640], targets=[3, 2, 1], d=128, h=4, M=2, r=2,
                       dtype="bf16", seed=10)
    check_full(wl, run_gpu(wl, gpu, split=split, attn_path=attn))


def test_split_change_rebuilds_the_plan(gpu):
    """The attention plan is kept on the device between forwards (and
    encodes) of one layout; a new STCA_OPT_SPLIT_KEYS must replace it.  64
    requests of 1280 keys (10 key tiles, one query tile): the default plan
    cuts a pair into at most 2 items and the step merges the partials itself;
    with 128-key items a pair has 10, more than the step merges, so each layer
    adds a combine launch.  All match the oracle on sampled requests."""
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import storage_weights, to_device
    wl = make_workload(lengths=[1280] * 64, targets=[3] * 64, d=128, h=4, M=2, r=2,
                       dtype="bf16", seed=12)
    X, xt = to_device(wl, wl.X, gpu), to_device(wl, wl.targets, gpu)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.encode(X, wl.offsets)
        counts = []
        for split in (0, 128, 0):
            st.set_option(S.STCA_OPT_SPLIT_KEYS, split)
            n0 = st.get_option(S.STCA_OPT_LAUNCHES)
            Z = torch.zeros((wl.T, wl.M, wl.d), dtype=torch.float32, device=gpu)
            st.forward(xt, wl.target_offsets, Z)
            torch.cuda.synchronize()
            st.status()
            counts.append(st.get_option(S.STCA_OPT_LAUNCHES) - n0)
            check_sampled(wl, Z.cpu().numpy(), 3, seed=len(counts))
        assert counts[1] == counts[0] + wl.M and counts[2] == counts[0], counts


def test_sharp_softmax_rescaling(gpu):
    # The first key tile of each request repeats one token, so its scores are
    # all equal and the running max jumps by far more than the lazy-rescale
    # threshold in later tiles: exercises the O / l correction path.
    wl = make_workload(lengths=[3000, 900], targets=[4, 3], d=128, h=4, M=2, r=2,
                       dtype="bf16", seed=16)
    wl.weights["Wq"] = [w * 3.0 for w in wl.weights["Wq"]]
    for r in range(2):
        lo = int(wl.offsets[r])
        wl.X[lo:lo + 256] = wl.X[lo]
    check_full(wl, run_gpu(wl, gpu, attn_path=ATTN_TC, split=1024))
    check_full(wl, run_gpu(wl, gpu, attn_path=ATTN_SIMT))


def test_attention_paths_agree_on_c2(gpu):
    wl = make_config_workload("c2")
    a = run_gpu(wl, gpu, attn_path=ATTN_TC)
    b = run_gpu(wl, gpu, attn_path=ATTN_SIMT)
    check_full(wl, a)
    assert normwise_err(a, b) <= 2e-2


def test_single_token_history_equals_closed_form(gpu):
    # L = 1: o = x~ W_V W_O whatever the query (softmax over one key)
    wl = make_workload(lengths=[1, 1], targets=[3, 2], d=128, h=8, M=2, r=2, dtype="bf16",
                       seed=11)
    Z = run_gpu(wl, gpu)
    W = wl.weights
    for r in range(2):
        Xr, _ = wl.request(r)
        rows = slice(int(wl.target_offsets[r]), int(wl.target_offsets[r + 1]))
        for i in range(2):
            want = O.encode_history(Xr, W, i)[0] @ W["Wv"][i].astype(float) @ W["Wo"][i].astype(float)
            assert normwise_err(Z[rows, i], np.broadcast_to(want, Z[rows, i].shape)) <= 2e-2


# ------------------------------------------------------------ API behaviour

def test_encode_once_forward_many(gpu):
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import storage_weights, to_device
    wl = make_workload(lengths=[900, 50, 2000], targets=[4, 1, 2], d=128, h=4, M=2, r=2,
                       dtype="bf16", seed=12)
    wl2 = make_workload(lengths=[900, 50, 2000], targets=[0, 6, 3], d=128, h=4, M=2, r=2,
                        dtype="bf16", seed=13)
    wl2.X, wl2.weights = wl.X, wl.weights     # same histories, other targets
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        for w in (wl, wl2, wl):
            Z = st.forward(to_device(w, w.targets, gpu), w.target_offsets)
            torch.cuda.synchronize()
            check_full(w, Z.cpu().numpy())
        st.status()


def test_run_host_matches_device(gpu):
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import storage_weights
    wl = make_workload(lengths=[400, 77], targets=[3, 2], d=128, h=4, M=2, r=2, dtype="bf16",
                       seed=14)
    Zd = run_gpu(wl, gpu)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        Xh = torch.from_numpy(wl.storage(wl.X)).pin_memory()
        th = torch.from_numpy(wl.storage(wl.targets)).pin_memory()
        Zh = torch.empty((wl.T, wl.M, wl.d), dtype=torch.float32).pin_memory()
        S.stca_run_host(st.handle, Xh, wl.offsets, th, wl.target_offsets, Zh)
        assert np.array_equal(Zh.numpy(), Zd)


def test_run_host_chunked_matches_device(gpu):
    """72,000 history rows: stca_run_host copies X in chunks on its own stream and
    encodes each chunk as it lands; the result is bit for bit the device path's."""
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import storage_weights
    wl = make_workload(lengths=[9000] * 8, targets=[2, 1, 3, 1, 2, 1, 1, 4], d=128, h=8, M=2, r=2,
                       dtype="bf16", seed=17)
    Zd = run_gpu(wl, gpu)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        Xh = torch.from_numpy(wl.storage(wl.X)).pin_memory()
        th = torch.from_numpy(wl.storage(wl.targets)).pin_memory()
        for _ in range(2):
            Zh = torch.full((wl.T, wl.M, wl.d), float("nan"), dtype=torch.float32).pin_memory()
            S.stca_run_host(st.handle, Xh, wl.offsets, th, wl.target_offsets, Zh)
            assert np.array_equal(Zh.numpy(), Zd)
        st.status()


def test_forward_before_encode_and_bad_offsets(gpu):
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import storage_weights, to_device
    wl = make_workload(lengths=[10, 20], targets=[1, 1], d=64, h=2, M=1, r=1, dtype="f32",
                       seed=15)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        xt = to_device(wl, wl.targets, gpu)
        with pytest.raises(S.StcaError) as e:
            st.forward(xt, wl.target_offsets)
        assert e.value.code == -2
        X = to_device(wl, wl.X, gpu)
        with pytest.raises(S.StcaError) as e:
            st.encode(X, [0, 30, 30])            # empty history
        assert e.value.code == -1
        with pytest.raises(S.StcaError):
            st.encode(X, [0, 20, 10])            # decreasing
        st.encode(X, wl.offsets)
        with pytest.raises(S.StcaError):
            st.forward(xt, [0, 1, 1, 2])         # wrong R
        Z = torch.empty((0, 1, 64), device=gpu)
        st.forward(xt[:0], [0, 0, 0], Z)         # T = 0 is a no-op
        st.status()


STEP_CC, STEP_TC = 1, 2


@pytest.mark.parametrize("step", [STEP_TC, STEP_CC])
@pytest.mark.parametrize("d,h,M,r,rln,dq", [(128, 8, 3, 4, False, False), (128, 4, 2, 2, True, True),
                                            (256, 16, 4, 2, True, False), (256, 8, 1, 1, False, True),
                                            (128, 2, 5, 1, True, True)])
def test_step_paths(gpu, step, d, h, M, r, rln, dq):
    """Both per-target step implementations against the oracle: 37 targets in
    requests of 1 to 17 targets (16-target CTAs, the last one ragged), heads of
    16 to 64 columns, one to five layers, affine LayerNorm, separate query FFN."""
    wl = make_workload(lengths=[900, 130, 1, 2100, 64], targets=[9, 1, 3, 17, 7], d=d, h=h, M=M,
                       r=r, dtype="bf16", seed=300 + d + h + M, random_ln=rln,
                       distinct_query_ffn=dq)
    check_full(wl, run_gpu(wl, gpu, step_path=step))


def test_tensor_core_step_rejected_when_unsupported(gpu):
    import target_attention_jagged_b200 as S
    wl = make_workload(lengths=[50], targets=[2], d=64, h=4, M=1, r=2, dtype="bf16", seed=13)
    with pytest.raises(S.StcaError):
        run_gpu(wl, gpu, step_path=STEP_TC)
    wl = make_workload(lengths=[50], targets=[2], d=128, h=4, M=1, r=2, dtype="bf16", seed=13)
    with pytest.raises(S.StcaError):
        run_gpu(wl, gpu, step_path=STEP_TC, attn_path=ATTN_SIMT)


# ------------------------------------------------------------ the two tensor-core attention kernels
# 0: the library's choice: for d = 128 the split-softmax kernel projects its
#    rows by W_V itself, and the step (or, with many items per row, the
#    combine kernel) merges the d_h-wide partials;
# 1: the split-softmax kernel followed by the split combine of the rows c_j;
# 2: the two-group kernel (d <= 128), which merges split partials itself.

KERNEL_AUTO, KERNEL_SPLIT_SOFTMAX, KERNEL_TWO_GROUP = 0, 1, 2
ALL_KERNELS = [KERNEL_AUTO, KERNEL_SPLIT_SOFTMAX, KERNEL_TWO_GROUP]


@pytest.mark.parametrize("kernel", ALL_KERNELS)
@pytest.mark.parametrize("d,h", [(128, 8), (64, 4), (128, 2), (128, 1)])
def test_tc_kernels_ragged(gpu, kernel, d, h):
    wl = make_workload(lengths=EDGE_L, targets=EDGE_T, d=d, h=h, M=2, r=2, dtype="bf16",
                       seed=400 + d + h)
    check_full(wl, run_gpu(wl, gpu, attn_path=ATTN_TC, attn_kernel=kernel))


@pytest.mark.parametrize("kernel", ALL_KERNELS)
@pytest.mark.parametrize("split", [0, 128, 384])
def test_tc_kernels_split_merge(gpu, kernel, split):
    """Pairs cut into many items (one 20k-key request over every CTA, a second
    with three query tiles, the last one ragged): every split is merged, by the
    last-arriving warp (two-group kernel) or the combine kernel."""
    wl = make_workload(lengths=[20000, 3000, 1], targets=[3, 40, 2], d=128, h=8, M=2, r=2,
                       dtype="bf16", seed=410)
    check_full(wl, run_gpu(wl, gpu, attn_path=ATTN_TC, split=split, attn_kernel=kernel))


@pytest.mark.parametrize("kernel", ALL_KERNELS)
def test_tc_kernels_sharp_softmax(gpu, kernel):
    wl = make_workload(lengths=[3000, 900, 130], targets=[4, 3, 1], d=128, h=4, M=2, r=2,
                       dtype="bf16", seed=411)
    wl.weights["Wq"] = [w * 3.0 for w in wl.weights["Wq"]]
    for r in range(3):
        lo = int(wl.offsets[r])
        n = min(256, int(wl.lengths[r]))
        wl.X[lo:lo + n] = wl.X[lo]
    check_full(wl, run_gpu(wl, gpu, attn_path=ATTN_TC, attn_kernel=kernel))


# The two-half pipeline (STCA_OPT_PIPELINE, on by default where it applies):
# the halves split the requests by attention work, and one launch runs one
# half's per-target step beside the other half's attention.  It applies when
# each pair (request, query tile) of the halves' plans has at most 8 items,
# i.e. with enough pairs per half, and when the batch holds at least 24 pairs
# (key tile, query tile) of attention work per SM; otherwise the forward runs
# in one piece.
def _forward_launches(wl, gpu, pipeline):
    """Z and the number of kernels one forward launched."""
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import storage_weights, to_device
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.set_option(S.STCA_OPT_PIPELINE, pipeline)
        st.encode(to_device(wl, wl.X, gpu), wl.offsets)
        n0 = st.get_option(S.STCA_OPT_LAUNCHES)
        Z = torch.zeros((wl.T, wl.M, wl.d), dtype=torch.float32, device=gpu)
        st.forward(to_device(wl, wl.targets, gpu), wl.target_offsets, Z)
        torch.cuda.synchronize()
        st.status()
        return Z.cpu().numpy(), st.get_option(S.STCA_OPT_LAUNCHES) - n0


@pytest.mark.parametrize("seed", [0, 1])
def test_pipeline_matches_oracle(gpu, seed):
    """80 requests of 4000..8000 keys (about 3700 pairs of attention work, 25
    per SM): the pipeline engages (2M + 2 launches against 2M + 1), matches
    the oracle on sampled requests and the one-piece forward on the whole
    batch.  Seed 1 has ragged targets (0 to 40 per request: several query
    tiles, empty requests)."""
    rng = np.random.default_rng(seed)
    R = 80
    lengths = rng.integers(4000, 8001, R).tolist()
    targets = [16] * R if seed == 0 else rng.integers(0, 41, R).tolist()
    wl = make_workload(lengths=lengths, targets=targets, d=128, h=8, M=3, r=2, dtype="bf16", seed=430 + seed)
    a, na = _forward_launches(wl, gpu, 1)
    b, nb = _forward_launches(wl, gpu, 0)
    assert na == 2 * wl.M + 2 and nb == 2 * wl.M + 1, (na, nb)
    check_sampled(wl, a, 4, seed=seed)
    assert normwise_err(a, b) <= 2e-2


@pytest.mark.parametrize("big", [True, False])
def test_encode_forward_matches_separate_calls(gpu, big):
    """stca_encode_forward (one call: the first half's query init may overlap
    the encoder's last tiles) gives the Z of stca_encode + stca_forward, bit
    for bit, twice in a row; big: 80 requests of 4000..8000 keys (the two-half
    pipeline engages), else a small ragged batch (one piece)."""
    import torch
    import target_attention_jagged_b200 as S
    from tests.gpu_helpers import storage_weights, to_device
    if big:
        rng = np.random.default_rng(3)
        wl = make_workload(lengths=rng.integers(4000, 8001, 80).tolist(), targets=[16] * 80, d=128, h=8,
                           M=3, r=2, dtype="bf16", seed=450)
    else:
        wl = make_workload(lengths=EDGE_L, targets=EDGE_T, d=128, h=4, M=2, r=2, dtype="bf16", seed=451)
    X, xt = to_device(wl, wl.X, gpu), to_device(wl, wl.targets, gpu)
    with S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype) as st:
        st.encode(X, wl.offsets)
        want = torch.zeros((wl.T, wl.M, wl.d), dtype=torch.float32, device=gpu)
        st.forward(xt, wl.target_offsets, want)
        n0 = st.get_option(S.STCA_OPT_LAUNCHES)
        for _ in range(2):
            got = torch.full((wl.T, wl.M, wl.d), float("nan"), dtype=torch.float32, device=gpu)
            st.encode_forward(X, wl.offsets, xt, wl.target_offsets, got)
            torch.cuda.synchronize()
            st.status()
            assert torch.equal(got, want)
        # the launches of one encode and one forward (the counter restarts at
        # each encode): the encoder, then 2M + 2 launches with the pipeline,
        # 2M + 1 without
        assert st.get_option(S.STCA_OPT_LAUNCHES) == n0 == 1 + (2 * wl.M + 2 if big else 2 * wl.M + 1)
        # T == 0: encodes only; a later forward reuses the encoding
        S.stca_encode_forward(st.handle, X, wl.offsets, xt[:0], np.zeros(wl.R + 1, dtype=np.int64), want[:0])
        again = torch.zeros_like(want)
        st.forward(xt, wl.target_offsets, again)
        torch.cuda.synchronize()
        assert torch.equal(again, want)
    check_sampled(wl, want.cpu().numpy(), 3, seed=6)


def test_pipeline_skips_small_batches(gpu):
    """32 requests of 200..2000 keys, 8 targets each: too little attention
    work per SM for the pipeline to pay, so the forward runs in one piece (the
    launches of the pipeline-off forward) and gives the same Z."""
    wl = make_workload(lengths=("uniform", 200, 2000), targets=("fixed", 8), d=128, h=4, M=2, r=2,
                       dtype="bf16", seed=442, R=32)
    a, na = _forward_launches(wl, gpu, 1)
    b, nb = _forward_launches(wl, gpu, 0)
    assert na == nb, (na, nb)
    assert normwise_err(a, b) == 0.0
    check_sampled(wl, a, 4, seed=5)


def test_pipeline_falls_back(gpu):
    """Two requests whose pairs would need far more than 8 items each: the
    forward runs in one piece (the same launches as with the pipeline off:
    here with the separate merge of the partials) and matches the oracle."""
    wl = make_workload(lengths=[20000, 300], targets=[3, 17], d=128, h=8, M=3, r=2, dtype="bf16", seed=441)
    a, na = _forward_launches(wl, gpu, 1)
    b, nb = _forward_launches(wl, gpu, 0)
    assert na == nb, (na, nb)
    check_full(wl, a)
    assert normwise_err(a, b) == 0.0


def test_tc_kernels_agree_on_c3(gpu):
    wl = make_config_workload("c3")
    a = run_gpu(wl, gpu, attn_kernel=KERNEL_TWO_GROUP)
    check_sampled(wl, a, 2, seed=3)
    b = run_gpu(wl, gpu, attn_kernel=KERNEL_SPLIT_SOFTMAX)
    assert normwise_err(a, b) <= 2e-2
    c = run_gpu(wl, gpu, attn_kernel=KERNEL_AUTO)
    check_sampled(wl, c, 2, seed=4)
    assert normwise_err(c, b) <= 2e-2
    e = run_gpu(wl, gpu, attn_kernel=KERNEL_AUTO, pipeline=0)
    assert normwise_err(c, e) <= 2e-2
