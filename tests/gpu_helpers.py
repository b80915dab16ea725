"""Helpers for the GPU tests: run a gen.Workload through the C ABI and compare.

Error metric: for every (target, layer) output vector v (length d), the max
absolute difference over the max magnitude of the oracle's vector; the worst
such ratio over the batch is compared with the tolerance (1e-3 for fp32
configurations, 2e-2 for bf16 ones).
"""
import numpy as np

TOL = {"f32": 1e-3, "bf16": 2e-2}


def storage_weights(wl):
    out = {}
    for k, v in wl.weights.items():
        if v is None:
            out[k] = None
        elif isinstance(v, list):
            out[k] = [None if a is None else wl.storage(a) for a in v]
        else:
            out[k] = wl.storage(v)
    return out


def to_device(wl, a, device):
    import torch
    s = wl.storage(a)
    t = torch.from_numpy(np.ascontiguousarray(s))
    if wl.dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.to(device)


def run_gpu(wl, device, attn_path=0, encode_path=0, split=0, handle=None, keep=False, step_path=0,
            attn_form=None, attn_kernel=None, pipeline=None):
    """Z (T x M x d, numpy fp32) from the CUDA path through the C ABI."""
    import torch
    import target_attention_jagged_b200 as S
    st = handle or S.Stca(storage_weights(wl), wl.d, wl.h, wl.r, wl.M, wl.dtype)
    try:
        if attn_path:
            st.set_option(S.STCA_OPT_ATTN_PATH, attn_path)
        if encode_path:
            st.set_option(S.STCA_OPT_ENCODE_PATH, encode_path)
        if split:
            st.set_option(S.STCA_OPT_SPLIT_KEYS, split)
        if step_path:
            st.set_option(S.STCA_OPT_STEP_PATH, step_path)
        if attn_form is not None:
            st.set_option(S.STCA_OPT_ATTN_FORM, attn_form)
        if pipeline is not None:
            st.set_option(S.STCA_OPT_PIPELINE, pipeline)
        if attn_kernel is not None:
            st.set_option(S.STCA_OPT_ATTN_KERNEL, attn_kernel)
        X = to_device(wl, wl.X, device)
        xt = to_device(wl, wl.targets, device)
        st.encode(X, wl.offsets)
        Z = torch.full((wl.T, wl.M, wl.d), float("nan"), dtype=torch.float32, device=device)
        st.forward(xt, wl.target_offsets, Z)
        torch.cuda.synchronize()
        st.status()
        return Z.cpu().numpy()
    finally:
        if not keep and handle is None:
            st.close()


def normwise_err(got, want):
    """Worst per-vector error max|g - o| / max|o| over all (target, layer) rows."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if got.size == 0:
        return 0.0
    num = np.abs(got - want).max(axis=-1)
    den = np.maximum(np.abs(want).max(axis=-1), 1e-30)
    e = num / den
    if not np.all(np.isfinite(got)):
        return float("inf")
    return float(e.max())


def sampled_requests(wl, k, seed=0):
    """k requests with targets, chosen reproducibly, always including the longest."""
    rng = np.random.default_rng(seed)
    cand = np.nonzero(wl.target_counts > 0)[0]
    longest = int(cand[np.argmax(wl.lengths[cand])])
    pick = set([longest])
    others = [int(x) for x in rng.permutation(cand) if int(x) != longest]
    pick.update(others[:max(0, k - 1)])
    return sorted(pick)


def rows_of(wl, reqs):
    idx = []
    for r in reqs:
        idx.extend(range(int(wl.target_offsets[r]), int(wl.target_offsets[r + 1])))
    return np.asarray(idx, dtype=np.int64)
