"""The batch builder's device gather (stca_sl_gather) and the training-batch
forward, against the oracle: the packed rows and the per-row user index are
compared bit for bit with oracle/sparse_batch.py's gather; the forward over a
packed batch is compared with the oracle's forward on the same packed rows."""
import numpy as np
import pytest

from gen import TRAIN_BATCH, make_training_histories, make_workload
from oracle import sparse_batch as SB
from oracle import stca_oracle as O
from tests.gpu_helpers import TOL, normwise_err, storage_weights

pytestmark = pytest.mark.gpu


def _dev(th, a, device):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(th.storage(a)))
    if th.dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.to(device)


def _bits(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy().view(np.uint32)


def _want_bits(th, a):
    s = th.storage(a)
    return s if th.dtype == "bf16" else s.view(np.uint32)


def _build(th, device, L_min, L_max, L_avg, L_infer):
    import torch
    import target_attention_jagged_b200 as S
    X = _dev(th, th.X, device)
    Xp, seg, plan = S.build_training_batch(X, th.hist_offsets, th.s, L_min, L_max, L_avg, L_infer)
    torch.cuda.synchronize()
    return Xp, seg, plan


@pytest.mark.parametrize("dtype,d,B,hist,L", [
    ("bf16", 256, 37, ("lognormal", 900.0, 0.8, 1, 4000), (16, 2048, 320, 2048)),
    ("f32", 64, 9, [1, 2, 3, 700, 5, 6, 1000, 8, 9], (8, 512, 96, 300)),
    ("bf16", 8, 5, [1, 17, 40, 3, 200], (8, 64, 24, 48)),          # 16-byte rows
    ("bf16", 128, 1, [5000], (64, 4096, 1000, 3000)),              # one user
    ("f32", 520, 6, [50, 60, 70, 80, 90, 100], (8, 128, 40, 128)), # rows longer than 32 vectors
])
def test_gather_bit_exact(gpu, dtype, d, B, hist, L):
    L_min, L_max, L_avg, L_infer = L
    beta = SB.beta_for_mean(0.3, L_min, L_max, L_avg)
    th = make_training_histories(B=B, hist=hist, d=d, alpha=0.3, beta=beta, dtype=dtype,
                                 seed=B + d)
    Xp, seg, plan = _build(th, gpu, L_min, L_max, L_avg, L_infer)
    want = SB.plan_batch(th.hist_offsets, th.s, L_min, L_max, L_avg, L_infer)
    assert plan["packed_offsets"].tolist() == want["packed_offsets"].tolist()
    assert np.array_equal(_bits(Xp), _want_bits(th, SB.gather_packed(th.X, want)))
    assert np.array_equal(seg.cpu().numpy().astype(np.int64), want["seg"])


def test_training_batch_workload(gpu):
    """The full sparse-training batch (B = 256, L_avg = 2000, alpha = 0.02, d = 256):
    every packed row and index bit-exact."""
    cfg = TRAIN_BATCH
    beta = SB.beta_for_mean(cfg["alpha"], cfg["L_min"], cfg["L_max"], cfg["L_avg"])
    th = make_training_histories(B=cfg["B"], hist=cfg["hist"], d=cfg["d"], alpha=cfg["alpha"],
                                 beta=beta, dtype=cfg["dtype"], seed=cfg["seed"])
    args = (cfg["L_min"], cfg["L_max"], cfg["L_avg"], cfg["L_infer"])
    Xp, seg, plan = _build(th, gpu, *args)
    want = SB.plan_batch(th.hist_offsets, th.s, *args)
    assert int(plan["packed_offsets"][-1]) == cfg["B"] * cfg["L_avg"]
    assert np.array_equal(_bits(Xp), _want_bits(th, SB.gather_packed(th.X, want)))
    assert np.array_equal(seg.cpu().numpy().astype(np.int64), want["seg"])


def test_out_of_range_source_rows_are_skipped(gpu):
    import torch
    import target_attention_jagged_b200 as S
    X = torch.arange(10 * 8, dtype=torch.float32, device=gpu).reshape(10, 8)
    src = torch.tensor([8, -3], dtype=torch.int64, device=gpu)     # user 0 runs past row 9
    poff = torch.tensor([0, 4, 6], dtype=torch.int64, device=gpu)
    Xp = torch.full((6, 8), -1.0, device=gpu)
    seg = torch.full((6,), 99, dtype=torch.int32, device=gpu)
    S.stca_sl_gather(X, src, poff, Xp, seg)
    torch.cuda.synchronize()
    assert seg.cpu().tolist() == [0, 0, -1, -1, -1, -1]
    assert torch.equal(Xp[:2].cpu(), X[8:10].cpu()) and bool((Xp[2:] == -1).all())


def test_forward_on_packed_batch(gpu):
    """Sparse training's forward: encode + forward over the packed stream with its
    offsets, targets per user (request-level batching), against the oracle on the
    same packed rows."""
    import torch
    import target_attention_jagged_b200 as S
    d, h, M, r = 128, 4, 2, 2
    L_min, L_max, L_avg, L_infer = 8, 2048, 400, 1500
    beta = SB.beta_for_mean(0.02, L_min, L_max, L_avg)
    th = make_training_histories(B=12, hist=("uniform", 50, 3000), d=d, alpha=0.02, beta=beta,
                                 seed=21)
    Xp, seg, plan = _build(th, gpu, L_min, L_max, L_avg, L_infer)
    lengths = plan["lengths"].tolist()
    # model weights and 8 targets per user, drawn for the packed lengths
    wl = make_workload(lengths=lengths, targets=[8] * len(lengths), d=d, h=h, M=M, r=r,
                       dtype="bf16", seed=22)
    st = S.Stca(storage_weights(wl), d, h, r, M, "bf16")
    try:
        xt = _dev(th, wl.targets, gpu)
        st.encode(Xp, plan["packed_offsets"])
        Z = torch.full((wl.T, M, d), float("nan"), dtype=torch.float32, device=gpu)
        st.forward(xt, wl.target_offsets, Z)
        torch.cuda.synchronize()
        st.status()
        got = Z.cpu().numpy()
    finally:
        st.close()
    Xpk = SB.gather_packed(th.X, SB.plan_batch(th.hist_offsets, th.s, L_min, L_max, L_avg, L_infer))
    want = O.forward(Xpk, plan["packed_offsets"], wl.targets, wl.target_offsets, wl.weights, h)
    err = normwise_err(got, want)
    assert err <= TOL["bf16"], f"packed-batch forward normwise error {err:.3e}"
