"""The batch builder's host plan through the C ABI (stca_sl_beta, stca_sl_plan),
bit-exact against the oracle (oracle/sparse_batch.py) on seeded inputs: no GPU
needed.  The same integers must come out of both: the training lengths of
Eq. (16), the load-balanced lengths, the packed offsets and the suffix starts."""
import json
import os

import numpy as np
import pytest

import target_attention_jagged_b200 as S
from gen import TRAIN_BATCH, make_training_histories
from oracle import sparse_batch as SB

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
KEYS = ("train", "lengths", "packed_offsets", "src_start")


def _same(p, q):
    for k in KEYS:
        assert p[k].tolist() == q[k].tolist(), k


def test_worked_examples_through_the_abi():
    with open(os.path.join(GOLDEN, "sl_worked_examples.json")) as f:
        for ex in json.load(f)["examples"]:
            p = S.stca_sl_plan(ex["hist_offsets"], ex["s"], ex["L_min"], ex["L_max"],
                               ex["L_avg"], ex["L_infer"])
            for k in KEYS:
                assert p[k].tolist() == ex[k], (ex["what"], k)


@pytest.mark.parametrize("alpha", [0.02, 0.5, 10.0])
def test_beta_and_sparsity(alpha):
    beta, ss = S.stca_sl_beta(alpha, 64, 10000, 2000)
    assert beta == SB.beta_for_mean(alpha, 64, 10000, 2000)
    assert ss == SB.sequence_sparsity(2000, 10000)


def test_training_batch_workload_plan():
    cfg = TRAIN_BATCH
    beta = SB.beta_for_mean(cfg["alpha"], cfg["L_min"], cfg["L_max"], cfg["L_avg"])
    th = make_training_histories(B=cfg["B"], hist=cfg["hist"], d=8, alpha=cfg["alpha"],
                                 beta=beta, seed=cfg["seed"], with_x=False)
    args = (cfg["L_min"], cfg["L_max"], cfg["L_avg"], cfg["L_infer"])
    p = S.stca_sl_plan(th.hist_offsets, th.s, *args)
    _same(p, SB.plan_batch(th.hist_offsets, th.s, *args))
    assert int(p["packed_offsets"][-1]) == cfg["B"] * cfg["L_avg"]


@pytest.mark.parametrize("seed", range(12))
def test_random_batches_match_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 80))
    H = rng.integers(1, 3000, size=B)
    off = np.concatenate([[0], np.cumsum(H)]).astype(np.int64)
    L_min = int(rng.integers(0, 200))
    L_max = int(rng.integers(L_min + 16, 5000))
    L_avg = int(rng.integers(L_min + 1, L_max))
    L_infer = int(rng.integers(1, 6000))
    alpha = float(10 ** rng.uniform(-2, 1))
    s = rng.beta(alpha, SB.beta_for_mean(alpha, L_min, L_max, L_avg), size=B)
    if seed % 3 == 0:
        s[: B // 2] = rng.choice([0.0, 1.0], size=B // 2)     # the interval's ends
    _same(S.stca_sl_plan(off, s, L_min, L_max, L_avg, L_infer),
          SB.plan_batch(off, s, L_min, L_max, L_avg, L_infer))


def test_plan_rejects_bad_input():
    ok = dict(L_min=8, L_max=64, L_avg=32, L_infer=64)
    bad = [
        ([0, 5, 5], [0.5, 0.5], ok),                               # empty history
        ([1, 5], [0.5], ok),                                       # offsets[0] != 0
        ([0, 5], [1.5], ok),                                       # s outside [0, 1]
        ([0, 5], [float("nan")], ok),
        ([0, 5], [0.5], dict(ok, L_avg=8)),                        # L_avg == L_min
        ([0, 5], [0.5], dict(ok, L_avg=64)),                       # L_avg == L_max
        ([0, 5], [0.5], dict(ok, L_infer=0)),
    ]
    for off, s, kw in bad:
        with pytest.raises(S.StcaError):
            S.stca_sl_plan(off, s, kw["L_min"], kw["L_max"], kw["L_avg"], kw["L_infer"])
    with pytest.raises(S.StcaError):
        S.stca_sl_beta(0.0, 8, 64, 32)


def test_gather_rejects_bad_arguments_on_host():
    lib = S.stca._lib
    assert lib.stca_sl_gather(None, 4, 32, None, None, 1, 4, None, None, None) == S.stca.STCA_EINVAL
    assert lib.stca_sl_gather(16, 4, 24, 16, 16, 1, 4, 16, None, None) == S.stca.STCA_EINVAL  # row bytes
    assert lib.stca_sl_gather(8, 4, 32, 16, 16, 1, 4, 16, None, None) == S.stca.STCA_EINVAL   # alignment
