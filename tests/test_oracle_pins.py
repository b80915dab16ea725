"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test checks the oracle against a fact that the STCA pages or the
mathematics fix: brute force on tiny inputs, the PyTorch library routines,
closed forms, the structural invariants of single-query target attention, and
the one number the pages print about the method's arithmetic (the ~64x
reordering saving).  tests/test_oracle_mutations.py checks that a plausible
mistake planted in the oracle fails at least one of these.
"""
import json
import math
import os

import numpy as np
import pytest

from gen import make_workload
from oracle import stca_oracle as O
from tests import bruteforce, torch_reference

HERE = os.path.dirname(os.path.abspath(__file__))


def rel_err(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def tiny(seed, L, T, d, h, M, r, **kw):
    return make_workload(lengths=[L], targets=[T], d=d, h=h, M=M, r=r, dtype="f32",
                         seed=seed, **kw)


# ---------------------------------------------------------------- brute force

TINY = [
    # (seed, L, T, d, h, M, r, extra)
    (0, 1, 1, 2, 1, 1, 1, {}),
    (1, 3, 2, 4, 2, 2, 1, {}),
    (2, 4, 1, 4, 1, 3, 2, {"random_ln": True}),
    (3, 2, 3, 4, 2, 3, 2, {"random_ln": True, "distinct_query_ffn": True}),
    (4, 4, 2, 4, 4, 2, 1, {"distinct_query_ffn": True}),
]


@pytest.mark.parametrize("case", TINY)
def test_bruteforce_tiny(case):
    seed, L, T, d, h, M, r, kw = case
    wl = tiny(seed, L, T, d, h, M, r, **kw)
    got = O.forward_request(wl.X, wl.targets, wl.weights, h)
    want = np.asarray(bruteforce.forward_request(wl.X, wl.targets, wl.weights, h))
    assert got.shape == (T, M, d)
    assert rel_err(got, want) < 1e-12


def test_bruteforce_scaled_up_keys():
    # larger weights make the softmax sharp: checks the max-subtraction path
    wl = tiny(7, 4, 2, 4, 2, 2, 1)
    for k in ("Wq", "Wk"):
        wl.weights[k] = [w * 8.0 for w in wl.weights[k]]
    got = O.forward_request(wl.X, wl.targets, wl.weights, 2)
    want = np.asarray(bruteforce.forward_request(wl.X, wl.targets, wl.weights, 2))
    assert rel_err(got, want) < 1e-11


# ---------------------------------------------------- library cross-check

@pytest.mark.parametrize("kw", [
    dict(L=37, T=5, d=16, h=4, M=3, r=2, seed=11),
    dict(L=200, T=3, d=32, h=8, M=2, r=4, seed=12, random_ln=True, distinct_query_ffn=True),
    dict(L=1, T=2, d=8, h=2, M=2, r=1, seed=13),
])
def test_torch_library_crosscheck(kw):
    kw = dict(kw)
    L, T, d, h, M, r, seed = (kw.pop(k) for k in ("L", "T", "d", "h", "M", "r", "seed"))
    wl = tiny(seed, L, T, d, h, M, r, **kw)
    got = O.forward_request(wl.X, wl.targets, wl.weights, h)
    want = torch_reference.forward_request(wl.X, wl.targets, wl.weights, h)
    assert rel_err(got, want) < 1e-11


def test_silu_and_sigmoid_match_torch():
    import torch
    z = np.concatenate([np.linspace(-800, 800, 4001), np.linspace(-5, 5, 1001)])
    assert np.allclose(O.sigmoid(z), torch.sigmoid(torch.tensor(z)).numpy(), rtol=1e-15, atol=1e-300)
    assert np.allclose(O.silu(z), torch.nn.functional.silu(torch.tensor(z)).numpy(),
                       rtol=1e-14, atol=1e-300)


def test_layer_norm_matches_torch():
    import torch
    rng = np.random.default_rng(5)
    y = rng.standard_normal((9, 24)) * 3 + 1
    g, b = rng.uniform(0.5, 1.5, 24), rng.uniform(-1, 1, 24)
    want = torch.nn.functional.layer_norm(torch.tensor(y), (24,), torch.tensor(g),
                                          torch.tensor(b), 1e-5).numpy()
    assert rel_err(O.layer_norm(y, g, b), want) < 1e-14


# ------------------------------------------------ the two attention forms

@pytest.mark.parametrize("L,d,h,T", [(1, 8, 2, 1), (50, 16, 4, 3), (333, 64, 2, 2), (129, 32, 8, 5)])
def test_naive_equals_reordered(L, d, h, T):
    """Eq. (12) and Eq. (13) are the same function by associativity."""
    rng = np.random.default_rng(L * 7 + d)
    q = rng.standard_normal((T, d))
    Xt = rng.standard_normal((L, d))
    Ws = [rng.uniform(-1, 1, (d, d)) / math.sqrt(d) for _ in range(4)]
    a = O.attention_naive(q, Xt, *Ws, h)
    b = O.attention_reordered(q, Xt, *Ws, h)
    assert rel_err(b, a) < 1e-12


def test_softmax_rows_sum_to_one_and_shape():
    rng = np.random.default_rng(3)
    d, h, L, T = 32, 4, 77, 6
    q, Xt = rng.standard_normal((T, d)), rng.standard_normal((L, d))
    Ws = [rng.uniform(-1, 1, (d, d)) for _ in range(4)]
    _, alphas = O.attention_reordered(q, Xt, *Ws, h, return_alpha=True)
    assert len(alphas) == h
    for a in alphas:
        assert a.shape == (T, L)           # one query row per target: 1 x L each
        assert np.all(a >= 0)
        assert np.abs(a.sum(axis=-1) - 1.0).max() < 1e-13


# --------------------------------------------------------------- closed forms

def test_single_token_history_closed_form():
    """With L = 1 the softmax is [1], so o = x~ W_V W_O whatever the query."""
    for seed in range(3):
        wl = tiny(20 + seed, 1, 4, 16, 4, 3, 2, random_ln=True)
        Z = O.forward_request(wl.X, wl.targets, wl.weights, 4)
        W = wl.weights
        for i in range(3):
            xt_i = O.encode_history(wl.X, W, i)[0]
            want = xt_i @ W["Wv"][i].astype(np.float64) @ W["Wo"][i].astype(np.float64)
            for k in range(4):
                assert rel_err(Z[k, i], want) < 1e-12


def test_zero_query_projection_gives_mean():
    """W_Q = 0 makes every score 0: alpha is uniform and o = mean(X~) W_V W_O."""
    wl = tiny(30, 23, 2, 16, 2, 2, 2)
    W = wl.weights
    W["Wq"] = [np.zeros_like(w) for w in W["Wq"]]
    Z = O.forward_request(wl.X, wl.targets, W, 2)
    for i in range(2):
        Xt = O.encode_history(wl.X, W, i)
        want = Xt.mean(axis=0) @ W["Wv"][i].astype(np.float64) @ W["Wo"][i].astype(np.float64)
        assert rel_err(Z[0, i], want) < 1e-12
        assert rel_err(Z[1, i], want) < 1e-12


def test_hard_selection_limit():
    """Scaling the scores up makes each head select its argmax token."""
    rng = np.random.default_rng(9)
    d, h, L = 16, 4, 40
    dh = d // h
    q = rng.standard_normal((1, d))
    Xt = rng.standard_normal((L, d))
    Wq, Wk, Wv = (rng.uniform(-1, 1, (d, d)) for _ in range(3))
    Wo = np.eye(d)
    o = O.attention_reordered(q, Xt, Wq * 1e6, Wk, Wv, Wo, h)
    for j in range(h):
        c = slice(j * dh, (j + 1) * dh)
        scores = Xt @ (Wk[:, c] @ (q[0] @ Wq[:, c]))
        k = int(np.argmax(scores))
        assert np.allclose(o[0, c], Xt[k] @ Wv[:, c], rtol=1e-9, atol=1e-12)


def test_zero_gate_gives_beta():
    """W_g = 0 makes SiLU(0) = 0, the FFN output 0, and LN(0) = beta exactly."""
    wl = tiny(40, 9, 1, 8, 2, 2, 2, random_ln=True)
    W = wl.weights
    W["Wg"] = [np.zeros_like(w) for w in W["Wg"]]
    for i in range(2):
        Xt = O.encode_history(wl.X, W, i)
        assert np.array_equal(Xt, np.broadcast_to(W["ln_b"][i].astype(np.float64), Xt.shape))


def test_constant_row_layer_norm_is_beta():
    g, b = np.full(6, 2.0), np.arange(6.0)
    assert np.array_equal(O.layer_norm(np.full((3, 6), 4.25), g, b), np.broadcast_to(b, (3, 6)))


def test_fusion_keeps_raw_target_last():
    """Eq. (7) with W_C^(2) = [0; I] selects x_t: q^(2) = FFN^(2)(x_t)."""
    d, h = 8, 2
    wl = tiny(50, 11, 3, d, h, 2, 2)
    W = wl.weights
    W["Wc"][1] = np.concatenate([np.zeros((d, d)), np.eye(d)]).astype(np.float32)
    Z = O.forward_request(wl.X, wl.targets, W, h)
    q2 = O.swiglu_ffn(wl.targets, W["Wu"][1], W["Wg"][1], W["Wd"][1])
    Xt2 = O.encode_history(wl.X, W, 1)
    want = O.attention_naive(q2, Xt2, W["Wq"][1], W["Wk"][1], W["Wv"][1], W["Wo"][1], h)
    assert rel_err(Z[:, 1], want) < 1e-12
    # and with W_C^(2) = [I; 0] the second layer's query is FFN^(2)(o^(1))
    W["Wc"][1] = np.concatenate([np.eye(d), np.zeros((d, d))]).astype(np.float32)
    Z = O.forward_request(wl.X, wl.targets, W, h)
    q2 = O.swiglu_ffn(Z[:, 0], W["Wu"][1], W["Wg"][1], W["Wd"][1])
    want = O.attention_naive(q2, Xt2, W["Wq"][1], W["Wk"][1], W["Wv"][1], W["Wo"][1], h)
    assert rel_err(Z[:, 1], want) < 1e-12


# ---------------------------------------------------------------- invariants

def test_history_permutation_invariance():
    """Each history token is handled independently given the target (blog,
    appendix on generalisation): reordering the history leaves Z unchanged."""
    wl = tiny(60, 57, 4, 16, 4, 3, 2, random_ln=True)
    Z = O.forward_request(wl.X, wl.targets, wl.weights, 4)
    perm = np.random.default_rng(1).permutation(57)
    Zp = O.forward_request(wl.X[perm], wl.targets, wl.weights, 4)
    assert rel_err(Zp, Z) < 1e-12


def test_history_duplication_invariance():
    """Duplicating every token doubles each exp-sum term alike: Z unchanged."""
    wl = tiny(61, 31, 2, 16, 2, 2, 2)
    Z = O.forward_request(wl.X, wl.targets, wl.weights, 2)
    Zd = O.forward_request(np.repeat(wl.X, 2, axis=0), wl.targets, wl.weights, 2)
    assert rel_err(Zd, Z) < 1e-12


def test_batch_and_target_independence():
    wl = make_workload(lengths=[5, 17, 1, 40], targets=[2, 0, 3, 1], d=16, h=4, M=2, r=2,
                       dtype="f32", seed=70)
    Z = O.forward_workload(wl)
    assert Z.shape == (6, 2, 16)
    # each request alone
    for r in range(4):
        Xr, tr = wl.request(r)
        lo, hi = wl.target_offsets[r], wl.target_offsets[r + 1]
        if hi > lo:
            assert rel_err(O.forward_request(Xr, tr, wl.weights, 4), Z[lo:hi]) < 1e-15
            # each target alone
            for k in range(hi - lo):
                one = O.forward_request(Xr, tr[k:k + 1], wl.weights, 4)
                assert rel_err(one[0], Z[lo + k]) < 1e-12
    # requests in reverse order
    order = [3, 2, 1, 0]
    X2 = np.concatenate([wl.request(r)[0] for r in order])
    t2 = np.concatenate([wl.request(r)[1] for r in order])
    L2 = wl.lengths[order]
    T2 = wl.target_counts[order]
    off2 = np.concatenate([[0], np.cumsum(L2)])
    toff2 = np.concatenate([[0], np.cumsum(T2)])
    Z2 = O.forward(X2, off2, t2, toff2, wl.weights, 4)
    for new_r, r in enumerate(order):
        a = Z2[toff2[new_r]:toff2[new_r + 1]]
        b = Z[wl.target_offsets[r]:wl.target_offsets[r + 1]]
        assert a.shape == b.shape and (a.size == 0 or rel_err(a, b) < 1e-15)


def test_empty_history_rejected_and_no_target_rows():
    wl = tiny(80, 3, 0, 8, 2, 1, 1)
    assert O.forward_request(wl.X, wl.targets, wl.weights, 2).shape == (0, 1, 8)
    with pytest.raises(ValueError):
        O.forward_request(wl.X[:0], np.ones((1, 8)), wl.weights, 2)


# ---------------------------------------------------------- the page's number

def test_reordering_saving_matches_page():
    with open(os.path.join(HERE, "golden", "reordering_saving.json")) as f:
        fx = json.load(f)
    for c in fx["cases"]:
        assert c["d"] // c["h"] == c["d_h"]
        assert O.reordering_saving_factor(c["d"], c["h"]) == c["saving"]


def test_length_flop_model():
    # the full reordered count per head (scores + alpha X~ over d) is 4 L d;
    # the naive one is dominated by the 4 L d d_h projection term
    for d, h in [(256, 8), (128, 8), (64, 2)]:
        dh = d // h
        n = O.attention_length_flops(1000, d, h, "naive")
        r = O.attention_length_flops(1000, d, h, "reordered")
        assert r == 4 * 1000 * d * h
        assert n == h * 1000 * (4 * d * dh + 4 * dh)
        assert abs(n / r - dh) < 1e-9 * dh + dh / d


# ------------------------------------------------------------ prediction head, Eq. (9)

def _z_of(wl):
    Z = O.forward_request(wl.X, wl.targets, wl.weights, wl.h)
    return Z, O.head_from_outputs(Z, wl.targets, wl.weights)


@pytest.mark.parametrize("seed,M,r", [(21, 1, 1), (22, 2, 2), (23, 3, 1)])
def test_head_bruteforce_tiny(seed, M, r):
    wl = make_workload(lengths=[3], targets=[2], d=4, h=2, M=M, r=r, dtype="f32", seed=seed)
    Z, z = _z_of(wl)
    want = np.array([bruteforce.prediction_head([Z[t, i] for i in range(M)], wl.targets[t],
                                                wl.weights) for t in range(2)])
    assert z.shape == (2, 4)
    assert np.abs(z - want).max() <= 1e-12 * max(1.0, np.abs(want).max())


def test_head_torch_library_crosscheck():
    wl = make_workload(lengths=[30], targets=[5], d=16, h=4, M=3, r=2, dtype="f32", seed=24)
    Z, z = _z_of(wl)
    want = torch_reference.prediction_head(Z, wl.targets, wl.weights)
    assert np.abs(z - want).max() <= 1e-12 * np.abs(want).max()


def test_head_block_order():
    # W_Z with one nonzero row block: z then depends on that block's input alone.
    # Blocks are o(1), ..., o(M), then x_t (Eq. (9)).
    wl = make_workload(lengths=[10], targets=[3], d=8, h=2, M=3, r=1, dtype="f32", seed=25)
    d, M = 8, 3
    Z, _ = _z_of(wl)
    rng = np.random.default_rng(0)
    for blk in range(M + 1):
        W = dict(wl.weights)
        Wz = np.zeros_like(np.asarray(W["Wz"], dtype=np.float64))
        Wz[blk * d:(blk + 1) * d] = np.asarray(wl.weights["Wz"])[blk * d:(blk + 1) * d]
        W["Wz"] = Wz
        base = O.head_from_outputs(Z, wl.targets, W)
        for other in range(M + 1):
            Z2, xt2 = Z.copy(), np.array(wl.targets, dtype=np.float64)
            if other < M:
                Z2[:, other] += rng.standard_normal((3, d))
            else:
                xt2 += rng.standard_normal((3, d))
            moved = np.abs(O.head_from_outputs(Z2, xt2, W) - base).max()
            if other == blk:
                assert moved > 1e-6, (blk, other)
            else:
                assert moved == 0.0, (blk, other)
