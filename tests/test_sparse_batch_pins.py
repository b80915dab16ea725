"""Pins of the sparse-training batch builder oracle (oracle/sparse_batch.py)
against what the pages and the mathematics fix, not against itself:

  * Eq. (17) against the Beta distribution's closed-form mean and against
    numpy's Beta sampler (E[L_raw] = L_avg under Eq. (16));
  * Eq. (15) against the sparsities the pages print in Table 4;
  * Eq. (17) against the curriculum shapes Table 5 names for its alphas;
  * the aligned length of Eq. (16) against an exact-rational brute force;
  * the largest-remainder share against an independent Fraction version;
  * the load balance against its defining properties and hand-worked examples;
  * the temporal suffix and the packing against row identities.
A mutation test plants plausible mistakes and checks that these pins fail.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from gen import make_training_histories
from oracle import sparse_batch as SB

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------- Eqs. (15)-(17)

def pin_beta_mean():
    rng = np.random.default_rng(1)
    for _ in range(200):
        L_min = int(rng.integers(0, 500))
        L_max = int(rng.integers(L_min + 10, 30000))
        L_avg = int(rng.integers(L_min + 1, L_max))
        alpha = float(10 ** rng.uniform(-2, 1.5))
        beta = SB.beta_for_mean(alpha, L_min, L_max, L_avg)
        mean_s = alpha / (alpha + beta)                # textbook mean of Beta(alpha, beta)
        assert math.isclose(L_min + mean_s * (L_max - L_min), L_avg, rel_tol=1e-12)


def pin_beta_sampling():
    rng = np.random.default_rng(2)
    for alpha, L_min, L_max, L_avg in [(0.02, 64, 10000, 2000), (0.5, 0, 10000, 2000),
                                       (10.0, 100, 4000, 1000)]:
        beta = SB.beta_for_mean(alpha, L_min, L_max, L_avg)
        s = rng.beta(alpha, beta, size=400_000)
        raw = np.asarray(SB.raw_length(s, L_min, L_max), dtype=np.float64)
        se = raw.std() / math.sqrt(raw.size)
        assert abs(raw.mean() - L_avg) < 5 * se + 1e-9
        # Eq. (15): the mean training length over L_max is the sparsity
        assert abs(raw.mean() / L_max - SB.sequence_sparsity(L_avg, L_max)) < 5 * se / L_max + 1e-12


def pin_table4():
    g = _golden("sl_table4_sparsity.json")
    for row in g["rows"]:
        assert round(100 * SB.sequence_sparsity(row["L_avg"], g["L_max"]), 9) == row["SS_percent"]


def _shape(a, b):
    if a < 1 and b < 1:
        return "u"
    if a <= 1 < b:
        return "decreasing"
    if a > 1 and b > 1:
        return "unimodal"
    return "other"


def pin_table5():
    g = _golden("sl_table5_shapes.json")
    for row in g["rows"]:
        for L_min in g["L_min_range"]:
            b = SB.beta_for_mean(row["alpha"], L_min, g["L_max"], g["L_avg"])
            assert _shape(row["alpha"], b) == row["shape"], (row, L_min, b)


def test_beta_mean_closed_form():
    pin_beta_mean()


def test_beta_sampling_matches_target_mean():
    pin_beta_sampling()


def test_sparsity_matches_table4():
    pin_table4()


def test_beta_shapes_match_table5():
    pin_table5()


# ------------------------------------------------------------- Eq. (16) alignment

def pin_train_length():
    rng = np.random.default_rng(3)
    for _ in range(3000):
        L_min = int(rng.integers(0, 300))
        L_max = int(rng.integers(L_min + 1, 20000))
        s = float(rng.random())
        exact = Fraction(L_min) + Fraction(s) * (L_max - L_min)
        if abs(exact - round(exact / 8) * 8) < Fraction(1, 10 ** 6):
            continue                   # a float64 rounding could land either side of a multiple
        want = 0
        while want + 8 <= exact:       # largest multiple of 8 not above the exact L_raw
            want += 8
        want = max(8, want)
        assert SB.train_length(s, L_min, L_max) == want
    assert SB.train_length(0.0, 0, 100) == 8          # never below one aligned block
    assert SB.train_length(1.0, 0, 10000) == 10000


def test_train_length_bruteforce():
    pin_train_length()


# ------------------------------------------------------------- load balance

def hamilton(weights, total):
    """Largest-remainder (Hamilton) apportionment with exact fractions."""
    W = sum(weights)
    q = [Fraction(w * total, W) for w in weights]
    base = [math.floor(x) for x in q]
    order = sorted(range(len(q)), key=lambda i: (-(q[i] - base[i]), i))
    for i in order[:total - sum(base)]:
        base[i] += 1
    return base


def pin_largest_remainder():
    rng = np.random.default_rng(4)
    for _ in range(500):
        n = int(rng.integers(1, 40))
        w = [int(x) for x in rng.integers(0, 5000, size=n)]
        if sum(w) == 0:
            w[0] = 1
        total = int(rng.integers(0, 100000))
        assert SB.largest_remainder(w, total) == hamilton(w, total)
    # ties go to the lower index
    assert SB.largest_remainder([1, 1, 1], 2) == [1, 1, 0]


def pin_balance_properties():
    rng = np.random.default_rng(5)
    for _ in range(500):
        B = int(rng.integers(1, 30))
        usable = [int(x) for x in rng.integers(1, 3000, size=B)]
        lengths = [int(rng.integers(1, u + 1)) for u in usable]
        budget = int(rng.integers(B, 2 * sum(usable) + 2))
        out = SB.balance_lengths(lengths, usable, budget)
        S = sum(lengths)
        assert all(1 <= o <= u for o, u in zip(out, usable))
        if S > budget:
            assert sum(out) == budget and all(o <= x for o, x in zip(out, lengths))
            quota = [1 + Fraction((x - 1) * (budget - B), S - B) for x in lengths]
            assert all(abs(o - q) < 1 for o, q in zip(out, quota))
        elif S < budget:
            assert all(o >= x for o, x in zip(out, lengths))
            if sum(usable) >= budget:
                assert sum(out) == budget
            else:
                assert out == usable
        else:
            assert out == lengths


def pin_worked_examples():
    for ex in _golden("sl_worked_examples.json")["examples"]:
        p = SB.plan_batch(ex["hist_offsets"], ex["s"], ex["L_min"], ex["L_max"], ex["L_avg"],
                          ex["L_infer"])
        for k in ("train", "lengths", "packed_offsets", "src_start"):
            assert p[k].tolist() == ex[k], (ex["what"], k, p[k].tolist())


def pin_suffix_and_packing():
    rng = np.random.default_rng(6)
    for _ in range(50):
        B = int(rng.integers(1, 12))
        H = [int(x) for x in rng.integers(1, 400, size=B)]
        off = np.concatenate([[0], np.cumsum(H)])
        s = rng.random(B)
        p = SB.plan_batch(off, s, 8, 512, 96, 300)
        X = np.arange(int(off[-1]), dtype=np.int64)[:, None] * np.ones((1, 3), np.int64)
        Y = SB.gather_packed(X, p)
        assert Y.shape[0] == int(p["packed_offsets"][-1]) == p["seg"].shape[0]
        for b in range(B):
            n = int(p["lengths"][b])
            assert 1 <= n <= min(H[b], 300)
            rows = Y[int(p["packed_offsets"][b]):int(p["packed_offsets"][b + 1]), 0]
            # the most recent n rows of the user's history, oldest first
            assert rows.tolist() == list(range(int(off[b + 1]) - n, int(off[b + 1])))
            assert np.all(p["seg"][int(p["packed_offsets"][b]):int(p["packed_offsets"][b + 1])] == b)


def test_largest_remainder_matches_fractions():
    pin_largest_remainder()


def test_balance_properties():
    pin_balance_properties()


def test_worked_examples():
    pin_worked_examples()


def test_suffix_and_packing():
    pin_suffix_and_packing()


def test_plan_rejects_bad_input():
    with pytest.raises(ValueError):
        SB.plan_batch([0, 5, 5], [0.5, 0.5], 8, 64, 32, 64)       # empty history
    with pytest.raises(ValueError):
        SB.beta_for_mean(0.5, 100, 1000, 100)                     # L_avg at L_min
    with pytest.raises(ValueError):
        SB.plan_batch([0, 5], [0.5, 0.1], 8, 64, 32, 64)          # one draw per user


def test_generator_draws_are_inputs_only():
    # the generator takes beta from the caller; two seeds give different draws
    a = make_training_histories(B=4, hist=[5, 6, 7, 8], d=8, alpha=0.5, beta=2.0, seed=1)
    b = make_training_histories(B=4, hist=[5, 6, 7, 8], d=8, alpha=0.5, beta=2.0, seed=2)
    assert a.hist_offsets.tolist() == [0, 5, 11, 18, 26]
    assert not np.array_equal(a.s, b.s) and a.X.shape == (26, 8)


# ------------------------------------------------------------- mutations

def _align_up(s, L_min, L_max):
    raw = float(SB.raw_length(s, L_min, L_max))
    return max(8, int(math.ceil(raw / 8)) * 8)


def _align_nearest(s, L_min, L_max):
    raw = float(SB.raw_length(s, L_min, L_max))
    return max(8, int(round(raw / 8)) * 8)


def _beta_inverted(alpha, L_min, L_max, L_avg):
    return alpha * (L_avg - L_min) / (L_max - L_avg)


def _ss_inverted(L_avg, L_max):
    return L_max / L_avg


def _lr_ties_high(weights, total):
    W = sum(weights)
    q = [w * total // W for w in weights]
    rem = [w * total % W for w in weights]
    for b in sorted(range(len(q)), key=lambda i: (-rem[i], -i))[:total - sum(q)]:
        q[b] += 1
    return q


def _lr_round(weights, total):
    W = sum(weights)
    return [int(round(w * total / W)) for w in weights]


def _balance_waterfill(lengths, usable, budget):
    lengths = [int(x) for x in lengths]
    while sum(lengths) > budget:
        i = max(range(len(lengths)), key=lambda j: lengths[j])
        lengths[i] -= 1
    return lengths


_balance = SB.balance_lengths


def _balance_no_extend(lengths, usable, budget):
    if sum(int(x) for x in lengths) > budget:
        return _balance(lengths, usable, budget)
    return [int(x) for x in lengths]


def _gather_prefix(X, plan):
    off = plan["hist_offsets"]
    parts = [np.asarray(X)[int(off[b]):int(off[b]) + int(n)] for b, n in enumerate(plan["lengths"])]
    return np.concatenate(parts, axis=0)


MUTANTS = {
    "align_up": ("train_length", _align_up),
    "align_nearest": ("train_length", _align_nearest),
    "beta_inverted": ("beta_for_mean", _beta_inverted),
    "ss_inverted": ("sequence_sparsity", _ss_inverted),
    "remainder_ties_high": ("largest_remainder", _lr_ties_high),
    "remainder_rounding": ("largest_remainder", _lr_round),
    "balance_waterfill": ("balance_lengths", _balance_waterfill),
    "balance_no_extend": ("balance_lengths", _balance_no_extend),
    "gather_prefix": ("gather_packed", _gather_prefix),
}

PINS = [pin_beta_mean, pin_beta_sampling, pin_table4, pin_table5, pin_train_length,
        pin_largest_remainder, pin_balance_properties, pin_worked_examples,
        pin_suffix_and_packing]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(SB, attr, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, ZeroDivisionError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passes every pin"
