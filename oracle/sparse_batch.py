"""Plain CPU oracle of the sparse-training batch builder -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
legs may import or run this module.  The product path (the CUDA library and its
Python binding) never calls it and shares no code with it.

Sources (the pages this follows):
  [digest]  "Make It Long, Keep It Fast: End-to-End 10k-Sequence Modeling at
            Billion Scale on Douyin" (paper digest), §2.3 "Extrapolation: Train
            Sparsely, Infer Densely": Stochastic Length Sampling (Eqs. (15)-(17)),
            the element-selection strategy, and the batch-level load balance.
  [blog]    "字节跳动-STCA：抖音 10k 长序列端到端建模的架构、系统与外推三件套"
            (STCA blog), §2.6 (random-length curriculum and load balance),
            §3.3 (Tables 4 and 5).

What it builds, for a batch of B users with full histories (rows of X, oldest
first, user b owning rows hist_offsets[b] .. hist_offsets[b+1]-1):
  1. a training length per user from a Beta draw s_b (Eq. (16)), aligned to
     a multiple of 8;
  2. the temporal suffix: the most recent L rows of the history, itself first
     cut to its most recent L_infer rows;
  3. the batch-level load balance: (a) the lengths are adjusted so the batch
     holds exactly B * L_avg tokens, (b) the suffixes are packed back to back
     into one padding-free token stream, which read as rows of L_avg tokens is
     the compacted [B, L_avg] batch, with an index tensor giving each packed
     row's user (the segment boundaries the ragged attention reads).
Integers are exact (Python ints); the one floating-point step (Eq. (16)) is
float64, as is the decision it feeds (the floor).

Readings taken where the pages are silent or garbled:
  S1  Random numbers are inputs: the caller draws s_b ~ Beta(alpha, beta) with
      beta from Eq. (17); this module never draws.
  S2  "Aligned to a multiple of 8" is read as rounding down:
      L_b = 8 * floor(L_raw_b / 8), and at least 8.  L_raw is evaluated as
      L_min + s * (L_max - L_min) in float64, in that order.
  S3  A user's usable history is its most recent min(H_b, L_infer) rows; a
      length above that is cut to it.  Histories are stored oldest first, so
      the temporal suffix is the last rows of the user's segment.  H_b >= 1 is
      required (an empty history has no softmax).
  S4  Step (a) of the load balance: with S = sum of the lengths and budget
      T = B * L_avg,
        S > T:  every user keeps one row, and the other T - B rows are shared
                out in proportion to (L_b - 1) by the largest-remainder method
                (floor of each exact quota, then one more row to the users with
                the largest remainders, ties to the lower index), so no length
                grows and the total is exactly T;
        S < T:  the T - S missing rows are shared out the same way in
                proportion to each user's unused history (usable - L_b); if the
                unused history cannot cover them, every user takes all of its
                usable history and the batch holds fewer than T tokens;
        S = T:  unchanged.
      The pages call this step a random truncation without saying which rows
      go; the proportional share is the plainest exact rule that keeps the
      sampled mix of short and long windows.
  S5  Step (b): the packed stream concatenates the users' suffixes in user
      order; packed row p belongs to user seg[p]; read as rows of L_avg tokens
      a long user's rows run on into the next rows, so no row is padding.
"""
from __future__ import annotations

import math

import numpy as np

ALIGN = 8


def beta_for_mean(alpha, L_min, L_max, L_avg):
    """Eq. (17): the Beta shape beta that makes E[L_raw] = L_avg under Eq. (16)."""
    if not (L_min < L_avg < L_max):
        raise ValueError("need L_min < L_avg < L_max")
    return alpha * (L_max - L_avg) / (L_avg - L_min)


def sequence_sparsity(L_avg, L_max):
    """Eq. (15): SS = E[L_train] / L_max = L_avg / L_max."""
    return L_avg / L_max


def raw_length(s, L_min, L_max):
    """Eq. (16): L_raw = L_min + s (L_max - L_min), float64 (reading S2)."""
    return np.float64(L_min) + np.float64(s) * np.float64(L_max - L_min)


def train_length(s, L_min, L_max):
    """Eq. (16) aligned down to a multiple of 8, at least 8 (reading S2)."""
    raw = float(raw_length(s, L_min, L_max))
    return max(ALIGN, (math.floor(raw) // ALIGN) * ALIGN)


def largest_remainder(weights, total):
    """Split the integer `total` in proportion to non-negative integer weights:
    floor of each exact quota w_b total / W, then +1 to the `total - sum(floors)`
    users with the largest remainders (ties to the lower index)."""
    weights = [int(w) for w in weights]
    W = sum(weights)
    if total == 0:
        return [0] * len(weights)
    if W <= 0:
        raise ValueError("no weight to share rows by")
    quota = [w * total // W for w in weights]
    rem = [w * total % W for w in weights]
    left = total - sum(quota)
    for b in sorted(range(len(weights)), key=lambda i: (-rem[i], i))[:left]:
        quota[b] += 1
    return quota


def balance_lengths(lengths, usable, budget):
    """Step (a) of the batch-level load balance (reading S4)."""
    lengths = [int(x) for x in lengths]
    usable = [int(x) for x in usable]
    B = len(lengths)
    S = sum(lengths)
    if S > budget:
        if budget < B:
            raise ValueError("budget below one row per user")
        share = largest_remainder([x - 1 for x in lengths], budget - B)
        return [1 + x for x in share]
    if S < budget:
        spare = [u - x for u, x in zip(usable, lengths)]
        if sum(spare) <= budget - S:
            return list(usable)
        share = largest_remainder(spare, budget - S)
        return [x + y for x, y in zip(lengths, share)]
    return lengths


def plan_batch(hist_offsets, s, L_min, L_max, L_avg, L_infer):
    """Lengths and packed layout of one training batch.

    Returns a dict of int64 arrays: `train` (Eq. (16) aligned, per user),
    `lengths` (after the load balance), `packed_offsets` (B+1), `src_start`
    (first history row of each user's suffix), and `seg` (user of each packed
    row)."""
    off = [int(x) for x in hist_offsets]
    B = len(off) - 1
    if len(s) != B:
        raise ValueError("one draw per user")
    hist = [off[b + 1] - off[b] for b in range(B)]
    if min(hist) < 1:
        raise ValueError("empty history")
    usable = [min(hb, int(L_infer)) for hb in hist]
    train = [train_length(s[b], L_min, L_max) for b in range(B)]
    capped = [min(t, u) for t, u in zip(train, usable)]
    lengths = balance_lengths(capped, usable, B * int(L_avg))
    packed = [0]
    for x in lengths:
        packed.append(packed[-1] + x)
    src_start = [off[b + 1] - lengths[b] for b in range(B)]
    seg = np.repeat(np.arange(B, dtype=np.int64), lengths)
    as64 = lambda v: np.asarray(v, dtype=np.int64)  # noqa: E731
    return {"hist_offsets": as64(off), "train": as64(train), "usable": as64(usable),
            "capped": as64(capped), "lengths": as64(lengths), "packed_offsets": as64(packed),
            "src_start": as64(src_start), "seg": seg}


def gather_packed(X, plan):
    """The packed token stream: user b's suffix rows src_start[b] .. +lengths[b]-1
    of X, users back to back (reading S5).  A plain copy: rows keep their bits."""
    X = np.asarray(X)
    parts = [X[int(a):int(a) + int(n)] for a, n in zip(plan["src_start"], plan["lengths"])]
    return np.concatenate(parts, axis=0) if parts else X[:0]
