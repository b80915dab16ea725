"""Seeded synthetic STCA workloads.

Shapes follow the STCA pages: one request carries a user history of L
interaction tokens and T_r target videos that share it (request-level batching,
"Make It Long, Keep It Fast" digest §2.2; STCA blog §2.5).  The histories of
all requests are concatenated row-wise into one jagged buffer indexed by an
offsets tensor (the ragged target attention index, digest §2.3).

Recipe (the same for every configuration):
  * draw order: history lengths, target counts, X, targets, then the weights of
    layer 1..M in the order Wu, Wg, Wd, Wq, Wk, Wv, Wo, Wc (Wc from layer 2
    on), then the optional random LayerNorm affine, then the optional separate
    query-side FFN;
  * X and the target embeddings x_t are iid N(0, 1);
  * every stored weight matrix is Xavier-uniform, U(-a, a) with
    a = sqrt(6 / (fan_in + fan_out)) for its own (rows, cols);
  * LayerNorm gamma = 1 and beta = 0 unless random_ln is set;
  * bf16 configurations round every input and weight to bf16
    (round-to-nearest-even) here, so the oracle and the GPU see the same values.

Nothing in this module computes any part of the method.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# Named workloads.  Lengths: ("fixed", L) | ("uniform", lo, hi) |
# ("lognormal", mean, sigma, lo, hi) | ("list", [...]).  Targets per request:
# ("fixed", t) | ("1+poisson", lam) | ("list", [...]).
CONFIGS = {
    # one request, L=500, one target, d=64, h=2, M=1, r=2, fp32, seed 0
    "c1": dict(name="pr1-R1-L500-T1-d64-h2-M1-r2-f32", R=1, lengths=("fixed", 500),
               targets=("fixed", 1), d=64, h=2, M=1, r=2, dtype="f32", seed=0),
    # 32 requests, L ~ U[200, 2000], 4 targets each, d=128, h=4, M=2, r=2, bf16
    "c2": dict(name="ragged-R32-Lu200_2000-T4-d128-h4-M2-r2-bf16", R=32,
               lengths=("uniform", 200, 2000), targets=("fixed", 4), d=128, h=4, M=2,
               r=2, dtype="bf16", seed=1),
    # request-level-batched serving: 64 requests, L=10000, 16 targets each
    "c3": dict(name="rlb-serving-R64-L10000-T16-d128-h8-M3-r4-bf16", R=64,
               lengths=("fixed", 10000), targets=("fixed", 16), d=128, h=8, M=3, r=4,
               dtype="bf16", seed=2),
    # sparse-training mix: lognormal lengths (mean 2000) clipped to [100, 10000]
    "c4": dict(name="train-mix-R256-Llogn2000-T1pPois8-d256-h8-M4-r2-bf16", R=256,
               lengths=("lognormal", 2000.0, 1.0, 100, 10000), targets=("1+poisson", 8.0),
               d=256, h=8, M=4, r=2, dtype="bf16", seed=3),
    # tensor-core stress: 32 requests, L=20000, 64 targets each
    "c5": dict(name="stress-R32-L20000-T64-d256-h16-M6-r2-bf16", R=32,
               lengths=("fixed", 20000), targets=("fixed", 64), d=256, h=16, M=6, r=2,
               dtype="bf16", seed=4),
}

WEIGHT_KEYS = ("Wu", "Wg", "Wd", "ln_g", "ln_b", "Wq", "Wk", "Wv", "Wo", "Wc")
QUERY_KEYS = ("qWu", "qWg", "qWd", "q_ln_g", "q_ln_b")


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round-to-nearest-even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the fp32 values they denote (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 value, returned as fp32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(a))


@dataclasses.dataclass
class Workload:
    """One jagged STCA batch: histories, targets and all M layers' weights.

    X[offsets[r]:offsets[r+1]] is request r's history (L_r x d);
    targets[target_offsets[r]:target_offsets[r+1]] are its T_r target
    embeddings.  All arrays are fp32 holding values exactly representable in
    `dtype` ("f32" or "bf16").
    """
    name: str
    d: int
    h: int
    M: int
    r: int
    dtype: str
    seed: int
    lengths: np.ndarray
    target_counts: np.ndarray
    offsets: np.ndarray
    target_offsets: np.ndarray
    X: np.ndarray
    targets: np.ndarray
    weights: dict

    @property
    def R(self) -> int:
        return int(self.lengths.shape[0])

    @property
    def N(self) -> int:
        return int(self.offsets[-1])

    @property
    def T(self) -> int:
        return int(self.target_offsets[-1])

    def storage(self, a: np.ndarray) -> np.ndarray:
        """An array in the element type the GPU path reads (bf16 bits or fp32)."""
        if self.dtype == "bf16":
            return f32_to_bf16_bits(a)
        return np.ascontiguousarray(a, dtype=np.float32)

    def request(self, r: int):
        """(X_r, targets_r) views of request r."""
        lo, hi = int(self.offsets[r]), int(self.offsets[r + 1])
        tlo, thi = int(self.target_offsets[r]), int(self.target_offsets[r + 1])
        return self.X[lo:hi], self.targets[tlo:thi]


def _draw_lengths(spec, R, rng):
    kind = spec[0]
    if kind == "fixed":
        return np.full(R, int(spec[1]), dtype=np.int64)
    if kind == "uniform":
        return rng.integers(int(spec[1]), int(spec[2]) + 1, size=R).astype(np.int64)
    if kind == "lognormal":
        mean, sigma, lo, hi = float(spec[1]), float(spec[2]), int(spec[3]), int(spec[4])
        mu = math.log(mean) - sigma * sigma / 2.0      # pre-clip mean equals `mean`
        raw = rng.lognormal(mu, sigma, size=R)
        return np.clip(np.rint(raw), lo, hi).astype(np.int64)
    if kind == "list":
        return np.asarray(spec[1], dtype=np.int64)
    raise ValueError(f"unknown length spec {spec!r}")


def _draw_targets(spec, R, rng):
    kind = spec[0]
    if kind == "fixed":
        return np.full(R, int(spec[1]), dtype=np.int64)
    if kind == "1+poisson":
        return (1 + rng.poisson(float(spec[1]), size=R)).astype(np.int64)
    if kind == "list":
        return np.asarray(spec[1], dtype=np.int64)
    raise ValueError(f"unknown target spec {spec!r}")


def _xavier(rng, rows, cols):
    a = math.sqrt(6.0 / (rows + cols))
    return rng.uniform(-a, a, size=(rows, cols)).astype(np.float32)


def _offsets(counts):
    off = np.zeros(counts.shape[0] + 1, dtype=np.int64)
    np.cumsum(counts, out=off[1:])
    return off


def make_workload(*, lengths, targets, d, h, M, r, dtype="bf16", seed=0,
                  name="custom", random_ln=False, distinct_query_ffn=False,
                  R: Optional[int] = None) -> Workload:
    """Draw one workload.  `lengths`/`targets` are specs (see CONFIGS) or lists."""
    if isinstance(lengths, (list, tuple, np.ndarray)) and (len(lengths) == 0 or
                                                           not isinstance(lengths[0], str)):
        lengths = ("list", list(lengths))
    if isinstance(targets, (list, tuple, np.ndarray)) and (len(targets) == 0 or
                                                           not isinstance(targets[0], str)):
        targets = ("list", list(targets))
    if R is None:
        R = len(lengths[1]) if lengths[0] == "list" else len(targets[1])
    assert dtype in ("f32", "bf16")
    rng = np.random.default_rng(seed)
    L = _draw_lengths(lengths, R, rng)
    Tr = _draw_targets(targets, R, rng)
    assert L.shape == (R,) and Tr.shape == (R,)
    N, T = int(L.sum()), int(Tr.sum())
    X = rng.standard_normal((N, d), dtype=np.float32)
    xt = rng.standard_normal((T, d), dtype=np.float32)
    rd = r * d
    W = {k: [] for k in WEIGHT_KEYS}
    for i in range(M):
        W["Wu"].append(_xavier(rng, d, rd))
        W["Wg"].append(_xavier(rng, d, rd))
        W["Wd"].append(_xavier(rng, rd, d))
        W["Wq"].append(_xavier(rng, d, d))
        W["Wk"].append(_xavier(rng, d, d))
        W["Wv"].append(_xavier(rng, d, d))
        W["Wo"].append(_xavier(rng, d, d))
        W["Wc"].append(None if i == 0 else _xavier(rng, (i + 1) * d, d))
    for i in range(M):
        if random_ln:
            W["ln_g"].append(rng.uniform(0.5, 1.5, size=d).astype(np.float32))
            W["ln_b"].append(rng.uniform(-0.5, 0.5, size=d).astype(np.float32))
        else:
            W["ln_g"].append(np.ones(d, dtype=np.float32))
            W["ln_b"].append(np.zeros(d, dtype=np.float32))
    for k in QUERY_KEYS:
        W[k] = None
    if distinct_query_ffn:
        W["qWu"] = [_xavier(rng, d, rd) for _ in range(M)]
        W["qWg"] = [_xavier(rng, d, rd) for _ in range(M)]
        W["qWd"] = [_xavier(rng, rd, d) for _ in range(M)]
        W["q_ln_g"] = rng.uniform(0.5, 1.5, size=d).astype(np.float32)
        W["q_ln_b"] = rng.uniform(-0.5, 0.5, size=d).astype(np.float32)
    # prediction-head weights of Eq. (9), from a stream of their own so that
    # the draws above do not depend on them
    hrng = np.random.default_rng([seed, 9])
    W["Wz"] = _xavier(hrng, (M + 1) * d, d)
    W["zWu"] = _xavier(hrng, d, rd)
    W["zWg"] = _xavier(hrng, d, rd)
    W["zWd"] = _xavier(hrng, rd, d)
    if dtype == "bf16":
        X = round_to_bf16(X)
        xt = round_to_bf16(xt)
        for k, v in W.items():
            if v is None:
                continue
            if isinstance(v, list):
                W[k] = [None if a is None else round_to_bf16(a) for a in v]
            else:
                W[k] = round_to_bf16(v)
    return Workload(name=name, d=d, h=h, M=M, r=r, dtype=dtype, seed=seed, lengths=L,
                    target_counts=Tr, offsets=_offsets(L), target_offsets=_offsets(Tr),
                    X=X, targets=xt, weights=W)


# A sparse-training batch ("Make It Long, Keep It Fast" digest §2.3; STCA blog
# §2.6, §3.3): full histories cut to L_infer = 10k at inference, trained at an
# average length of 2k (SS = 20%) with L_max = L_infer, the U-shaped Beta
# curriculum of alpha = 0.02, 8 targets per user (request-level batching,
# m = 8), and the recommended 4-layer, d = 256, h = 8, r = 4 encoder.  The
# full-history lengths and L_min are not given on the pages: lognormal with
# mean 6000 clipped to [100, 20000], and L_min = 64.
TRAIN_BATCH = dict(name="sparse-train-B256-Lavg2000-Lmax10000-a0.02-T8-d256-h8-M4-r4-bf16",
                   B=256, hist=("lognormal", 6000.0, 0.8, 100, 20000), L_min=64,
                   L_max=10000, L_avg=2000, L_infer=10000, alpha=0.02, targets=8,
                   d=256, h=8, M=4, r=4, dtype="bf16", seed=5)


@dataclasses.dataclass
class TrainingHistories:
    """Full user histories of one training batch and the per-user Beta draws."""
    hist_lengths: np.ndarray   # B int64
    hist_offsets: np.ndarray   # B+1 int64
    s: np.ndarray              # B float64, s_b ~ Beta(alpha, beta)
    X: np.ndarray              # N x d float32 values (bf16-valued for bf16)
    dtype: str

    def storage(self, a):
        return f32_to_bf16_bits(a) if self.dtype == "bf16" else np.ascontiguousarray(a, np.float32)


def make_training_histories(*, B, hist, d, alpha, beta, dtype="bf16", seed=0, with_x=True):
    """Draw, in this order, the B full-history lengths (a length spec as in
    CONFIGS, or a list), the B Beta(alpha, beta) draws and the N x d history
    rows (iid N(0, 1)).  beta is the caller's: this module does not derive it."""
    rng = np.random.default_rng(seed)
    if isinstance(hist, (list, tuple, np.ndarray)) and (len(hist) == 0 or not isinstance(hist[0], str)):
        hist = ("list", list(hist))
    H = _draw_lengths(hist, B, rng)
    s = rng.beta(alpha, beta, size=B).astype(np.float64)
    N = int(H.sum())
    X = rng.standard_normal((N, d), dtype=np.float32) if with_x else np.zeros((0, d), np.float32)
    if dtype == "bf16":
        X = round_to_bf16(X)
    return TrainingHistories(hist_lengths=H, hist_offsets=_offsets(H), s=s, X=X, dtype=dtype)


def config_shapes(key: str, seed=None):
    """History lengths and target counts of configuration `key` without drawing
    the embeddings: the same first two draws as make_config_workload."""
    cfg = CONFIGS[key]
    rng = np.random.default_rng(cfg["seed"] if seed is None else seed)
    L = _draw_lengths(cfg["lengths"], cfg["R"], rng)
    Tr = _draw_targets(cfg["targets"], cfg["R"], rng)
    return L, Tr, _offsets(L), _offsets(Tr)


def make_config_workload(key: str, **overrides) -> Workload:
    """The named configuration `key` ("c1".."c5"), optionally with overrides."""
    cfg = dict(CONFIGS[key])
    cfg.update(overrides)
    return make_workload(lengths=cfg["lengths"], targets=cfg["targets"], d=cfg["d"],
                         h=cfg["h"], M=cfg["M"], r=cfg["r"], dtype=cfg["dtype"],
                         seed=cfg["seed"], name=cfg["name"], R=cfg["R"],
                         random_ln=cfg.get("random_ln", False),
                         distinct_query_ffn=cfg.get("distinct_query_ffn", False))
