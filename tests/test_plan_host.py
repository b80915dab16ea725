"""The attention work planner (host only, through the C ABI): every unit of
work is covered exactly once, partial rows are contiguous, and the tensor-core
split gives every CTA the same number of key tiles (stream-K)."""
import numpy as np
import pytest

import target_attention_jagged_b200 as S
from gen import CONFIGS, config_shapes, make_workload


def check(off, toff, h, path, num_ctas=148, split=0):
    plan = S.stca_plan_attention(off, toff, h, path, num_ctas, split)
    it = plan["items"]
    R = len(off) - 1
    # partial rows are laid out contiguously, in item order
    rows = it[:, 5]
    assert np.array_equal(it[:, 6], np.concatenate([[0], np.cumsum(rows)[:-1]]) if len(it) else it[:, 6])
    assert plan["partial_rows"] == rows.sum()
    # every (request, query tile, key) unit exactly once
    for r in range(R):
        Tr = toff[r + 1] - toff[r]
        mine = it[it[:, 0] == r]
        if Tr == 0:
            assert path == 1 or len(mine) == 0
            continue
        ntile = (Tr * h + 127) // 128 if path == 2 else 1
        assert sorted(set(mine[:, 1].tolist())) == list(range(ntile))
        for mt in range(ntile):
            sub = mine[mine[:, 1] == mt]
            keys = np.concatenate([np.arange(k0, k0 + n) for k0, n in zip(sub[:, 2], sub[:, 3])])
            assert np.array_equal(np.sort(keys), np.arange(off[r], off[r + 1]))
            want_rows = min(128, Tr * h - mt * 128) if path == 2 else Tr * h
            assert np.all(sub[:, 5] == want_rows)
            q0 = toff[r] * h + (mt * 128 if path == 2 else 0)
            assert np.all(sub[:, 4] == q0)
    if path == 2:
        cta = plan["cta_begin"]
        # without a split cap the runs fill at most num_ctas CTAs; a cap may need more
        assert (split > 0 or plan["grid"] <= num_ctas) and cta[0] == 0 and cta[-1] == len(it)
        assert np.all(np.diff(cta) >= 0)
        tiles = [int(((it[cta[c]:cta[c + 1], 3] + 127) // 128).sum()) for c in range(plan["grid"])]
        cap = max(tiles)
        if split > 0:
            assert cap <= max(1, split // 128)
        assert all(t <= cap for t in tiles) and all(t == cap for t in tiles[:-1])
    return plan


@pytest.mark.parametrize("key", sorted(CONFIGS))
@pytest.mark.parametrize("path", [1, 2])
def test_named_configs(key, path):
    L, Tr, off, toff = config_shapes(key)
    h = CONFIGS[key]["h"]
    plan = check(off, toff, h, path)
    if path == 2 and key == "c3":
        # 64 requests x 79 key tiles over 148 CTAs: at most 2 items per CTA
        assert plan["grid"] == 148 or plan["grid"] <= 148
        assert np.max(np.diff(plan["cta_begin"])) <= 2


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("path", [1, 2])
def test_random_ragged(seed, path):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 40))
    L = rng.integers(1, 3000, size=R)
    Tr = rng.integers(0, 30, size=R)
    Tr[rng.integers(0, R)] = max(1, Tr[0])
    off = np.concatenate([[0], np.cumsum(L)])
    toff = np.concatenate([[0], np.cumsum(Tr)])
    h = int(rng.choice([1, 2, 4, 8, 16]))
    for ctas in (1, 7, 148):
        for split in (0, 128, 1024):
            check(off, toff, h, path, ctas, split)


def test_rejects_bad_offsets():
    with pytest.raises(S.StcaError):
        S.stca_plan_attention([0, 5, 5], [0, 1, 2], 4, 2)    # empty history
    with pytest.raises(S.StcaError):
        S.stca_plan_attention([0, 5], [0, 1], 4, 3)          # bad path
