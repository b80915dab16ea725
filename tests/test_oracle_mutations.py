"""Plant plausible mistakes in the oracle (on the CPU) and check the pins catch them.

Each mutant replaces one oracle function for the duration of a test.  The
compact pin set below (brute force, the PyTorch cross-check, closed forms)
must reject every mutant; otherwise a mistake of that kind could hide.
"""
import math

import numpy as np
import pytest

from gen import make_workload
from oracle import stca_oracle as O
from tests import bruteforce, torch_reference


def _rel(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def _cases():
    return [
        make_workload(lengths=[3], targets=[2], d=4, h=2, M=3, r=2, dtype="f32", seed=1,
                      random_ln=True),
        make_workload(lengths=[4], targets=[1], d=4, h=1, M=2, r=1, dtype="f32", seed=2),
        make_workload(lengths=[1], targets=[2], d=4, h=2, M=2, r=1, dtype="f32", seed=3,
                      distinct_query_ffn=True, random_ln=True),
    ]


def pins_reject():
    """True when at least one pin fails against the current oracle."""
    for wl in _cases():
        got = O.forward_request(wl.X, wl.targets, wl.weights, wl.h)
        bf = np.asarray(bruteforce.forward_request(wl.X, wl.targets, wl.weights, wl.h))
        if got.shape != bf.shape or _rel(got, bf) > 1e-10:
            return True
    wl = make_workload(lengths=[40], targets=[3], d=16, h=4, M=3, r=2, dtype="f32", seed=4,
                       random_ln=True, distinct_query_ffn=True)
    got = O.forward_request(wl.X, wl.targets, wl.weights, 4)
    if _rel(got, torch_reference.forward_request(wl.X, wl.targets, wl.weights, 4)) > 1e-10:
        return True
    return False


def _reordered_with(q, Xt, Wq, Wk, Wv, Wo, h, scale=None, transpose_k=False, cols=None):
    q, Xt = np.asarray(q, float), np.asarray(Xt, float)
    d = q.shape[-1]
    dh = d // h
    scale = 1 / math.sqrt(dh) if scale is None else scale
    heads = []
    for j in range(h):
        c = cols(j) if cols else slice(j * dh, (j + 1) * dh)
        Wk_ = np.asarray(Wk, float).T if transpose_k else np.asarray(Wk, float)
        u = (q @ np.asarray(Wq, float)[:, c]) @ Wk_[:, c].T
        a = O.softmax(u @ Xt.T * scale)
        heads.append((a @ Xt) @ np.asarray(Wv, float)[:, c])
    return np.concatenate(heads, -1) @ np.asarray(Wo, float)


def _f(a):
    return np.asarray(a, dtype=np.float64)


def _ln_no_centering(y, g, b, eps=1e-5):
    y = _f(y)
    return y / np.sqrt((y ** 2).mean(-1, keepdims=True) + eps) * g + b


def _ln_unbiased(y, g, b, eps=1e-5):
    y = _f(y)
    return (y - y.mean(-1, keepdims=True)) / np.sqrt(y.var(-1, ddof=1, keepdims=True) + eps) * g + b


def _ln_no_affine(y, g, b, eps=1e-5):
    y = _f(y)
    return (y - y.mean(-1, keepdims=True)) / np.sqrt(y.var(-1, keepdims=True) + eps)


def _fusion_xt_first(outs, xt, W, i):
    cat = np.concatenate([_f(xt)] + [_f(o) for o in outs], -1)
    return O.swiglu_ffn(cat @ _f(W["Wc"][i]), *O._query_ffn(W, i))


def _fusion_history_ffn(outs, xt, W, i):
    cat = np.concatenate([_f(o) for o in outs] + [_f(xt)], -1)
    return O.swiglu_ffn(cat @ _f(W["Wc"][i]), W["Wu"][i], W["Wg"][i], W["Wd"][i])


def _fusion_last_only(outs, xt, W, i):
    # only o^(i) and x_t, zero-padded to the expected width (drops the dense links)
    d = _f(xt).shape[-1]
    cat = np.concatenate([np.zeros_like(_f(o)) for o in outs[:-1]] + [_f(outs[-1]), _f(xt)], -1)
    assert cat.shape[-1] == (len(outs) + 1) * d
    return O.swiglu_ffn(cat @ _f(W["Wc"][i]), *O._query_ffn(W, i))


def _query_init_no_ln(xt, W):
    return O.swiglu_ffn(xt, *O._query_ffn(W, 0))


def _softmax_wrong_axis(s):
    e = np.exp(_f(s))
    return e / e.sum(axis=0, keepdims=True)


def _attn_scale_sqrt_d(q, Xt, Wq, Wk, Wv, Wo, h, **_):
    return _reordered_with(q, Xt, Wq, Wk, Wv, Wo, h, scale=1 / math.sqrt(_f(q).shape[-1]))


def _attn_wk_transposed(q, Xt, Wq, Wk, Wv, Wo, h, **_):
    return _reordered_with(q, Xt, Wq, Wk, Wv, Wo, h, transpose_k=True)


def _attn_strided_heads(q, Xt, Wq, Wk, Wv, Wo, h, **_):
    return _reordered_with(q, Xt, Wq, Wk, Wv, Wo, h, cols=lambda j: slice(j, None, h))


def _attn_no_wo(q, Xt, Wq, Wk, Wv, Wo, h, **_):
    return _reordered_with(q, Xt, Wq, Wk, Wv, np.eye(_f(Wo).shape[0]), h)


MUTANTS = {
    "scale 1/sqrt(d) instead of 1/sqrt(d_h)": ("attention_reordered", _attn_scale_sqrt_d),
    "W_K transposed": ("attention_reordered", _attn_wk_transposed),
    "heads take strided columns": ("attention_reordered", _attn_strided_heads),
    "W_O dropped": ("attention_reordered", _attn_no_wo),
    "gate is sigmoid, not SiLU": ("silu", lambda z: O.sigmoid(z)),
    "gate sign flipped": ("silu", lambda z: _f(z) * O.sigmoid(-_f(z))),
    "LayerNorm without mean subtraction": ("layer_norm", _ln_no_centering),
    "LayerNorm unbiased variance": ("layer_norm", _ln_unbiased),
    "LayerNorm affine dropped": ("layer_norm", _ln_no_affine),
    "x_t first in the fusion concat": ("query_fusion", _fusion_xt_first),
    "fusion ignores the query-side FFN weights": ("query_fusion", _fusion_history_ffn),
    "fusion keeps only the last layer's output": ("query_fusion", _fusion_last_only),
    "query init without LayerNorm": ("query_init", _query_init_no_ln),
    "encodings chained across layers": ("encode_history", None),  # built in the test
    "softmax over the wrong axis": ("softmax", _softmax_wrong_axis),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, monkeypatch):
    assert not pins_reject(), "pins must accept the unmodified oracle"
    attr, fn = MUTANTS[name]
    if name == "encodings chained across layers":
        orig = O.encode_history

        def chained(X, W, i):
            base = X if i == 0 else chained(X, W, i - 1)
            return orig(base, W, i)
        fn = chained
    monkeypatch.setattr(O, attr, fn)
    assert pins_reject(), f"mutant not caught: {name}"



# ------------------------------------------------------------ prediction head, Eq. (9)

def head_pins_reject():
    """True when a head pin fails: brute force on tiny cases, the PyTorch cross-check."""
    for seed, M in ((31, 1), (32, 3)):
        wl = make_workload(lengths=[3], targets=[2], d=4, h=2, M=M, r=2, dtype="f32", seed=seed)
        Z = O.forward_request(wl.X, wl.targets, wl.weights, wl.h)
        z = O.head_from_outputs(Z, wl.targets, wl.weights)
        bf = np.array([bruteforce.prediction_head([Z[t, i] for i in range(M)], wl.targets[t],
                                                  wl.weights) for t in range(2)])
        if z.shape != bf.shape or _rel(z, bf) > 1e-10:
            return True
    wl = make_workload(lengths=[20], targets=[3], d=8, h=2, M=2, r=2, dtype="f32", seed=33)
    Z = O.forward_request(wl.X, wl.targets, wl.weights, wl.h)
    if _rel(O.head_from_outputs(Z, wl.targets, wl.weights),
            torch_reference.prediction_head(Z, wl.targets, wl.weights)) > 1e-10:
        return True
    return False


def _head_xt_first(outs, xt, W):
    cat = np.concatenate([_f(xt)] + [_f(o) for o in outs], axis=-1)
    return O.swiglu_ffn(cat @ _f(W["Wz"]), _f(W["zWu"]), _f(W["zWg"]), _f(W["zWd"]))


def _head_last_only(outs, xt, W):
    d = _f(xt).shape[-1]
    cat = np.concatenate([_f(outs[-1]), _f(xt)], axis=-1)
    return O.swiglu_ffn(cat @ _f(W["Wz"])[-2 * d:], _f(W["zWu"]), _f(W["zWg"]), _f(W["zWd"]))


def _head_query_ffn(outs, xt, W):
    cat = np.concatenate([_f(o) for o in outs] + [_f(xt)], axis=-1)
    return O.swiglu_ffn(cat @ _f(W["Wz"]), _f(W["Wu"][-1]), _f(W["Wg"][-1]), _f(W["Wd"][-1]))


def _head_with_ln(outs, xt, W):
    cat = np.concatenate([_f(o) for o in outs] + [_f(xt)], axis=-1)
    y = O.swiglu_ffn(cat @ _f(W["Wz"]), _f(W["zWu"]), _f(W["zWg"]), _f(W["zWd"]))
    d = y.shape[-1]
    return O.layer_norm(y, np.ones(d), np.zeros(d))


HEAD_MUTANTS = {
    "x_t first in the head concat": _head_xt_first,
    "head keeps only the last layer's output": _head_last_only,
    "head reuses the history FFN weights": _head_query_ffn,
    "head adds a LayerNorm": _head_with_ln,
}


@pytest.mark.parametrize("name", sorted(HEAD_MUTANTS))
def test_head_pins_reject_mutant(name, monkeypatch):
    assert not head_pins_reject(), "head pins must accept the unmodified oracle"
    monkeypatch.setattr(O, "prediction_head", HEAD_MUTANTS[name])
    assert head_pins_reject(), f"mutant not caught: {name}"
