"""ctypes binding of libstca.so (include/stca.h): argument marshalling only.

Every step of the STCA forward runs in the library's CUDA kernels; this module
only turns tensors and arrays into pointers and sizes, and error codes into
exceptions.  There is no fallback: if libstca.so is missing, importing this
module raises.

Functions carry the C names.  Device buffers are torch CUDA tensors; offsets
are host int64 arrays; weights may be host numpy arrays or torch tensors
(bf16 handles take torch.bfloat16 tensors or numpy uint16 bf16 bit patterns,
fp32 handles take float32).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstca.so")

STCA_F32, STCA_BF16 = 0, 1
STCA_OK, STCA_EINVAL, STCA_ESTATE, STCA_ENOMEM, STCA_ECUDA, STCA_EDEVICE = 0, -1, -2, -3, -4, -5
STCA_OPT_ATTN_PATH, STCA_OPT_ENCODE_PATH, STCA_OPT_SPLIT_KEYS, STCA_OPT_TIMING = 1, 2, 3, 4
STCA_OPT_STEP_PATH = 5
STCA_OPT_ATTN_FORM = 6
STCA_OPT_ATTN_KERNEL = 7
STCA_OPT_TEST_STOP_TILES = 8
STCA_OPT_BW_GEMM = 9
STCA_OPT_PIPELINE = 10
STCA_OPT_LAUNCHES = 100
STCA_OPT_LAST_FORM = 101
STCA_K_ENCODE, STCA_K_ATTN, STCA_K_STEP, STCA_K_HEAD, STCA_K_PIPE, STCA_K_CLASSES = 0, 1, 2, 3, 4, 5
_NAMES = {STCA_EINVAL: "EINVAL", STCA_ESTATE: "ESTATE", STCA_ENOMEM: "ENOMEM",
          STCA_ECUDA: "ECUDA", STCA_EDEVICE: "EDEVICE"}

EXPORTS = ("stca_init", "stca_destroy", "stca_encode", "stca_forward", "stca_encode_forward", "stca_run_host",
           "stca_validate_offsets", "stca_device_status", "stca_set_option",
           "stca_get_option", "stca_kernel_times", "stca_get_encoded", "stca_plan_attention",
           "stca_forward_static", "stca_head", "stca_forward_head", "stca_sl_beta", "stca_sl_plan",
           "stca_sl_gather", "stca_encode_backward", "stca_attention_backward",
           "stca_output_backward", "stca_query_backward", "stca_query_init_backward",
           "stca_fusion_backward", "stca_selftest_ex2", "stca_last_error")


class StcaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"STCA_{_NAMES.get(code, code)}: {msg}")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python target_attention_jagged_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    PI64 = ctypes.POINTER(ctypes.c_int64)
    lib.stca_init.argtypes = [P, I, I, I, I, I, I, ctypes.POINTER(P)]
    lib.stca_destroy.argtypes = [P]
    lib.stca_destroy.restype = None
    lib.stca_encode.argtypes = [P, P, PI64, I64, I64, P]
    lib.stca_forward.argtypes = [P, P, PI64, I64, P, P]
    lib.stca_encode_forward.argtypes = [P, P, PI64, I64, I64, P, PI64, I64, P, P]
    lib.stca_forward_static.argtypes = [P, P, PI64, I64, P, P]
    lib.stca_head.argtypes = [P, P, I64, P, P, P]
    lib.stca_forward_head.argtypes = [P, P, PI64, I64, P, P, P]
    D, PD = ctypes.c_double, ctypes.POINTER(ctypes.c_double)
    lib.stca_sl_beta.argtypes = [D, I64, I64, I64, PD, PD]
    lib.stca_sl_plan.argtypes = [PI64, I64, PD, I64, I64, I64, I64, PI64, PI64, PI64, PI64]
    lib.stca_sl_gather.argtypes = [P, I64, I64, P, P, I64, I64, P, P, P]
    lib.stca_encode_backward.argtypes = [P, I, P, I64, P, P, P, P, P, P, P, P]
    lib.stca_attention_backward.argtypes = [P, I, P, PI64, I64, P, P, P, P]
    lib.stca_output_backward.argtypes = [P, I, P, I64, P, P, P, P, P]
    lib.stca_query_backward.argtypes = [P, I, P, I64, P, P, P, P, P]
    lib.stca_query_init_backward.argtypes = [P, P, I64, P, P, P, P, P, P, P, P]
    lib.stca_fusion_backward.argtypes = [P, I, P, P, I64, P, I, P, P, P, P, P, P, P]
    lib.stca_run_host.argtypes = [P, P, PI64, I64, I64, P, PI64, I64, P, P]
    lib.stca_validate_offsets.argtypes = [PI64, I64, I64, I]
    lib.stca_device_status.argtypes = [P, P]
    lib.stca_selftest_ex2.argtypes = [P, P, I64, I, P]
    lib.stca_set_option.argtypes = [P, I, I64]
    lib.stca_get_option.argtypes = [P, I, PI64]
    lib.stca_get_encoded.argtypes = [P, I, P, P]
    lib.stca_plan_attention.argtypes = [PI64, PI64, I64, I, I, I, I64, PI64, PI64, PI64, PI64,
                                        I64, ctypes.POINTER(ctypes.c_int32), I64]
    lib.stca_kernel_times.argtypes = [P, ctypes.POINTER(ctypes.c_double), PI64, I]
    lib.stca_last_error.restype = ctypes.c_char_p
    lib.stca_last_error.argtypes = []
    for name in EXPORTS:
        if name not in ("stca_destroy", "stca_last_error"):
            getattr(lib, name).restype = ctypes.c_int
    return lib


_lib = _load()


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.POINTER(ctypes.c_void_p)) for n in (
        "Wu", "Wg", "Wd", "ln_gamma", "ln_beta", "Wq", "Wk", "Wv", "Wo", "Wc",
        "qWu", "qWg", "qWd")] + [(n, ctypes.c_void_p) for n in (
        "q_ln_gamma", "q_ln_beta", "Wz", "zWu", "zWg", "zWd")]


def stca_last_error() -> str:
    return _lib.stca_last_error().decode()


def _check(rc: int):
    if rc != STCA_OK:
        raise StcaError(rc, stca_last_error())


def _offsets(a) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int64))
    return a


def _i64p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    return getattr(stream, "cuda_stream", stream)


def _host_buffer(a, dtype_code: int, keep: list) -> int:
    """Pointer to a host copy of weight `a` in the handle's element type."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu()
            if dtype_code == STCA_BF16:
                if a.dtype != torch.bfloat16:
                    raise TypeError("bf16 handle: weights must be torch.bfloat16")
                a = a.contiguous().view(torch.int16).numpy().view(np.uint16)
            else:
                if a.dtype != torch.float32:
                    raise TypeError("fp32 handle: weights must be torch.float32")
                a = a.contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    want = np.uint16 if dtype_code == STCA_BF16 else np.float32
    if a.dtype != want:
        raise TypeError(f"weights must be {np.dtype(want).name} for this handle, got {a.dtype}")
    keep.append(a)
    return a.ctypes.data


def stca_init(weights: dict, d: int, h: int, r: int, M: int, dtype: int) -> int:
    """Create a handle from host weights (dict of per-layer lists, the keys of
    stca_weights).  Returns the opaque handle (an int)."""
    keep: list = []

    def arr(key, optional=False, skip0=False):
        v = weights.get(key)
        if v is None:
            if optional:
                return None
            raise ValueError(f"weight {key} missing")
        if len(v) != M:
            raise ValueError(f"weight {key} needs {M} entries")
        ptrs = (ctypes.c_void_p * M)()
        for i, a in enumerate(v):
            if a is None:
                if skip0 and i == 0:
                    ptrs[i] = None
                    continue
                raise ValueError(f"weight {key}[{i}] is None")
            ptrs[i] = _host_buffer(a, dtype, keep)
        keep.append(ptrs)
        return ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p))

    w = _Weights()
    for k in ("Wu", "Wg", "Wd", "Wq", "Wk", "Wv", "Wo"):
        setattr(w, k, arr(k))
    w.ln_gamma = arr("ln_g", optional=True)
    w.ln_beta = arr("ln_b", optional=True)
    w.Wc = arr("Wc", optional=(M == 1), skip0=True)
    w.qWu = arr("qWu", optional=True)
    w.qWg = arr("qWg", optional=True)
    w.qWd = arr("qWd", optional=True)
    w.q_ln_gamma = _host_buffer(weights["q_ln_g"], dtype, keep) if weights.get("q_ln_g") is not None else None
    w.q_ln_beta = _host_buffer(weights["q_ln_b"], dtype, keep) if weights.get("q_ln_b") is not None else None
    for k in ("Wz", "zWu", "zWg", "zWd"):     # optional prediction head (Eq. (9))
        if weights.get(k) is not None:
            setattr(w, k, _host_buffer(weights[k], dtype, keep))
    out = ctypes.c_void_p()
    _check(_lib.stca_init(ctypes.byref(w), d, h, r, M, dtype, 0, ctypes.byref(out)))
    return out.value


def stca_destroy(handle: int) -> None:
    _lib.stca_destroy(handle)


def stca_encode(handle: int, X, offsets, stream=None) -> None:
    """X: CUDA tensor (N x d) in the handle's dtype; offsets: host int64 (R+1)."""
    off = _offsets(offsets)
    R = off.shape[0] - 1
    N = int(off[-1]) if R >= 0 else 0
    _check(_lib.stca_encode(handle, X.data_ptr(), _i64p(off), R, N, _stream_ptr(stream)))


def stca_forward(handle: int, targets, target_offsets, Z=None, stream=None):
    """targets: CUDA tensor (T x d); returns Z (T x M x d fp32 CUDA tensor)."""
    import torch
    toff = _offsets(target_offsets)
    T = int(toff[-1])
    if Z is None:
        raise ValueError("pass Z: a CUDA float32 tensor of shape (T, M, d)")
    assert Z.dtype == torch.float32 and Z.is_cuda and Z.is_contiguous()
    _check(_lib.stca_forward(handle, targets.data_ptr() if T > 0 else None, _i64p(toff), T,
                             Z.data_ptr() if T > 0 else None, _stream_ptr(stream)))
    return Z


def stca_encode_forward(handle: int, X, offsets, targets, target_offsets, Z, stream=None):
    """stca_encode then stca_forward in one call (see include/stca.h): X (N x d)
    and targets (T x d) CUDA tensors in the handle's dtype, host int64 offsets;
    fills and returns Z (T x M x d fp32 CUDA tensor)."""
    import torch
    off, toff = _offsets(offsets), _offsets(target_offsets)
    R = off.shape[0] - 1
    N = int(off[-1]) if R >= 0 else 0
    T = int(toff[-1])
    assert Z.dtype == torch.float32 and Z.is_cuda and Z.is_contiguous()
    _check(_lib.stca_encode_forward(handle, X.data_ptr(), _i64p(off), R, N,
                                    targets.data_ptr() if T > 0 else None, _i64p(toff), T,
                                    Z.data_ptr() if T > 0 else None, _stream_ptr(stream)))
    return Z


def stca_forward_static(handle: int, targets, target_offsets, Z, stream=None):
    """stca_forward with its workspace in the library's static device array
    (no device allocation); Z: CUDA float32 (T, M, d)."""
    import torch
    toff = _offsets(target_offsets)
    T = int(toff[-1])
    assert Z.dtype == torch.float32 and Z.is_cuda and Z.is_contiguous()
    _check(_lib.stca_forward_static(handle, targets.data_ptr() if T > 0 else None, _i64p(toff),
                                    T, Z.data_ptr() if T > 0 else None, _stream_ptr(stream)))
    return Z


def stca_head(handle: int, targets, Z, zout, stream=None):
    """Prediction-head token of Eq. (9): zout (T x d fp32 CUDA) from Z (T x M x d
    fp32 CUDA, the forward's output) and targets (T x d CUDA, handle dtype)."""
    import torch
    T = int(Z.shape[0])
    assert Z.dtype == torch.float32 and Z.is_cuda and Z.is_contiguous()
    assert zout.dtype == torch.float32 and zout.is_cuda and zout.is_contiguous()
    assert targets.is_contiguous() and int(targets.shape[0]) == T and int(zout.shape[0]) == T
    _check(_lib.stca_head(handle, targets.data_ptr() if T > 0 else None, T,
                          Z.data_ptr() if T > 0 else None, zout.data_ptr() if T > 0 else None,
                          _stream_ptr(stream)))
    return zout


def stca_sl_beta(alpha: float, L_min: int, L_max: int, L_avg: int):
    """Eq. (17) beta and Eq. (15) sequence sparsity: returns (beta, ss)."""
    beta, ss = ctypes.c_double(), ctypes.c_double()
    _check(_lib.stca_sl_beta(alpha, L_min, L_max, L_avg, ctypes.byref(beta), ctypes.byref(ss)))
    return beta.value, ss.value


def stca_sl_plan(hist_offsets, s, L_min: int, L_max: int, L_avg: int, L_infer: int) -> dict:
    """Host plan of a training batch: int64 arrays train, lengths, packed_offsets, src_start."""
    off = _offsets(hist_offsets)
    B = off.shape[0] - 1
    sd = np.ascontiguousarray(np.asarray(s, dtype=np.float64))
    if sd.shape != (B,):
        raise ValueError("one draw per user")
    out = {k: np.zeros(B + (k == "packed_offsets"), dtype=np.int64)
           for k in ("train", "lengths", "packed_offsets", "src_start")}
    _check(_lib.stca_sl_plan(_i64p(off), B, sd.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                             L_min, L_max, L_avg, L_infer, _i64p(out["train"]),
                             _i64p(out["lengths"]), _i64p(out["packed_offsets"]),
                             _i64p(out["src_start"])))
    return out


def stca_sl_gather(X, src_start, packed_offsets, X_packed, seg=None, stream=None):
    """Device gather of the packed stream.  X, X_packed: CUDA tensors (rows x d);
    src_start, packed_offsets: CUDA int64 tensors (B, B+1); seg: CUDA int32 (P) or None."""
    import torch
    assert X.is_cuda and X_packed.is_cuda and X.is_contiguous() and X_packed.is_contiguous()
    assert src_start.dtype == torch.int64 and packed_offsets.dtype == torch.int64
    B = int(src_start.shape[0])
    P = int(X_packed.shape[0])
    row_bytes = X.element_size() * (X.numel() // max(1, X.shape[0])) if X.shape[0] else \
        X_packed.element_size() * (X_packed.numel() // max(1, P))
    _check(_lib.stca_sl_gather(X.data_ptr(), int(X.shape[0]), row_bytes, src_start.data_ptr(),
                               packed_offsets.data_ptr(), B, P, X_packed.data_ptr(),
                               seg.data_ptr() if seg is not None else None, _stream_ptr(stream)))
    return X_packed


def build_training_batch(X, hist_offsets, s, L_min: int, L_max: int, L_avg: int, L_infer: int,
                         stream=None):
    """Plan (host) and gather (device) one sparse-training batch: returns
    (X_packed, seg, plan) with plan's packed_offsets the stca_encode offsets."""
    import torch
    plan = stca_sl_plan(hist_offsets, s, L_min, L_max, L_avg, L_infer)
    P = int(plan["packed_offsets"][-1])
    dev = X.device
    src = torch.from_numpy(plan["src_start"]).to(dev)
    poff = torch.from_numpy(plan["packed_offsets"]).to(dev)
    Xp = torch.empty((P,) + tuple(X.shape[1:]), dtype=X.dtype, device=dev)
    seg = torch.empty(P, dtype=torch.int32, device=dev)
    stca_sl_gather(X, src, poff, Xp, seg, stream)
    return Xp, seg, plan


def stca_encode_backward(handle: int, layer: int, X, dXt, d: int, rd: int, with_dx=True, stream=None):
    """Gradients of the layer's history encoding (Eqs. (1)-(2)) from dXt (N x d
    fp32 CUDA); X: the CUDA rows (N x d, handle dtype).  Returns a dict of fp32
    CUDA tensors dX (or None), dWu, dWg, dWd, dgamma, dbeta."""
    import torch
    N = int(X.shape[0])
    dev = X.device
    f = lambda *sh: torch.empty(sh, dtype=torch.float32, device=dev)  # noqa: E731
    out = {"dX": f(N, d) if with_dx else None, "dWu": f(d, rd), "dWg": f(d, rd), "dWd": f(rd, d),
           "dgamma": f(d), "dbeta": f(d)}
    assert dXt.dtype == torch.float32 and dXt.is_contiguous() and X.is_contiguous()
    ptr = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
    _check(_lib.stca_encode_backward(handle, layer, X.data_ptr(), N, dXt.data_ptr(), ptr(out["dX"]),
                                     ptr(out["dWu"]), ptr(out["dWg"]), ptr(out["dWd"]),
                                     ptr(out["dgamma"]), ptr(out["dbeta"]), _stream_ptr(stream)))
    return out


def stca_attention_backward(handle: int, layer: int, U, target_offsets, dC, N: int, stream=None):
    """Gradients of the merged attention rows (Eq. (13)) of the last encode's
    layer: dU (T h x d) and dXt (N x d), fp32 CUDA tensors."""
    import torch
    toff = _offsets(target_offsets)
    T = int(toff[-1])
    assert U.dtype == torch.float32 and dC.dtype == torch.float32
    dU = torch.empty_like(U)
    dX = torch.empty((N, U.shape[1]), dtype=torch.float32, device=U.device)
    _check(_lib.stca_attention_backward(handle, layer, U.data_ptr() if T > 0 else None, _i64p(toff), T,
                                        dC.data_ptr() if T > 0 else None,
                                        dU.data_ptr() if T > 0 else None, dX.data_ptr(),
                                        _stream_ptr(stream)))
    return dU, dX


def _f32_out(*shape, device):
    import torch
    return torch.empty(shape, dtype=torch.float32, device=device)


def stca_output_backward(handle: int, layer: int, C, dZ, h: int, stream=None):
    """Gradients of o = [c_j W_V^j]_j W_O (Eqs. (6), (13)): C (T, h, d) or (T h, d)
    and dZ (T, d), fp32 contiguous CUDA.  Returns dC (T h, d), dWv, dWo (d, d)."""
    import torch
    T, d = int(dZ.shape[0]), int(dZ.shape[1])
    assert C.dtype == torch.float32 and dZ.dtype == torch.float32
    assert C.is_contiguous() and dZ.is_contiguous() and C.numel() == T * h * d
    dC = _f32_out(T * h, d, device=dZ.device)
    dWv, dWo = _f32_out(d, d, device=dZ.device), _f32_out(d, d, device=dZ.device)
    live = lambda t: t.data_ptr() if T > 0 else None  # noqa: E731
    _check(_lib.stca_output_backward(handle, layer, live(C), T, live(dZ), live(dC), dWv.data_ptr(),
                                     dWo.data_ptr(), _stream_ptr(stream)))
    return dC, dWv, dWo


def stca_query_backward(handle: int, layer: int, Q, dU, h: int, stream=None):
    """Gradients of u_j = (q W_Q^j) W_K^j^T / sqrt(d_h) (Eq. (13)): Q (T, d) and
    dU (T h, d), fp32 contiguous CUDA.  Returns dQ (T, d), dWq, dWk (d, d)."""
    import torch
    T, d = int(Q.shape[0]), int(Q.shape[1])
    assert Q.dtype == torch.float32 and dU.dtype == torch.float32
    assert Q.is_contiguous() and dU.is_contiguous() and dU.numel() == T * h * d
    dQ = _f32_out(T, d, device=Q.device)
    dWq, dWk = _f32_out(d, d, device=Q.device), _f32_out(d, d, device=Q.device)
    live = lambda t: t.data_ptr() if T > 0 else None  # noqa: E731
    _check(_lib.stca_query_backward(handle, layer, live(Q), T, live(dU), live(dQ), dWq.data_ptr(),
                                    dWk.data_ptr(), _stream_ptr(stream)))
    return dQ, dWq, dWk


def stca_query_init_backward(handle: int, targets, dq, rd: int, stream=None):
    """Gradients of q^(1) = LN(SwiGLUFFN(x_t)) (Eq. (3)) from dq (T x d fp32
    CUDA); targets: (T, d) CUDA, handle dtype.  Returns a dict of fp32 CUDA
    tensors dxt, dWu, dWg, dWd, dgamma, dbeta."""
    import torch
    T, d = int(targets.shape[0]), int(targets.shape[1])
    assert dq.dtype == torch.float32 and dq.is_contiguous() and targets.is_contiguous()
    dev = targets.device
    out = {"dxt": _f32_out(T, d, device=dev), "dWu": _f32_out(d, rd, device=dev),
           "dWg": _f32_out(d, rd, device=dev), "dWd": _f32_out(rd, d, device=dev),
           "dgamma": _f32_out(d, device=dev), "dbeta": _f32_out(d, device=dev)}
    _check(_lib.stca_query_init_backward(handle, targets.data_ptr(), T, dq.data_ptr(), out["dxt"].data_ptr(),
                                         out["dWu"].data_ptr(), out["dWg"].data_ptr(), out["dWd"].data_ptr(),
                                         out["dgamma"].data_ptr(), out["dbeta"].data_ptr(), _stream_ptr(stream)))
    return out


def stca_fusion_backward(handle: int, block: int, Z, targets, dy, rd: int, dZ=None, dxt=None,
                         accumulate=False, stream=None):
    """Gradients of the block-`block` fusion (Eq. (7) for block < M, the Eq. (9)
    head for block = M): Z (T, M, d) fp32, targets (T, d) handle dtype, dy
    (T, d) fp32, all CUDA.  dZ (T, M, d) / dxt (T, d) are written (or added to,
    with accumulate) in place when given, else allocated as zeros.  Returns a
    dict dZ, dxt, dW ((block+1) d, d), dWu, dWg, dWd."""
    import torch
    T, M, d = int(Z.shape[0]), int(Z.shape[1]), int(Z.shape[2])
    assert Z.dtype == torch.float32 and dy.dtype == torch.float32
    assert Z.is_contiguous() and dy.is_contiguous() and targets.is_contiguous()
    dev = Z.device
    if dZ is None:
        dZ = torch.zeros((T, M, d), dtype=torch.float32, device=dev)
    if dxt is None:
        dxt = torch.zeros((T, d), dtype=torch.float32, device=dev)
    assert dZ.is_contiguous() and dxt.is_contiguous()
    out = {"dZ": dZ, "dxt": dxt, "dW": _f32_out((block + 1) * d, d, device=dev),
           "dWu": _f32_out(d, rd, device=dev), "dWg": _f32_out(d, rd, device=dev),
           "dWd": _f32_out(rd, d, device=dev)}
    live = lambda t: t.data_ptr() if T > 0 else None  # noqa: E731
    _check(_lib.stca_fusion_backward(handle, block, live(Z), live(targets), T, live(dy), int(bool(accumulate)),
                                     live(dZ), live(dxt), out["dW"].data_ptr(), out["dWu"].data_ptr(),
                                     out["dWg"].data_ptr(), out["dWd"].data_ptr(), _stream_ptr(stream)))
    return out


def stca_forward_head(handle: int, targets, target_offsets, Z, zout, stream=None):
    """stca_forward and the Eq. (9) head token: Z (T, M, d) and zout (T, d), fp32 CUDA."""
    import torch
    toff = _offsets(target_offsets)
    T = int(toff[-1])
    assert Z.dtype == torch.float32 and zout.dtype == torch.float32
    _check(_lib.stca_forward_head(handle, targets.data_ptr() if T > 0 else None, _i64p(toff), T,
                                  Z.data_ptr() if T > 0 else None, zout.data_ptr() if T > 0 else None,
                                  _stream_ptr(stream)))
    return Z, zout


def stca_run_host(handle: int, X_host, offsets, targets_host, target_offsets, Z_host,
                  stream=None) -> None:
    """End-to-end on host buffers (numpy arrays or CPU tensors, ideally pinned)."""
    off, toff = _offsets(offsets), _offsets(target_offsets)

    def ptr(a):
        return a.data_ptr() if hasattr(a, "data_ptr") else a.ctypes.data
    _check(_lib.stca_run_host(handle, ptr(X_host), _i64p(off), off.shape[0] - 1, int(off[-1]),
                              ptr(targets_host), _i64p(toff), int(toff[-1]), ptr(Z_host),
                              _stream_ptr(stream)))


def stca_validate_offsets(offsets, total: int, require_nonempty: bool = True) -> int:
    off = _offsets(offsets)
    return _lib.stca_validate_offsets(_i64p(off), off.shape[0] - 1, total, int(require_nonempty))


def stca_device_status(handle: int, stream=None) -> None:
    _check(_lib.stca_device_status(handle, _stream_ptr(stream)))


def stca_selftest_ex2(x, y, method: int, stream=None) -> None:
    """y = 2^x on the device by the attention softmax's exponential: method 0
    the MUFU, 1 the FMA-pipe polynomial, 2 the same in pairs (packed fp32)."""
    import torch
    assert x.dtype == torch.float32 and y.dtype == torch.float32 and x.is_cuda and y.is_cuda
    assert x.is_contiguous() and y.is_contiguous() and x.numel() == y.numel()
    _check(_lib.stca_selftest_ex2(x.data_ptr(), y.data_ptr(), x.numel(), method, _stream_ptr(stream)))


def stca_set_option(handle: int, option: int, value: int) -> None:
    _check(_lib.stca_set_option(handle, option, value))


def stca_get_option(handle: int, option: int) -> int:
    v = ctypes.c_int64()
    _check(_lib.stca_get_option(handle, option, ctypes.byref(v)))
    return v.value


def stca_get_encoded(handle: int, layer: int, dst, stream=None):
    """Copy X~(layer+1) of the last encode into `dst` (CUDA tensor, N x d)."""
    _check(_lib.stca_get_encoded(handle, layer, dst.data_ptr(), _stream_ptr(stream)))
    return dst


def stca_plan_attention(offsets, target_offsets, h: int, path: int, num_ctas: int = 148,
                        split_keys: int = 0) -> dict:
    """The attention work split for a batch (host only).  Returns items as an
    (n, 7) int64 array: request, query tile, first key row, keys, first query
    row, query rows, first partial row; plus grid, partial_rows, cta_begin."""
    off, toff = _offsets(offsets), _offsets(target_offsets)
    R = off.shape[0] - 1
    n, g, rows = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(_lib.stca_plan_attention(_i64p(off), _i64p(toff), R, h, path, num_ctas, split_keys,
                                    ctypes.byref(n), ctypes.byref(g), ctypes.byref(rows),
                                    None, 0, None, 0))
    items = np.zeros((n.value, 7), dtype=np.int64)
    cta = np.zeros(g.value + 1, dtype=np.int32)
    _check(_lib.stca_plan_attention(_i64p(off), _i64p(toff), R, h, path, num_ctas, split_keys,
                                    ctypes.byref(n), ctypes.byref(g), ctypes.byref(rows),
                                    _i64p(items), items.shape[0],
                                    cta.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                    cta.shape[0]))
    return {"items": items, "grid": g.value, "partial_rows": rows.value, "cta_begin": cta}


def stca_kernel_times(handle: int):
    """{class: (ms, launches)} since the previous call (needs STCA_OPT_TIMING = 1)."""
    ms = (ctypes.c_double * STCA_K_CLASSES)()
    n = (ctypes.c_int64 * STCA_K_CLASSES)()
    _check(_lib.stca_kernel_times(handle, ms, n, STCA_K_CLASSES))
    names = ("encode", "attention", "target_step", "head", "pipe")
    return {names[c]: (ms[c], n[c]) for c in range(STCA_K_CLASSES)}


class Stca:
    """Owning wrapper: Stca(weights, d, h, r, M, dtype) then encode / forward."""

    def __init__(self, weights: dict, d: int, h: int, r: int, M: int, dtype: str = "bf16"):
        self.d, self.h, self.r, self.M = d, h, r, M
        self.dtype = STCA_BF16 if dtype == "bf16" else STCA_F32
        self.handle = stca_init(weights, d, h, r, M, self.dtype)

    def encode(self, X, offsets, stream=None):
        stca_encode(self.handle, X, offsets, stream)

    def forward(self, targets, target_offsets, Z=None, stream=None):
        import torch
        T = int(np.asarray(target_offsets)[-1])
        if Z is None:
            Z = torch.empty((T, self.M, self.d), dtype=torch.float32, device=targets.device)
        return stca_forward(self.handle, targets, target_offsets, Z, stream)

    def encode_forward(self, X, offsets, targets, target_offsets, Z=None, stream=None):
        """encode then forward in one call; returns Z."""
        import torch
        T = int(np.asarray(target_offsets)[-1])
        if Z is None:
            Z = torch.empty((T, self.M, self.d), dtype=torch.float32, device=targets.device)
        return stca_encode_forward(self.handle, X, offsets, targets, target_offsets, Z, stream)

    def forward_head(self, targets, target_offsets, Z=None, zout=None, stream=None):
        """Z of the forward and z of Eq. (9) in one call."""
        import torch
        T = int(np.asarray(target_offsets)[-1])
        if Z is None:
            Z = torch.empty((T, self.M, self.d), dtype=torch.float32, device=targets.device)
        if zout is None:
            zout = torch.empty((T, self.d), dtype=torch.float32, device=targets.device)
        return stca_forward_head(self.handle, targets, target_offsets, Z, zout, stream)

    def head(self, targets, Z, zout=None, stream=None):
        """z of Eq. (9) for every target: (T, d) fp32."""
        import torch
        if zout is None:
            zout = torch.empty((int(Z.shape[0]), self.d), dtype=torch.float32, device=Z.device)
        return stca_head(self.handle, targets, Z, zout, stream)

    def set_option(self, option: int, value: int):
        stca_set_option(self.handle, option, value)

    def get_option(self, option: int) -> int:
        return stca_get_option(self.handle, option)

    def status(self, stream=None):
        stca_device_status(self.handle, stream)

    def close(self):
        if self.handle:
            stca_destroy(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass
