"""Plain fp64 CPU oracle for the predictor-gated bank-wise top-k sparse SwiGLU FFN.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library ``libsfn.so`` and its Python binding) never calls it, and the
two share no code: the only thing both sides see is the seeded input generator,
which holds none of the method's arithmetic.

The arithmetic lives in ``sfn_oracle.c`` (double-precision loops, OpenMP over
tokens only), following "Continual LLM Upcycling: A Predictor-Gated Bank-Wise
Sparsity Training Recipe for Dense-to-Sparse LLMs" as summarised on
gist.science, "Methodologie / 1. Architectuur" and "3. Hardware Implicaties".
This module only marshals arrays into it.

Every function takes arrays as numpy float64 / float32, numpy uint16 holding
bf16 bit patterns, or CPU torch tensors of those types (bf16 included); they
are widened exactly to double inside the C code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sfn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsfn_oracle.so")

F64, F32, BF16 = 0, 1, 2

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile sfn_oracle.c into libsfn_oracle.so with gcc (no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fno-fast-math", "-ffp-contract=off",
           "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _open(path: str):
    """Open a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.sfn_oracle_sigmoid.restype = ctypes.c_double
    lib.sfn_oracle_sigmoid.argtypes = [ctypes.c_double]
    lib.sfn_oracle_predict.argtypes = [vp, ci, vp, ci, vp, ci, i64, ci, ci, ci, vp]
    lib.sfn_oracle_bank_topk.argtypes = [vp, i64, ci, ci, ci, vp]
    lib.sfn_oracle_forward_given_mask.argtypes = [
        vp, ci, vp, vp, vp, ci, vp, ci, vp, ci, i64, ci, ci, ci, vp]
    lib.sfn_oracle_forward.argtypes = [
        vp, ci, vp, ci, vp, ci, vp, ci, vp, ci, vp, ci, i64, ci, ci, ci, ci, ci,
        vp, vp, vp]
    lib.sfn_oracle_dense_then_mask.argtypes = [
        vp, ci, vp, vp, vp, ci, vp, ci, vp, ci, i64, ci, ci, ci, vp]
    lib.sfn_oracle_backward.argtypes = [vp, ci, vp, ci, vp, ci, vp, ci, vp, ci, vp, ci, vp, ci,
                                        i64, ci, ci, ci, ci, ci, ctypes.c_double, vp, vp, vp,
                                        vp, vp, vp, vp, vp]
    lib.sfn_oracle_num_threads.restype = ci
    lib.sfn_oracle_dense4x.argtypes = [vp, ci, vp, ci, vp, ci, vp, ci, i64, ci, ci, ci, ci, ci,
                                       vp, vp, vp]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(build())
        return _lib


def _arr(a):
    """Return (contiguous numpy array, dtype code) for a supported input."""
    if hasattr(a, "detach") and hasattr(a, "dtype"):  # torch tensor
        import torch  # local: the oracle itself does not need torch
        t = a.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16), BF16
        a = t.numpy()
    a = np.ascontiguousarray(a)
    if a.dtype == np.float64:
        return a, F64
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle: unsupported dtype {a.dtype}")


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def num_threads() -> int:
    return int(_load().sfn_oracle_num_threads())


def sigmoid(z: float) -> float:
    """Logistic function in double precision."""
    return float(_load().sfn_oracle_sigmoid(float(z)))


def predict(x, A, B) -> np.ndarray:
    """Predictor logits p = B (A x) per token: float64 [T, d_i]."""
    xa, xd = _arr(x)
    Aa, Ad = _arr(A)
    Ba, Bd = _arr(B)
    T, d = xa.shape
    r, d2 = Aa.shape
    d_i, r2 = Ba.shape
    assert d2 == d and r2 == r
    out = np.empty((T, d_i), np.float64)
    _load().sfn_oracle_predict(_ptr(xa), xd, _ptr(Aa), Ad, _ptr(Ba), Bd, T, d, d_i, r,
                               _ptr(out))
    return out


def bank_topk(logits, bank: int, k: int) -> np.ndarray:
    """Bank-wise hard top-k mask: uint64 [T, d_i // bank]; ties to the lower index.

    float32 logits are widened exactly, so this is also the bit-exact reference
    for a top-k that runs on float32 logits.
    """
    la = np.ascontiguousarray(np.asarray(logits, dtype=np.float64))
    T, d_i = la.shape
    assert d_i % bank == 0 and 1 <= k <= bank <= 64
    out = np.empty((T, d_i // bank), np.uint64)
    _load().sfn_oracle_bank_topk(_ptr(la), T, d_i, bank, k, _ptr(out))
    return out


def forward_given_mask(x, logits, mask, Wg, Wu, Wd, bank: int) -> np.ndarray:
    """Sparse gate/up/down for a given mask: y float64 [T, d]."""
    xa, xd = _arr(x)
    la = np.ascontiguousarray(np.asarray(logits, dtype=np.float64))
    ma = np.ascontiguousarray(np.asarray(mask, dtype=np.uint64))
    ga, gd = _arr(Wg)
    ua, ud = _arr(Wu)
    da, dd = _arr(Wd)
    T, d = xa.shape
    d_i = la.shape[1]
    assert ga.shape == (d_i, d) and ua.shape == (d_i, d) and da.shape == (d_i, d)
    assert ma.shape == (T, d_i // bank)
    y = np.empty((T, d), np.float64)
    _load().sfn_oracle_forward_given_mask(_ptr(xa), xd, _ptr(la), _ptr(ma), _ptr(ga), gd,
                                          _ptr(ua), ud, _ptr(da), dd, T, d, d_i, bank,
                                          _ptr(y))
    return y


def forward(x, A, B, Wg, Wu, Wd, bank: int, k: int):
    """Whole forward.  Returns (y [T, d], logits [T, d_i], mask [T, d_i/bank])."""
    xa, xd = _arr(x)
    Aa, Ad = _arr(A)
    Ba, Bd = _arr(B)
    ga, gd = _arr(Wg)
    ua, ud = _arr(Wu)
    da, dd = _arr(Wd)
    T, d = xa.shape
    r = Aa.shape[0]
    d_i = Ba.shape[0]
    assert d_i % bank == 0 and 1 <= k <= bank <= 64
    logits = np.empty((T, d_i), np.float64)
    mask = np.empty((T, d_i // bank), np.uint64)
    y = np.empty((T, d), np.float64)
    _load().sfn_oracle_forward(_ptr(xa), xd, _ptr(Aa), Ad, _ptr(Ba), Bd, _ptr(ga), gd,
                               _ptr(ua), ud, _ptr(da), dd, T, d, d_i, r, bank, k,
                               _ptr(logits), _ptr(mask), _ptr(y))
    return y, logits, mask


def dense_then_mask(x, logits, mask, Wg, Wu, Wd, bank: int) -> np.ndarray:
    """Dense gate/up for every channel, multiply by the 0/1 mask, dense down."""
    xa, xd = _arr(x)
    la = np.ascontiguousarray(np.asarray(logits, dtype=np.float64))
    ma = np.ascontiguousarray(np.asarray(mask, dtype=np.uint64))
    ga, gd = _arr(Wg)
    ua, ud = _arr(Wu)
    da, dd = _arr(Wd)
    T, d = xa.shape
    d_i = la.shape[1]
    y = np.empty((T, d), np.float64)
    _load().sfn_oracle_dense_then_mask(_ptr(xa), xd, _ptr(la), _ptr(ma), _ptr(ga), gd,
                                       _ptr(ua), ud, _ptr(da), dd, T, d, d_i, bank,
                                       _ptr(y))
    return y


def dense4x(x, Wg, Wu, Wd, bank: int, k: int, mask=None, want_act: bool = False):
    """The Dense-4x comparison: SwiGLU act = silu(g) u, per bank keep the k
    largest |act|, y = sum of kept act_j Wd[j].  Returns (y [T, d], mask) and,
    with want_act, also act [T, d_i].  With ``mask`` given, that mask is
    applied instead of the amplitude top-k."""
    xa, xd = _arr(x)
    ga, gd = _arr(Wg)
    ua, ud = _arr(Wu)
    da, dd = _arr(Wd)
    T, d = xa.shape
    d_i = ga.shape[0]
    assert d_i % bank == 0 and 1 <= k <= bank <= 64
    given = mask is not None
    m = (np.ascontiguousarray(np.asarray(mask, dtype=np.uint64)).copy() if given
         else np.empty((T, d_i // bank), np.uint64))
    act = np.empty((T, d_i), np.float64) if want_act else None
    y = np.empty((T, d), np.float64)
    _load().sfn_oracle_dense4x(_ptr(xa), xd, _ptr(ga), gd, _ptr(ua), ud, _ptr(da), dd, T, d, d_i,
                               bank, k, int(given), _ptr(m),
                               _ptr(act) if want_act else None, _ptr(y))
    return (y, m, act) if want_act else (y, m)


def mask_to_bool(mask, bank: int) -> np.ndarray:
    """Expand a uint64 [T, nb] mask into a bool [T, nb*bank] channel mask."""
    m = np.asarray(mask, dtype=np.uint64)
    bits = (m[..., None] >> np.arange(bank, dtype=np.uint64)) & np.uint64(1)
    return bits.reshape(m.shape[0], -1).astype(bool)


def backward(x, A, B, Wg, Wu, Wd, dy, bank: int, k: int, temp: float, mask=None) -> dict:
    """Gradients of L = sum(dy * y) through the whole layer, with the soft
    surrogate gradient of the hard top-k (threshold tau_b = midpoint of the
    bank's k-th and (k+1)-th logits, held constant; dm/dp := sigma'((p -
    tau_b) / temp) / temp).  Returns float64 arrays dx [T, d], dA [r, d],
    dB [d_i, r], dWg, dWu, dWd [d_i, d] and the mask used (uint64 [T, d_i /
    bank]).  With ``mask`` given, that mask replaces the own top-k."""
    xa, xd = _arr(x)
    Aa, Ad = _arr(A)
    Ba, Bd = _arr(B)
    ga, gd = _arr(Wg)
    ua, ud = _arr(Wu)
    wa, wd = _arr(Wd)
    ya, yd = _arr(dy)
    T, d = xa.shape
    r = Aa.shape[0]
    d_i = Ba.shape[0]
    assert Aa.shape == (r, d) and Ba.shape == (d_i, r) and ya.shape == (T, d)
    assert ga.shape == ua.shape == wa.shape == (d_i, d)
    assert d_i % bank == 0 and 1 <= k <= bank <= 64 and temp > 0
    nb = d_i // bank
    out = {"dx": np.empty((T, d)), "dA": np.empty((r, d)), "dB": np.empty((d_i, r)),
           "dWg": np.empty((d_i, d)), "dWu": np.empty((d_i, d)), "dWd": np.empty((d_i, d)),
           "mask": np.empty((T, nb), np.uint64)}
    m_in = None
    if mask is not None:
        if hasattr(mask, "detach"):
            mask = mask.detach().cpu().numpy()
        m_in = np.ascontiguousarray(np.asarray(mask))
        m_in = m_in.view(np.uint64) if m_in.dtype == np.int64 else m_in.astype(np.uint64)
        assert m_in.shape == (T, nb)
    _load().sfn_oracle_backward(_ptr(xa), xd, _ptr(Aa), Ad, _ptr(Ba), Bd, _ptr(ga), gd, _ptr(ua),
                                ud, _ptr(wa), wd, _ptr(ya), yd, T, d, d_i, r, bank, k,
                                float(temp), None if m_in is None else _ptr(m_in),
                                _ptr(out["dx"]), _ptr(out["dA"]), _ptr(out["dB"]),
                                _ptr(out["dWg"]), _ptr(out["dWu"]), _ptr(out["dWd"]),
                                _ptr(out["mask"]))
    return out
