"""Predictor-gated bank-wise top-k sparse SwiGLU FFN forward on B200 (sm_100a).

Thin PyTorch-facing binding of the C ABI in ``include/sfn.h``: these functions
only check tensors and pass their device pointers and the current CUDA stream
to ``libsfn.so``; every step of the computation runs in the library's CUDA
kernels.  There is no CPU path: without the built library or a CUDA device
every call raises.

Method: "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity
Training Recipe for Dense-to-Sparse LLMs" (arXiv 2606.10722), gist.science
summary, "1. Architectuur" and "3. Hardware Implicaties".
"""
from __future__ import annotations

from . import _capi
from ._capi import SfnError

__all__ = ["predict", "bank_topk", "sparse_ffn_forward", "dense4x_forward", "workspace_bytes",
           "kernel_launch_count", "SfnError"]


def _torch():
    import torch
    return torch


def _stream_ptr(stream, device):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _dev(t, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _elt(dtype):
    torch = _torch()
    if dtype == torch.bfloat16:
        return _capi.SFN_DTYPE_BF16
    if dtype == torch.float32:
        return _capi.SFN_DTYPE_F32
    raise ValueError(f"unsupported dtype {dtype}: bf16 or float32")


def kernel_launch_count() -> int:
    """Kernels libsfn has launched in this process."""
    return int(_capi.lib().sfn_kernel_launch_count())


def workspace_bytes(T: int, d: int, d_i: int, r: int, bank: int, k: int, dtype) -> int:
    return int(_capi.lib().sfn_workspace_bytes(T, d, d_i, r, bank, k, _elt(dtype)))


def predict(x, A, B, out=None, stream=None):
    """Predictor logits p = B (A x) per token -> float32 [T, d_i]."""
    torch = _torch()
    for n, t in (("x", x), ("A", A), ("B", B)):
        _dev(t, n)
    T, d = x.shape
    r, d_i = A.shape[0], B.shape[0]
    if A.shape != (r, d) or B.shape != (d_i, r) or not (x.dtype == A.dtype == B.dtype):
        raise ValueError("predict: x [T,d], A [r,d], B [d_i,r] of one dtype")
    if out is None:
        out = torch.empty((T, d_i), dtype=torch.float32, device=x.device)
    _dev(out, "out")
    fn = (_capi.lib().sfn_predict if _elt(x.dtype) == _capi.SFN_DTYPE_BF16
          else _capi.lib().sfn_predict_f32)
    _capi.check(fn(x.data_ptr(), A.data_ptr(), B.data_ptr(), out.data_ptr(), T, d, d_i, r,
                   _stream_ptr(stream, x.device)), "sfn_predict")
    return out


def bank_topk(logits, bank: int = 64, k: int = 16, out=None, stream=None):
    """Bank-wise hard top-k of float32 logits [T, d_i] -> int64 [T, d_i/bank]
    holding the uint64 mask bit patterns (bit i of word b = channel b*bank+i)."""
    torch = _torch()
    _dev(logits, "logits")
    if logits.dtype != torch.float32:
        raise ValueError("bank_topk: logits must be float32")
    T, d_i = logits.shape
    if out is None:
        out = torch.empty((T, max(d_i // max(bank, 1), 0)), dtype=torch.int64,
                          device=logits.device)
    _dev(out, "out")
    _capi.check(_capi.lib().sfn_bank_topk(logits.data_ptr(), out.data_ptr(), T, d_i, bank, k,
                                          _stream_ptr(stream, logits.device)), "sfn_bank_topk")
    return out


PATHS = {"auto": _capi.SFN_PATH_AUTO, "cuda_core": _capi.SFN_PATH_CUDA_CORE,
         "tensor": _capi.SFN_PATH_TENSOR}


def sparse_ffn_forward(x, A, B, Wg, Wu, Wd, bank: int = 64, k: int = 16, y=None, mask=None,
                       workspace=None, want_mask: bool = True, path: str = "auto",
                       stream=None):
    """The sparse FFN forward.  Wd is channel-major: Wd[j] = W_down[:, j].

    Returns (y [T, d] in x's dtype, mask int64 [T, d_i/bank] or None).  With
    ``workspace`` (a uint8 CUDA tensor of at least ``workspace_bytes(...)``)
    the call uses it as scratch instead of allocating stream-ordered memory.
    ``path`` ("auto", "cuda_core" or "tensor") picks the kernels; a bf16
    call with an explicit path always uses caller scratch (allocated here
    when ``workspace`` is None).
    """
    torch = _torch()
    names = ("x", "A", "B", "Wg", "Wu", "Wd")
    ts = (x, A, B, Wg, Wu, Wd)
    for n, t in zip(names, ts):
        _dev(t, n)
    if len({t.dtype for t in ts}) != 1:
        raise ValueError("sparse_ffn_forward: all inputs must share one dtype")
    elt = _elt(x.dtype)
    T, d = x.shape
    r, d_i = A.shape[0], B.shape[0]
    if (A.shape != (r, d) or B.shape != (d_i, r) or Wg.shape != (d_i, d)
            or Wu.shape != (d_i, d) or Wd.shape != (d_i, d)):
        raise ValueError("sparse_ffn_forward: shapes x [T,d], A [r,d], B [d_i,r], "
                         "Wg/Wu/Wd [d_i,d]")
    if y is None:
        y = torch.empty((T, d), dtype=x.dtype, device=x.device)
    _dev(y, "y")
    if mask is None and want_mask:
        mask = torch.empty((T, max(d_i // max(bank, 1), 0)), dtype=torch.int64,
                           device=x.device)
    mptr = None
    if mask is not None:
        _dev(mask, "mask")
        mptr = mask.data_ptr()
    st = _stream_ptr(stream, x.device)
    L = _capi.lib()
    args = [x.data_ptr(), A.data_ptr(), B.data_ptr(), Wg.data_ptr(), Wu.data_ptr(),
            Wd.data_ptr(), y.data_ptr(), mptr, T, d, d_i, r, bank, k]
    if path != "auto":
        if elt != _capi.SFN_DTYPE_BF16:
            raise ValueError("an explicit path is available for bf16 only")
        if workspace is None:
            nbytes = workspace_bytes(T, d, d_i, r, bank, k, x.dtype)
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
        _dev(workspace, "workspace")
        _capi.check(L.sfn_sparse_ffn_forward_path(
            *args, PATHS[path], workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), st), "sfn_sparse_ffn_forward_path")
        return y, mask
    if workspace is None:
        fn = (L.sfn_sparse_ffn_forward if elt == _capi.SFN_DTYPE_BF16
              else L.sfn_sparse_ffn_forward_f32)
        _capi.check(fn(*args, st), "sfn_sparse_ffn_forward")
    else:
        _dev(workspace, "workspace")
        fn = (L.sfn_sparse_ffn_forward_ws if elt == _capi.SFN_DTYPE_BF16
              else L.sfn_sparse_ffn_forward_f32_ws)
        _capi.check(fn(*args, workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                       st), "sfn_sparse_ffn_forward_ws")
    return y, mask


def bank_shard(n_banks: int, rank: int, world: int) -> tuple:
    """Banks [b0, b1) of shard ``rank`` of ``world``: contiguous, sizes differing by
    at most one, covering every bank once."""
    if not 0 <= rank < world:
        raise ValueError("bank_shard: rank outside [0, world)")
    return n_banks * rank // world, n_banks * (rank + 1) // world


def sparse_ffn_forward_partial(x, A, B, Wg, Wu, Wd, bank: int = 64, k: int = 16,
                               y_partial=None, mask=None, workspace=None, path: str = "auto",
                               stream=None):
    """One bank shard of the layer (bf16): B, Wg, Wu, Wd hold only the shard's
    rows.  Returns (y_partial float32 [T, d], mask int64 [T, shard banks]); the
    sum of y_partial over a partition of the banks is the layer's y before
    rounding."""
    torch = _torch()
    for n, t in (("x", x), ("A", A), ("B", B), ("Wg", Wg), ("Wu", Wu), ("Wd", Wd)):
        _dev(t, n)
    T, d = x.shape
    r, d_i = A.shape[0], B.shape[0]
    if y_partial is None:
        y_partial = torch.empty((T, d), dtype=torch.float32, device=x.device)
    if mask is None:
        mask = torch.empty((T, max(d_i // max(bank, 1), 0)), dtype=torch.int64,
                           device=x.device)
    if workspace is None:
        nbytes = workspace_bytes(T, d, d_i, r, bank, k, x.dtype)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
    L = _capi.lib()
    _capi.check(L.sfn_sparse_ffn_forward_partial(
        x.data_ptr(), A.data_ptr(), B.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), Wd.data_ptr(),
        y_partial.data_ptr(), mask.data_ptr(), T, d, d_i, r, bank, k, PATHS[path],
        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
        _stream_ptr(stream, x.device)), "sfn_sparse_ffn_forward_partial")
    return y_partial, mask


def dense4x_forward(x, Wg, Wu, Wd, bank: int = 64, k: int = 16, y=None, mask=None,
                    workspace=None, stream=None):
    """The Dense-4x comparison (post-hoc amplitude top-k of the SwiGLU
    activation, no predictor).  bf16.  Returns (y [T, d], mask int64)."""
    torch = _torch()
    for n, t in (("x", x), ("Wg", Wg), ("Wu", Wu), ("Wd", Wd)):
        _dev(t, n)
    T, d = x.shape
    d_i = Wg.shape[0]
    if y is None:
        y = torch.empty((T, d), dtype=x.dtype, device=x.device)
    if mask is None:
        mask = torch.empty((T, max(d_i // max(bank, 1), 0)), dtype=torch.int64, device=x.device)
    L = _capi.lib()
    if workspace is None:
        nbytes = int(L.sfn_dense4x_workspace_bytes(T, d, d_i, bank, k))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
    _capi.check(L.sfn_dense4x_forward(x.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), Wd.data_ptr(),
                                      y.data_ptr(), mask.data_ptr(), T, d, d_i, bank, k,
                                      workspace.data_ptr(),
                                      workspace.numel() * workspace.element_size(),
                                      _stream_ptr(stream, x.device)), "sfn_dense4x_forward")
    return y, mask


def sparse_ffn_backward(x, A, B, Wg, Wu, Wd, dy, bank: int = 64, k: int = 16,
                        temperature: float = 1.0, want=("dx", "dA", "dB", "dWg", "dWu", "dWd"),
                        workspace=None, stream=None) -> dict:
    """Gradients of the layer for dy = dL/dy (bf16 inputs, float32 outputs),
    with the soft surrogate gradient of the bank top-k (see
    ``sfn_sparse_ffn_backward`` in include/sfn.h).  Returns a dict holding
    the gradients named in ``want`` and the forward's ``mask``."""
    torch = _torch()
    for n, t in (("x", x), ("A", A), ("B", B), ("Wg", Wg), ("Wu", Wu), ("Wd", Wd), ("dy", dy)):
        _dev(t, n)
    T, d = x.shape
    r = A.shape[0]
    d_i = B.shape[0]
    f32 = dict(dtype=torch.float32, device=x.device)
    shapes = {"dx": (T, d), "dA": (r, d), "dB": (d_i, r), "dWg": (d_i, d), "dWu": (d_i, d),
              "dWd": (d_i, d)}
    out = {n: torch.empty(shapes[n], **f32) for n in want}
    out["mask"] = torch.empty((T, max(d_i // max(bank, 1), 0)), dtype=torch.int64,
                              device=x.device)
    L = _capi.lib()
    if workspace is None:
        nbytes = int(L.sfn_backward_workspace_bytes(T, d, d_i, r, bank, k))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)

    def ptr(n):
        return out[n].data_ptr() if n in out else None

    _capi.check(L.sfn_sparse_ffn_backward(
        x.data_ptr(), A.data_ptr(), B.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), Wd.data_ptr(),
        dy.data_ptr(), float(temperature), ptr("dx"), ptr("dA"), ptr("dB"), ptr("dWg"),
        ptr("dWu"), ptr("dWd"), out["mask"].data_ptr(), T, d, d_i, r, bank, k,
        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
        _stream_ptr(stream, x.device)), "sfn_sparse_ffn_backward")
    return out
