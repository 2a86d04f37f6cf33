"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before enqueueing anything (no GPU needed:
none of these calls reaches a kernel)."""
import ctypes
import os
import re

import pytest

from predictor_gated_channel_b200 import _capi
from predictor_gated_channel_b200 import build as sfn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    sfn_build.build()
    return _capi.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "sfn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sfn_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), f"{n} declared in sfn.h but not exported"
    assert set(names) == set(_capi.SIGNATURES), "binding and header disagree"


def test_status_strings_and_version(L):
    assert L.sfn_abi_version() == 2
    for s in range(6):
        assert L.sfn_status_string(s).decode().startswith("SFN_")
    assert b"unknown" in L.sfn_status_string(99)
    assert isinstance(L.sfn_kernel_launch_count(), int)


FAKE = 1 << 20          # 16-byte aligned, never dereferenced: rejected first
SHAPE = dict(T=1, d=4096, d_i=14336, r=448, bank=64, k=16)


def fwd(L, T=1, d=4096, d_i=14336, r=448, bank=64, k=16, ptrs=None, mask=None, f32=False):
    p = ptrs or [FAKE] * 7
    fn = L.sfn_sparse_ffn_forward_f32 if f32 else L.sfn_sparse_ffn_forward
    return fn(*p, mask, T, d, d_i, r, bank, k, None)


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), _capi.SFN_ERR_INVALID_VALUE),
    (dict(d=0), _capi.SFN_ERR_INVALID_VALUE),
    (dict(r=-3), _capi.SFN_ERR_INVALID_VALUE),
    (dict(d_i=14335), _capi.SFN_ERR_INVALID_VALUE),   # not a multiple of bank
    (dict(k=0), _capi.SFN_ERR_INVALID_VALUE),
    (dict(k=65, bank=64), _capi.SFN_ERR_INVALID_VALUE),
    (dict(bank=65, d_i=65 * 4), _capi.SFN_ERR_INVALID_VALUE),
    (dict(k=17, bank=16), _capi.SFN_ERR_INVALID_VALUE),
    (dict(d=4100), _capi.SFN_ERR_MISALIGNED),          # 4100 bf16 = 8200 B rows
    (dict(r=100), _capi.SFN_ERR_MISALIGNED),
    (dict(d=32768), _capi.SFN_ERR_UNSUPPORTED),
    (dict(r=4096), _capi.SFN_ERR_UNSUPPORTED),
])
def test_invalid_shapes_rejected(L, kw, status):
    assert fwd(L, **kw) == status


def test_null_and_misaligned_pointers(L):
    for i in range(7):
        p = [FAKE] * 7
        p[i] = None
        assert fwd(L, ptrs=p) == _capi.SFN_ERR_INVALID_VALUE
        p[i] = FAKE + 8
        assert fwd(L, ptrs=p) == _capi.SFN_ERR_MISALIGNED
    assert fwd(L, mask=FAKE + 4) == _capi.SFN_ERR_MISALIGNED


def test_f32_row_alignment(L):
    assert fwd(L, d=4098, f32=True) == _capi.SFN_ERR_MISALIGNED   # 4098*4 B rows
    assert fwd(L, d=4100, f32=True) != _capi.SFN_ERR_MISALIGNED


def test_zero_tokens_is_noop(L):
    # T == 0 returns OK without inspecting pointers or touching a device
    assert fwd(L, T=0, ptrs=[None] * 7) == _capi.SFN_OK
    assert L.sfn_predict(None, None, None, None, 0, 4096, 14336, 448, None) == _capi.SFN_OK
    assert L.sfn_bank_topk(None, None, 0, 14336, 64, 16, None) == _capi.SFN_OK


def test_workspace_checks(L):
    need = L.sfn_workspace_bytes(1, 4096, 14336, 448, 64, 16, _capi.SFN_DTYPE_BF16)
    assert need > 0 and need % 256 == 0
    assert L.sfn_workspace_bytes(0, 4096, 14336, 448, 64, 16, 0) == 0
    assert L.sfn_workspace_bytes(1, 4096, 14336, 448, 64, 16, 7) == 0
    assert L.sfn_workspace_bytes(-1, 4096, 14336, 448, 64, 16, 0) == 0
    args = [FAKE] * 7 + [None, 1, 4096, 14336, 448, 64, 16]
    assert L.sfn_sparse_ffn_forward_ws(*args, None, need, None) == _capi.SFN_ERR_WORKSPACE
    assert L.sfn_sparse_ffn_forward_ws(*args, FAKE, 256, None) == _capi.SFN_ERR_WORKSPACE
    assert L.sfn_sparse_ffn_forward_ws(*args, FAKE + 16, need, None) == _capi.SFN_ERR_WORKSPACE
    # scratch grows with T
    assert (L.sfn_workspace_bytes(64, 4096, 14336, 448, 64, 16, 0)
            > L.sfn_workspace_bytes(1, 4096, 14336, 448, 64, 16, 0))


def test_topk_and_predict_validation(L):
    assert L.sfn_bank_topk(FAKE, FAKE, 1, 14336, 64, 0, None) == _capi.SFN_ERR_INVALID_VALUE
    assert L.sfn_bank_topk(FAKE, FAKE, 1, 100, 64, 16, None) == _capi.SFN_ERR_INVALID_VALUE
    assert L.sfn_bank_topk(None, FAKE, 1, 128, 64, 16, None) == _capi.SFN_ERR_INVALID_VALUE
    assert L.sfn_bank_topk(FAKE + 2, FAKE, 1, 128, 64, 16, None) == _capi.SFN_ERR_MISALIGNED
    assert L.sfn_bank_topk(FAKE, FAKE + 4, 1, 128, 64, 16, None) == _capi.SFN_ERR_MISALIGNED
    assert L.sfn_predict(FAKE, FAKE, FAKE, FAKE, 1, 4096, 14336, 100, None) == \
        _capi.SFN_ERR_MISALIGNED
    assert L.sfn_predict(FAKE, None, FAKE, FAKE, 1, 4096, 14336, 448, None) == \
        _capi.SFN_ERR_INVALID_VALUE


def test_no_cpu_fallback():
    """Without a CUDA device a valid call fails with SFN_ERR_CUDA; it never
    computes on the host."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    sfn_build.build()
    assert fwd(_capi.lib()) == _capi.SFN_ERR_CUDA


def test_dense4x_validation(L):
    need = L.sfn_dense4x_workspace_bytes(4, 4096, 14336, 64, 16)
    assert need > 0 and need % 256 == 0
    assert L.sfn_dense4x_workspace_bytes(0, 4096, 14336, 64, 16) == 0
    args = [FAKE] * 5 + [None]
    # shapes the tensor cores do not cover
    assert L.sfn_dense4x_forward(*args, 4, 4096, 14336, 32, 8, FAKE, need, None) == \
        _capi.SFN_ERR_UNSUPPORTED
    assert L.sfn_dense4x_forward(*args, 4, 4160, 14336, 64, 16, FAKE, need, None) == \
        _capi.SFN_ERR_UNSUPPORTED
    assert L.sfn_dense4x_forward(*args, 4, 4096, 14336, 64, 0, FAKE, need, None) == \
        _capi.SFN_ERR_INVALID_VALUE
    assert L.sfn_dense4x_forward(*args, 0, 4096, 14336, 64, 16, None, 0, None) == _capi.SFN_OK
    assert L.sfn_dense4x_forward(*args, 4, 4096, 14336, 64, 16, FAKE, 256, None) == \
        _capi.SFN_ERR_WORKSPACE
    p = [FAKE] * 5
    p[0] = None
    assert L.sfn_dense4x_forward(*p, None, 4, 4096, 14336, 64, 16, FAKE, need, None) == \
        _capi.SFN_ERR_INVALID_VALUE
    p[0] = FAKE + 8
    assert L.sfn_dense4x_forward(*p, None, 4, 4096, 14336, 64, 16, FAKE, need, None) == \
        _capi.SFN_ERR_MISALIGNED


def test_path_selector_validation(L):
    args = [FAKE] * 7 + [None, 4, 4096, 14336, 448, 64, 16]
    need = L.sfn_workspace_bytes(4, 4096, 14336, 448, 64, 16, 0)
    assert L.sfn_sparse_ffn_forward_path(*args, 7, FAKE, need, None) == _capi.SFN_ERR_INVALID_VALUE
    bad = [FAKE] * 7 + [None, 4, 4096, 14336, 448, 32, 8]
    assert L.sfn_sparse_ffn_forward_path(*bad, _capi.SFN_PATH_TENSOR, FAKE, need, None) == \
        _capi.SFN_ERR_UNSUPPORTED
    assert L.sfn_last_error_string() is not None


def test_backward_validation(L):
    need = L.sfn_backward_workspace_bytes(4, 4096, 14336, 448, 64, 16)
    assert need > 0 and need % 256 == 0
    assert L.sfn_backward_workspace_bytes(0, 4096, 14336, 448, 64, 16) == 0
    assert L.sfn_backward_workspace_bytes(4, 4096, 14336, 448, 64, 0) == 0
    ins = [FAKE] * 7
    grads = [FAKE] * 6 + [None]

    def bwd(temp=1.0, T=4, d=4096, d_i=14336, r=448, bank=64, k=16, ins=ins, grads=grads,
            ws=FAKE, ws_bytes=need):
        return L.sfn_sparse_ffn_backward(*ins, temp, *grads, T, d, d_i, r, bank, k, ws,
                                         ws_bytes, None)
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert bwd(temp=bad) == _capi.SFN_ERR_INVALID_VALUE
    assert bwd(k=0) == _capi.SFN_ERR_INVALID_VALUE
    assert bwd(d_i=14330, bank=10, k=2) == _capi.SFN_ERR_UNSUPPORTED  # d_i % 4 != 0
    assert bwd(T=0, ws=None, ws_bytes=0) == _capi.SFN_OK
    assert bwd(ws_bytes=need - 256) == _capi.SFN_ERR_WORKSPACE
    p = list(ins)
    p[6] = None  # dy
    assert bwd(ins=p) == _capi.SFN_ERR_INVALID_VALUE
    g = list(grads)
    g[3] = FAKE + 4  # dWg misaligned
    assert bwd(grads=g) == _capi.SFN_ERR_MISALIGNED
