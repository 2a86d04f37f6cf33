"""sfn_sparse_ffn_forward_static, the forward that allocates nothing.

It exists for callers that cannot allocate device memory when they run the
layer (a plugin interface that passes only input and output pointers, a
process whose allocator already owns the GPU's memory, a latency-critical
loop that must not risk cudaMalloc's synchronisation).  Its scratch is a
fixed array inside the library.  These tests call it through the C ABI and
compare it with the entry point that takes caller scratch, on the same
inputs: both run the same kernels in the same order, so the results must be
identical bit for bit.  The file is named to be collected last, so that a run
stopping at the first failure has already run every other test.
"""
import os
import re

import pytest
import torch

import predictor_gated_channel_b200 as sfn
from predictor_gated_channel_b200 import _capi
from predictor_gated_channel_b200 import build as sfn_build
from predictor_gated_channel_b200.inputs import WORKLOADS, make_layer, make_tokens

DEV = "cuda:0"
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "sfn.h")


def _lib():
    sfn_build.build()
    return _capi.lib()


def _static_call(L, dev, x, y, m, wl):
    T = x.shape[0]
    return L.sfn_sparse_ffn_forward_static(
        x.data_ptr(), dev["A"].data_ptr(), dev["B"].data_ptr(), dev["Wg"].data_ptr(),
        dev["Wu"].data_ptr(), dev["Wd"].data_ptr(), y.data_ptr(), m.data_ptr(), T, wl.d,
        wl.d_i, wl.r, wl.bank, wl.k, torch.cuda.current_stream().cuda_stream)


def _fits(L, wl, T):
    need = L.sfn_workspace_bytes(T, wl.d, wl.d_i, wl.r, wl.bank, wl.k, _capi.SFN_DTYPE_BF16)
    return 0 < need <= _capi.SFN_STATIC_SCRATCH_BYTES


def _documented_ranges():
    """The token counts the header promises to fit, for the 4096 x 14336 layer."""
    text = " ".join(open(HEADER).read().replace("*", " ").split())
    m = re.search(r"every T up to (\d+) fits, and T = (\d+) to (\d+)", text)
    assert m, "sfn.h no longer states the static scratch's token ranges"
    return int(m.group(1)), (int(m.group(2)), int(m.group(3)))


def test_documented_token_ranges_match_workspace_bytes():
    """The ranges the header states are exactly the T that sfn_workspace_bytes
    puts within SFN_STATIC_SCRATCH_BYTES (CPU only: a size query)."""
    L = _lib()
    wl = WORKLOADS["decode"]
    upto, (lo, hi) = _documented_ranges()
    fits = [T for T in range(1, 4097) if _fits(L, wl, T)]
    assert fits == list(range(1, upto + 1)) + list(range(lo, hi + 1)), fits


@pytest.mark.gpu
def test_static_scratch_forward_matches_allocating_entry_point():
    L = _lib()
    wl = WORKLOADS["decode"]
    dev = {k: v.to(DEV) for k, v in make_layer(wl).items()}
    upto, (lo, hi) = _documented_ranges()
    # the few-token kernels (1, 5), the tensor-core kernels at one token tile
    # (7, the largest T of the first range) and at two tiles (the last range)
    sizes = (1, 5, 7, upto, hi)
    cases = [make_tokens(wl, T=T, seed=40 + T).to(DEV) for T in sizes]
    refs = []
    for x in cases:
        T = x.shape[0]
        ws = torch.empty(L.sfn_workspace_bytes(T, wl.d, wl.d_i, wl.r, wl.bank, wl.k,
                                               _capi.SFN_DTYPE_BF16),
                         dtype=torch.uint8, device=DEV)
        refs.append(sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                           dev["Wd"], workspace=ws))
    torch.cuda.synchronize()
    # calls in a row on the one shared scratch array, with different inputs
    outs = []
    for x in cases:
        y = torch.full((x.shape[0], wl.d), float("nan"), dtype=torch.bfloat16, device=DEV)
        m = torch.zeros((x.shape[0], wl.n_banks), dtype=torch.int64, device=DEV)
        assert _static_call(L, dev, x, y, m, wl) == _capi.SFN_OK
        outs.append((y, m))
    torch.cuda.synchronize()
    for T, (y, m), (y_ref, m_ref) in zip(sizes, outs, refs):
        assert torch.equal(m, m_ref), T
        assert torch.equal(y, y_ref), T


def test_static_scratch_rejects_oversize_before_enqueueing():
    L = _lib()
    wl = WORKLOADS["decode"]
    upto, (lo, hi) = _documented_ranges()
    fake = 1 << 20  # never dereferenced: the size check comes first
    for T in (upto + 1, lo - 1, hi + 1, 4096):
        assert not _fits(L, wl, T), T
        rc = L.sfn_sparse_ffn_forward_static(*([fake] * 7), fake, T, wl.d, wl.d_i, wl.r,
                                             wl.bank, wl.k, None)
        assert rc == _capi.SFN_ERR_WORKSPACE, T
    assert L.sfn_sparse_ffn_forward_static(*([fake] * 7), None, 0, wl.d, wl.d_i, wl.r,
                                           wl.bank, wl.k, None) == _capi.SFN_OK
    assert L.sfn_sparse_ffn_forward_static(*([fake] * 7), None, 1, wl.d, wl.d_i, wl.r,
                                           wl.bank, 0, None) == _capi.SFN_ERR_INVALID_VALUE
