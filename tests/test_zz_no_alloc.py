"""sfn_sparse_ffn_forward_static, the forward that allocates nothing.

It exists for callers that cannot allocate device memory when they run the
layer (a plugin interface that passes only input and output pointers, a
process whose allocator already owns the GPU's memory, a latency-critical
loop that must not risk cudaMalloc's synchronisation).  Its scratch is a
fixed array inside the library.  These tests call it through the C ABI and
compare it with the allocating entry point on the same inputs.  The file is
named to be collected last, so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import parity
import predictor_gated_channel_b200 as sfn
from predictor_gated_channel_b200 import _capi
from predictor_gated_channel_b200 import build as sfn_build
from predictor_gated_channel_b200.inputs import WORKLOADS, make_layer, make_tokens

DEV = "cuda:0"


def _static_call(L, dev, x, y, m, wl):
    T = x.shape[0]
    return L.sfn_sparse_ffn_forward_static(
        x.data_ptr(), dev["A"].data_ptr(), dev["B"].data_ptr(), dev["Wg"].data_ptr(),
        dev["Wu"].data_ptr(), dev["Wd"].data_ptr(), y.data_ptr(), m.data_ptr(), T, wl.d,
        wl.d_i, wl.r, wl.bank, wl.k, torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_static_scratch_forward_matches_allocating_entry_point():
    sfn_build.build()
    L = _capi.lib()
    wl = WORKLOADS["decode"]
    dev = {k: v.to(DEV) for k, v in make_layer(wl).items()}
    cases = [make_tokens(wl, T=T, seed=40 + T).to(DEV) for T in (1, 7)]
    refs = [sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"], dev["Wd"])
            for x in cases]
    torch.cuda.synchronize()
    # two calls in a row on the shared scratch, with different inputs
    outs = []
    for x in cases:
        y = torch.full((x.shape[0], wl.d), float("nan"), dtype=torch.bfloat16, device=DEV)
        m = torch.zeros((x.shape[0], wl.n_banks), dtype=torch.int64, device=DEV)
        assert _static_call(L, dev, x, y, m, wl) == _capi.SFN_OK
        outs.append((y, m))
    torch.cuda.synchronize()
    for (y, m), (y_ref, m_ref) in zip(outs, refs):
        assert torch.equal(m, m_ref)
        err = parity.y_error(y.float().cpu().numpy(), y_ref.float().cpu().numpy().astype(np.float64))
        assert err <= parity.Y_TOL["bf16"], err


def test_static_scratch_rejects_oversize_before_enqueueing():
    sfn_build.build()
    L = _capi.lib()
    wl = WORKLOADS["decode"]
    T = 4096
    assert L.sfn_workspace_bytes(T, wl.d, wl.d_i, wl.r, wl.bank, wl.k, 0) > \
        _capi.SFN_STATIC_SCRATCH_BYTES
    fake = 1 << 20  # never dereferenced: the size check comes first
    rc = L.sfn_sparse_ffn_forward_static(*([fake] * 7), fake, T, wl.d, wl.d_i, wl.r, wl.bank,
                                         wl.k, None)
    assert rc == _capi.SFN_ERR_WORKSPACE
    assert L.sfn_sparse_ffn_forward_static(*([fake] * 7), None, 0, wl.d, wl.d_i, wl.r,
                                           wl.bank, wl.k, None) == _capi.SFN_OK
    assert L.sfn_sparse_ffn_forward_static(*([fake] * 7), None, 1, wl.d, wl.d_i, wl.r,
                                           wl.bank, 0, None) == _capi.SFN_ERR_INVALID_VALUE
