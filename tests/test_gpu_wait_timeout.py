"""The bounded pipeline wait gives up instead of hanging, and the device
stays usable afterwards.

Every mbarrier wait in the library's kernels is bounded: after a limit of SM
clock cycles it sets bit 1 of the device error word and the kernel returns.
No correct pipeline reaches that branch, so sfn_debug_wait_timeout launches a
warp that waits on a barrier nothing completes, with a short limit (nothing
else is in flight).  The test checks that the wait gave up, that the host
reads the error bit, and that a full forward afterwards still matches the
oracle with the error word clear.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import parity
import predictor_gated_channel_b200 as sfn
from predictor_gated_channel_b200 import _capi
from predictor_gated_channel_b200 import build as sfn_build
from predictor_gated_channel_b200.inputs import WORKLOADS, make_layer, make_tokens

DEV = "cuda:0"


def _lib():
    sfn_build.build()
    return _capi.lib()


def test_wait_probe_rejects_bad_arguments():
    L = _lib()
    for limit in (0, -5, 10**9 + 1, 1 << 40):
        assert L.sfn_debug_wait_timeout(limit, None, None) == _capi.SFN_ERR_INVALID_VALUE
    assert L.sfn_debug_wait_timeout(1000, (1 << 20) + 2, None) == _capi.SFN_ERR_MISALIGNED


def _errors(L, clear):
    bits = ctypes.c_uint(0)
    assert L.sfn_device_errors(ctypes.byref(bits), 1 if clear else 0) == _capi.SFN_OK
    return bits.value


@pytest.mark.gpu
def test_bounded_wait_gives_up_and_device_stays_usable():
    L = _lib()
    assert _errors(L, clear=True) == 0
    gave_up = torch.zeros(1, dtype=torch.int32, device=DEV)
    st = torch.cuda.current_stream()
    # about a millisecond of SM clock
    assert L.sfn_debug_wait_timeout(2_000_000, gave_up.data_ptr(), st.cuda_stream) == \
        _capi.SFN_OK
    torch.cuda.synchronize()
    assert int(gave_up.item()) == 1
    assert _errors(L, clear=True) == 1  # kDevErrWaitTimeout, read and cleared
    assert _errors(L, clear=False) == 0

    # the context still works: a full-width forward on both kernel paths
    wl = WORKLOADS["decode"]
    host = make_layer(wl)
    dev = {k: v.to(DEV) for k, v in host.items()}
    for T in (1, 8):
        x = make_tokens(wl, T=T, seed=77 + T)
        y, mask = sfn.sparse_ffn_forward(x.to(DEV), dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                         dev["Wd"])
        torch.cuda.synchronize()
        logits = oracle.predict(x, host["A"], host["B"])
        gm = parity.to_u64(mask)
        parity.check_mask(gm, logits, wl.bank, wl.k)
        y_ref = oracle.forward_given_mask(x, logits, gm, host["Wg"], host["Wu"], host["Wd"],
                                          wl.bank)
        err = parity.y_error(y.float().cpu().numpy(), y_ref)
        assert err <= parity.Y_TOL["bf16"], err
    assert _errors(L, clear=False) == 0
