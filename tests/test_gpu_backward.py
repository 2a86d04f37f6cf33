"""Parity of the backward (soft surrogate gradient of the bank top-k) with the
fp64 oracle, through the C ABI.

The oracle runs on the GPU's own mask (a mask flip allowed by the forward's
rule changes which channels carry gradient, so it is not counted as error);
the mask itself is checked with the forward's rule.  Gradients come from bf16
GEMM operands with float32 accumulation, so each is compared row by row, like
the forward's y:

    max |gpu - oracle| over a row <= 2e-2 * max(max |oracle row|, 1e-4 * max |oracle|)

(2e-2 is the bf16 tolerance of the forward), and a row the oracle gives as
exactly zero (a channel no token keeps, in dWg, dWu, dWd) must be exactly
zero.  The floor covers rows that are small only because a factor of theirs
nearly cancels: in the full-width layer, g_j = W_gate[j] . x can be 1e-4 while
its terms sum to 40 in magnitude, and float32 accumulation in any order then
leaves about 1e-2 relative error in g_j and in the whole weight-gradient row
built from it.  Below 1e-4 of the matrix's largest row the check is absolute,
at 2e-6 of that row -- ten thousand times tighter than one bound for the
whole matrix.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
import predictor_gated_channel_b200 as sfn
from predictor_gated_channel_b200 import _capi
from predictor_gated_channel_b200 import build as sfn_build
from predictor_gated_channel_b200.inputs import WORKLOADS, Workload, make_layer, make_tokens

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GRAD_TOL = 2e-2
NAMES = ("dx", "dA", "dB", "dWg", "dWu", "dWd")
# small bf16 layer whose shapes the tensor-core kernels cover (d, d_i
# multiples of 256, r a multiple of 64, bank 64)
SMALL = Workload("bwd_small", 64, 256, 1024, 64, 64, 16, "bf16", "rmsnorm", 1.0 / math.sqrt(1024))


@pytest.fixture(scope="module", autouse=True)
def _built():
    sfn_build.build()
    _capi.lib()


@pytest.fixture(scope="module")
def full_layer():
    wl = WORKLOADS["decode"]
    host = make_layer(wl)
    return wl, host, {n: v.to(DEV) for n, v in host.items()}


def _dy(T, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((T, d), generator=g).to(torch.bfloat16)


def _run(wl, host, dev, T, bank, k, temp, want=NAMES):
    x = make_tokens(wl, T=T, seed=3)
    dy = _dy(T, wl.d, 5)
    out = sfn.sparse_ffn_backward(x.to(DEV), dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                  dev["Wd"], dy.to(DEV), bank=bank, k=k, temperature=temp,
                                  want=want)
    torch.cuda.synchronize()
    return x, dy, out


ROW_FLOOR = 1e-4


def _check_rows(name, g, ref):
    """Per-row error of a gradient matrix (see the module doc)."""
    assert np.isfinite(g).all(), name
    scale = np.abs(ref).max(axis=1)
    err = np.abs(g - ref).max(axis=1)
    zero = scale == 0
    assert (err[zero] == 0).all(), f"{name}: rows the oracle gives as zero are not zero"
    rel = err[~zero] / np.maximum(scale[~zero], ROW_FLOOR * scale.max())
    worst = int(np.argmax(rel)) if len(rel) else 0
    assert not len(rel) or rel.max() <= GRAD_TOL, (
        f"{name}: row {np.flatnonzero(~zero)[worst]} relative error {rel.max():.3g}")


def _check(wl, host, dev, T, bank, k, temp):
    x, dy, out = _run(wl, host, dev, T, bank, k, temp)
    gm = parity.to_u64(out["mask"])
    parity.check_mask(gm, oracle.predict(x, host["A"], host["B"]), bank, k)
    ref = oracle.backward(x, host["A"], host["B"], host["Wg"], host["Wu"], host["Wd"], dy,
                          bank, k, temp, mask=gm)
    for n in NAMES:
        _check_rows(n, out[n].cpu().numpy().astype(np.float64), ref[n])
    errs = np.zeros(1, np.int32)
    _capi.check(_capi.lib().sfn_device_errors(errs.ctypes.data, 1), "sfn_device_errors")
    assert errs[0] == 0


@pytest.mark.parametrize("T,bank,k,temp", [
    (64, 64, 16, 1.0),   # logits on the tensor cores (the forward's choice for T >= 6)
    (5, 64, 16, 0.5),    # logits on the CUDA-core kernels
    (33, 16, 4, 0.3),    # bank 16: CUDA-core logits
    (20, 64, 64, 1.0),   # k = bank: no threshold, no surrogate term
    (130, 64, 16, 0.5),  # two token tiles; the K = T contractions end mid-block
    (300, 64, 16, 1.0),  # three token tiles, ragged in M and in K
])
def test_backward_small(T, bank, k, temp):
    wl = SMALL.with_(bank=bank, k=k)
    host = make_layer(wl)
    _check(wl, host, {n: v.to(DEV) for n, v in host.items()}, T, bank, k, temp)


@pytest.mark.parametrize("T", [2, 9])
def test_backward_full_width(T, full_layer):
    wl, host, dev = full_layer
    _check(wl, host, dev, T, 64, 16, 1.0)


def test_backward_partial_outputs_and_determinism():
    wl = SMALL
    host = make_layer(wl)
    dev = {n: v.to(DEV) for n, v in host.items()}
    _, _, full1 = _run(wl, host, dev, 40, 64, 16, 0.7)
    _, _, full2 = _run(wl, host, dev, 40, 64, 16, 0.7)
    _, _, part = _run(wl, host, dev, 40, 64, 16, 0.7, want=("dWg", "dB"))
    for n in NAMES:
        assert torch.equal(full1[n], full2[n]), f"{n} not bit-identical across runs"
    assert torch.equal(part["dWg"], full1["dWg"]) and torch.equal(part["dB"], full1["dB"])
    assert torch.equal(part["mask"], full1["mask"])


def test_backward_zero_tokens():
    wl = SMALL
    host = {n: v.to(DEV) for n, v in make_layer(wl).items()}
    x = torch.empty((0, wl.d), dtype=torch.bfloat16, device=DEV)
    out = sfn.sparse_ffn_backward(x, host["A"], host["B"], host["Wg"], host["Wu"], host["Wd"],
                                  x, bank=64, k=16, temperature=1.0)
    assert out["dWg"].shape == (wl.d_i, wl.d)
