"""Comparison rules between the CUDA path and the oracle.

Mask rule (the top-k of "1. Architectuur", gist.science summary of arXiv
2606.10722, keeps 16 of every 64 channels; logits computed in different
precisions may legitimately order two channels differently only when they
sit at the selection threshold):
  * every GPU mask word holds exactly k bits (bits >= bank zero);
  * a bank may differ from the oracle's only if every channel in the
    difference lies within  1e-3 * max(|p_(k)|, |p_(k+1)|) + 1e-6 * rms(p_bank)
    of the threshold tau = (p_(k) + p_(k+1)) / 2, with p_(k) the k-th largest
    oracle logit of the bank (no difference is allowed when k == bank).

Output rule: y is compared with the oracle's y computed on the GPU's own mask
(so an allowed flip is not counted as error):
  max_t ||y_t - y*_t||_inf / ||y*_t||_inf <= tol
with tol = 2e-2 for bf16 and 1e-4 for float32.
"""
from __future__ import annotations

import numpy as np

import oracle

Y_TOL = {"bf16": 2e-2, "f32": 1e-4}
FLIP_REL = 1e-3


def to_u64(mask) -> np.ndarray:
    """GPU mask (int64 tensor of uint64 bit patterns) -> numpy uint64."""
    return mask.detach().cpu().numpy().view(np.uint64)


def popcount_ok(mask_u64: np.ndarray, bank: int, k: int) -> bool:
    m = mask_u64.astype(np.uint64)
    if bank < 64 and (m >> np.uint64(bank)).any():
        return False
    bits = np.unpackbits(m.view(np.uint8)).reshape(m.shape + (64,)).sum(-1)
    return bool((bits == k).all())


def check_mask(gpu_mask: np.ndarray, logits: np.ndarray, bank: int, k: int):
    """Return the number of banks that differ (all differences allowed);
    raise AssertionError on a disallowed difference."""
    assert popcount_ok(gpu_mask, bank, k), "a GPU mask word does not hold exactly k bits"
    ref = oracle.bank_topk(logits, bank, k)
    diff = np.argwhere(ref != gpu_mask)
    for t, b in diff:
        assert k < bank, "k == bank admits no difference"
        p = logits[t, b * bank:(b + 1) * bank]
        s = np.sort(p)[::-1]
        pk, pk1 = s[k - 1], s[k]
        tau = 0.5 * (pk + pk1)
        band = FLIP_REL * max(abs(pk), abs(pk1)) + 1e-6 * np.sqrt(np.mean(p * p))
        x = int(ref[t, b]) ^ int(gpu_mask[t, b])
        for i in range(bank):
            if (x >> i) & 1:
                assert abs(p[i] - tau) < band, (
                    f"token {t} bank {b} channel {i}: logit {p[i]!r} is "
                    f"{abs(p[i] - tau):.3g} from the threshold {tau!r} (band {band:.3g})")
    return len(diff)


def y_error(y_gpu: np.ndarray, y_ref: np.ndarray) -> float:
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    num = np.abs(y_gpu - y_ref).max(axis=1)
    den = np.abs(y_ref).max(axis=1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max()) if len(num) else 0.0
