"""Seeded synthetic inputs for the sparse FFN layer (weights and token states).

This module draws random numbers and casts them; it holds none of the FFN's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Recipe (the layer shape follows the predictor "R^d -> R^448 -> R^{d_i}" and the
"banks of 64, top-16, d_i = 14336" of "Continual LLM Upcycling: A
Predictor-Gated Bank-Wise Sparsity Training Recipe for Dense-to-Sparse LLMs",
gist.science summary, "1. Architectuur"; d = 4096 is an assumed hidden width):

* ``numpy.random.Generator(PCG64)`` seeded from ``SeedSequence([seed, layer])``,
  spawned into two children: child 0 draws the weights in the order
  A, B, W_gate, W_up, W_down; child 1 draws the activations.  Every layer
  shape shares child 0, so all full-width workloads see the same layer.
* Standard normals are drawn in float32 and scaled by 1/sqrt(fan_in):
  A ~ N(0, 1/d), B ~ N(0, 1/r), W_gate, W_up ~ N(0, 1/d).  W_down uses the
  workload's stated std (1/sqrt(d_s) for the full layer, 1/sqrt(d_i) for the
  tiny one).  W_down is drawn as [d][d_i] and stored transposed as
  Wd[d_i][d], so column j of W_down is the contiguous row j of Wd.
* Token states: "normal" is x ~ N(0, 1); "rmsnorm" is x = RMSNorm(z) with
  z ~ N(0, I_d), eps 1e-6, unit gain; "lowrank" is
  x_t = RMSNorm(z_t + 0.5 U c_t) with U [d][32] ~ N(0, 1/32) drawn once per
  seed and c_t ~ N(0, I_32) per token, which correlates the masks of
  different tokens through a shared rank-32 component.
* bf16 workloads cast with round-to-nearest-even (torch); the tiny workload
  stays float32.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    d_i: int
    r: int
    bank: int
    k: int
    dtype: str          # "bf16" or "f32"
    x_dist: str         # "normal", "rmsnorm" or "lowrank"
    wd_std: float

    @property
    def n_banks(self) -> int:
        return self.d_i // self.bank

    @property
    def d_s(self) -> int:
        return self.n_banks * self.k

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 8, 256, 1024, 64, 64, 16, "f32", "normal", 1.0 / math.sqrt(1024)),
    "decode": Workload("decode", 1, 4096, 14336, 448, 64, 16, "bf16", "rmsnorm",
                       1.0 / math.sqrt(3584)),
    "batched_decode": Workload("batched_decode", 64, 4096, 14336, 448, 64, 16, "bf16",
                               "rmsnorm", 1.0 / math.sqrt(3584)),
    "prefill": Workload("prefill", 4096, 4096, 14336, 448, 64, 16, "bf16", "lowrank",
                        1.0 / math.sqrt(3584)),
    "long_prefill": Workload("long_prefill", 32768, 4096, 14336, 448, 64, 16, "bf16",
                             "lowrank", 1.0 / math.sqrt(3584)),
}


def _children(seed: int, layer: int):
    ss = np.random.SeedSequence([seed, layer])
    w, a = ss.spawn(2)
    return np.random.Generator(np.random.PCG64(w)), np.random.Generator(np.random.PCG64(a))


def _normal(rng, shape, std) -> np.ndarray:
    out = rng.standard_normal(size=shape, dtype=np.float32)
    out *= np.float32(std)
    return out


def _cast(a: np.ndarray, wl: Workload) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(wl.torch_dtype)


def make_layer(wl: Workload, seed: int = 0, layer: int = 0) -> dict:
    """Weights of one layer as CPU tensors: A [r][d], B [d_i][r], Wg/Wu/Wd [d_i][d]."""
    rng, _ = _children(seed, layer)
    A = _cast(_normal(rng, (wl.r, wl.d), 1.0 / math.sqrt(wl.d)), wl)
    B = _cast(_normal(rng, (wl.d_i, wl.r), 1.0 / math.sqrt(wl.r)), wl)
    Wg = _cast(_normal(rng, (wl.d_i, wl.d), 1.0 / math.sqrt(wl.d)), wl)
    Wu = _cast(_normal(rng, (wl.d_i, wl.d), 1.0 / math.sqrt(wl.d)), wl)
    W_down = _normal(rng, (wl.d, wl.d_i), wl.wd_std)
    Wd = _cast(W_down.T, wl)
    return {"A": A, "B": B, "Wg": Wg, "Wu": Wu, "Wd": Wd}


def _rmsnorm(z: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    z = z.astype(np.float64)
    return z / np.sqrt(np.mean(z * z, axis=-1, keepdims=True) + eps)


def make_tokens(wl: Workload, T: int | None = None, seed: int = 0, layer: int = 0) -> torch.Tensor:
    """Token hidden states x [T][d] as a CPU tensor of the workload's dtype."""
    T = wl.T if T is None else T
    _, rng = _children(seed, layer)
    if wl.x_dist == "normal":
        x = _normal(rng, (T, wl.d), 1.0)
    elif wl.x_dist == "rmsnorm":
        x = _rmsnorm(_normal(rng, (T, wl.d), 1.0))
    elif wl.x_dist == "lowrank":
        U = _normal(rng, (wl.d, 32), 1.0 / math.sqrt(32))
        c = _normal(rng, (T, 32), 1.0)
        z = _normal(rng, (T, wl.d), 1.0)
        x = _rmsnorm(z.astype(np.float64) + 0.5 * (c.astype(np.float64) @ U.T.astype(np.float64)))
    else:
        raise ValueError(wl.x_dist)
    return _cast(x.astype(np.float32), wl)


# ---------------------------------------------------------------------------
# Device-side draws for benchmarking: the same distributions as above, drawn
# with torch's CUDA generator (a different random stream, same recipe), so a
# benchmark can hold many distinct layers without host generation time.

def make_layer_device(wl: Workload, device, seed: int = 0, layer: int = 0) -> dict:
    g = torch.Generator(device=device)
    g.manual_seed(1_000_003 * seed + 7919 * layer + 17)

    def draw(shape, std):
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        return t.mul_(std).to(wl.torch_dtype)

    A = draw((wl.r, wl.d), 1.0 / math.sqrt(wl.d))
    B = draw((wl.d_i, wl.r), 1.0 / math.sqrt(wl.r))
    Wg = draw((wl.d_i, wl.d), 1.0 / math.sqrt(wl.d))
    Wu = draw((wl.d_i, wl.d), 1.0 / math.sqrt(wl.d))
    Wd = draw((wl.d_i, wl.d), wl.wd_std)  # rows of W_down^T: i.i.d., so no transpose needed
    return {"A": A, "B": B, "Wg": Wg, "Wu": Wu, "Wd": Wd}


def make_tokens_device(wl: Workload, device, T: int | None = None, seed: int = 0,
                       layer: int = 0) -> torch.Tensor:
    T = wl.T if T is None else T
    g = torch.Generator(device=device)
    g.manual_seed(1_000_033 * seed + 104_729 * layer + 5)

    def rms(z):
        return z * torch.rsqrt(z.square().mean(dim=-1, keepdim=True) + 1e-6)

    z = torch.randn((T, wl.d), generator=g, device=device, dtype=torch.float32)
    if wl.x_dist == "normal":
        x = z
    elif wl.x_dist == "rmsnorm":
        x = rms(z)
    else:
        U = torch.randn((wl.d, 32), generator=g, device=device) / math.sqrt(32)
        c = torch.randn((T, 32), generator=g, device=device)
        x = rms(z + 0.5 * c @ U.T)
    return x.to(wl.torch_dtype)
