"""Pins of the CPU oracle to facts other than itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
something the pages or the mathematics fix: a hand-worked example, a library
routine on a special case, a closed form, an invariant, or brute force.  The
same functions are run against mutated copies of the oracle (see
``test_oracle_mutants.py``) to show that a plausible mistake fails at least
one of them.

Readings pinned here (gist.science summary of arXiv 2606.10722,
"1. Architectuur" and "3. Hardware Implicaties"): p = B (A x);
a_j = sigma(p_j) g_j u_j for kept channels, exactly 0 otherwise;
y = sum_j a_j W_down[:, j]; per 64-channel bank keep the k largest logits,
equal logits to the lower index.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
from scipy.special import expit

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _layer(rng, d, d_i, r, scale=1.0):
    x = rng.standard_normal((3, d))
    A = rng.standard_normal((r, d)) * scale / math.sqrt(d)
    B = rng.standard_normal((d_i, r)) / math.sqrt(r)
    Wg = rng.standard_normal((d_i, d)) / math.sqrt(d)
    Wu = rng.standard_normal((d_i, d)) / math.sqrt(d)
    Wd = rng.standard_normal((d_i, d)) / math.sqrt(d_i)
    return x, A, B, Wg, Wu, Wd


def _mask_by_stable_sort(p, bank, k):
    """Reference top-k: numpy's stable argsort of -p per bank, first k."""
    T, d_i = p.shape
    out = np.zeros((T, d_i // bank), np.uint64)
    for t in range(T):
        for b in range(d_i // bank):
            seg = p[t, b * bank:(b + 1) * bank]
            order = np.argsort(-seg, kind="stable")  # NaN sorts last, ties keep index order
            w = 0
            for i in order[:k]:
                w |= 1 << int(i)
            out[t, b] = w
    return out


# --------------------------------------------------------------------------- top-k

def pin_topk_golden():
    cases = json.load(open(os.path.join(GOLDEN, "bank_topk_ties.json")))["cases"]
    for c in cases:
        if c["logits"] == "ramp64":
            p = np.arange(64, dtype=np.float64)[None, :]
        else:
            p = np.array([[float(v) for v in c["logits"]]], dtype=np.float64)
        got = oracle.bank_topk(p, c["bank"], c["k"])
        assert [int(v) for v in got[0]] == c["expected"], (c, got)


def pin_topk_popcount():
    rng = _rng(1)
    for bank, k in [(64, 16), (64, 1), (64, 63), (64, 64), (32, 5), (8, 3)]:
        p = rng.standard_normal((5, bank * 7))
        m = oracle.bank_topk(p, bank, k)
        for w in m.ravel():
            w = int(w)
            assert bin(w).count("1") == k
            assert w >> bank == 0


def pin_topk_stable_sort():
    rng = _rng(2)
    for bank, k in [(64, 16), (16, 4), (64, 40)]:
        p = rng.standard_normal((6, bank * 5))
        # force ties and signed zeros into every row
        p = np.round(p * 2) / 2
        p[:, ::7] = -0.0
        p[:, 3::11] = 0.0
        assert (oracle.bank_topk(p, bank, k) == _mask_by_stable_sort(p, bank, k)).all()
        # fp32 logits widen exactly: the same rule on float32 data
        p32 = rng.standard_normal((4, bank * 3)).astype(np.float32)
        assert (oracle.bank_topk(p32, bank, k)
                == _mask_by_stable_sort(p32.astype(np.float64), bank, k)).all()


def pin_topk_brute_force():
    """Enumerate every k-subset; the kept set maximises the sum and, among
    maximal sets, has the lexicographically smallest sorted index tuple.
    Integer logits make the sums exact and create many ties."""
    rng = _rng(3)
    for bank in (4, 6, 8):
        for k in range(1, bank + 1):
            p = rng.integers(-3, 4, size=(4, bank * 2)).astype(np.float64)
            m = oracle.bank_topk(p, bank, k)
            for t in range(p.shape[0]):
                for b in range(2):
                    seg = p[t, b * bank:(b + 1) * bank]
                    best = max(itertools.combinations(range(bank), k),
                               key=lambda s: (sum(seg[list(s)]), [-i for i in s]))
                    want = sum(1 << i for i in best)
                    assert int(m[t, b]) == want, (seg, k, bin(int(m[t, b])), bin(want))


# ----------------------------------------------------------------------- predictor

def pin_predict_matmul():
    """p = B (A x) equals numpy's (B A) x^T: a different association of the
    same contraction, on non-square shapes so a transposed factor fails."""
    rng = _rng(4)
    x, A, B, *_ = _layer(rng, d=48, d_i=80, r=12)
    p = oracle.predict(x, A, B)
    ref = ((B @ A) @ x.T).T
    assert p.shape == (3, 80)
    assert np.allclose(p, ref, rtol=1e-12, atol=1e-12)


def pin_predict_selector():
    """Closed form: A = [I_r | 0] and one-hot B rows with B[j][j mod r] = 1
    give p_j = x[j mod r]."""
    rng = _rng(5)
    d, r, d_i = 24, 6, 32
    x = rng.standard_normal((2, d))
    A = np.zeros((r, d))
    A[:, :r] = np.eye(r)
    B = np.zeros((d_i, r))
    B[np.arange(d_i), np.arange(d_i) % r] = 1.0
    p = oracle.predict(x, A, B)
    assert np.array_equal(p, x[:, np.arange(d_i) % r])


def pin_predict_integer_exact():
    """Small integers: double sums are exact, so p equals numpy's int64 matmul."""
    rng = _rng(6)
    x = rng.integers(-4, 5, size=(3, 40))
    A = rng.integers(-4, 5, size=(9, 40))
    B = rng.integers(-4, 5, size=(24, 9))
    p = oracle.predict(x.astype(np.float64), A.astype(np.float64), B.astype(np.float64))
    assert np.array_equal(p, (B @ (A @ x.T)).T.astype(np.float64))


# ------------------------------------------------------------------------- sigmoid

def pin_sigmoid():
    assert oracle.sigmoid(0.0) == 0.5
    assert abs(oracle.sigmoid(math.log(3.0)) - 0.75) < 1e-15
    assert abs(oracle.sigmoid(-math.log(3.0)) - 0.25) < 1e-15
    for z in np.concatenate([np.linspace(-40, 40, 161), [-700.0, 700.0, 1e-9, -1e-9]]):
        assert abs(oracle.sigmoid(float(z)) - float(expit(z))) <= 1e-15 * max(1.0, expit(z))


# --------------------------------------------------------------------------- forward

def pin_forward_golden():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    arr = {k: np.array(g[k], dtype=np.float64) for k in ("x", "A", "B", "Wg", "Wu", "Wd")}
    y, p, m = oracle.forward(arr["x"], arr["A"], arr["B"], arr["Wg"], arr["Wu"], arr["Wd"],
                             g["bank"], g["k"])
    assert np.array_equal(p, np.array(g["expected_logits"]))
    assert [int(v) for v in m[0]] == g["expected_mask"]
    assert np.allclose(y, np.array(g["expected_y"]), rtol=1e-14, atol=0)


def _dense_gated_ffn(x, p, Wg, Wu, Wd, keep):
    """numpy: y = W_down (keep * sigma(p) * (Wg x) * (Wu x)), W_down = Wd^T."""
    g = x @ Wg.T
    u = x @ Wu.T
    a = keep * expit(p) * g * u
    W_down = Wd.T
    return (W_down @ a.T).T


def pin_forward_k_equals_bank():
    """k = bank keeps every channel: the predictor-gated dense FFN (the
    "Predictor-Gated Dense FFN" stage of the recipe)."""
    rng = _rng(7)
    x, A, B, Wg, Wu, Wd = _layer(rng, d=40, d_i=128, r=10)
    y, p, m = oracle.forward(x, A, B, Wg, Wu, Wd, bank=64, k=64)
    assert all(int(w) == (1 << 64) - 1 for w in m.ravel())
    ref = _dense_gated_ffn(x, (B @ (A @ x.T)).T, Wg, Wu, Wd, 1.0)
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-12)


def pin_forward_masked_dense():
    """Skipping channels equals the dense FFN with the intermediate zeroed
    outside the mask (numpy), and equals the oracle's own dense-then-mask loop."""
    rng = _rng(8)
    for bank, k in [(64, 16), (32, 3), (16, 16), (64, 1)]:
        x, A, B, Wg, Wu, Wd = _layer(rng, d=36, d_i=192, r=8)
        y, p, m = oracle.forward(x, A, B, Wg, Wu, Wd, bank=bank, k=k)
        keep = oracle.mask_to_bool(m, bank).astype(np.float64)
        assert keep.sum(axis=1).tolist() == [k * (192 // bank)] * 3
        ref = _dense_gated_ffn(x, p, Wg, Wu, Wd, keep)
        assert np.allclose(y, ref, rtol=1e-11, atol=1e-12)
        ydm = oracle.dense_then_mask(x, p, m, Wg, Wu, Wd, bank)
        assert np.allclose(y, ydm, rtol=1e-11, atol=1e-12)


def pin_forward_invariants():
    """Permuting channels inside each bank (rows of B, Wg, Wu, Wd alike)
    permutes the mask bits and leaves y unchanged; permuting tokens permutes y;
    y is linear in Wd."""
    rng = _rng(9)
    bank, k = 32, 8
    x, A, B, Wg, Wu, Wd = _layer(rng, d=28, d_i=128, r=7)
    y, p, m = oracle.forward(x, A, B, Wg, Wu, Wd, bank, k)
    perm = np.concatenate([b * bank + rng.permutation(bank) for b in range(128 // bank)])
    y2, p2, m2 = oracle.forward(x, A, B[perm], Wg[perm], Wu[perm], Wd[perm], bank, k)
    assert np.array_equal(oracle.mask_to_bool(m2, bank), oracle.mask_to_bool(m, bank)[:, perm])
    assert np.allclose(y2, y, rtol=1e-12, atol=1e-13)
    tp = np.array([2, 0, 1])
    y3, _, m3 = oracle.forward(x[tp], A, B, Wg, Wu, Wd, bank, k)
    assert np.array_equal(m3, m[tp]) and np.array_equal(y3, y[tp])
    y4, _, _ = oracle.forward(x, A, B, Wg, Wu, 2.0 * Wd, bank, k)
    assert np.array_equal(y4, 2.0 * y)


def pin_forward_bf16_widening():
    """bf16 inputs are widened exactly: feeding bf16 bit patterns equals
    feeding their float64 values."""
    rng = _rng(10)
    x, A, B, Wg, Wu, Wd = _layer(rng, d=32, d_i=64, r=8)

    def to_bf16_bits(a):
        f = a.astype(np.float32).view(np.uint32)
        # round to nearest even on the upper 16 bits
        f = ((f + 0x7FFF + ((f >> 16) & 1)) >> 16).astype(np.uint16)
        return f

    def widen(bits):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    ins = [to_bf16_bits(a) for a in (x, A, B, Wg, Wu, Wd)]
    y1, p1, m1 = oracle.forward(*ins, bank=64, k=16)
    y2, p2, m2 = oracle.forward(*[widen(b) for b in ins], bank=64, k=16)
    assert np.array_equal(p1, p2) and np.array_equal(m1, m2) and np.array_equal(y1, y2)


def pin_dense4x():
    """Dense-4x against numpy: amplitudes |silu(g) u|, the stable-sort top-k
    of them, the masked SwiGLU FFN; k = bank is the dense SwiGLU FFN."""
    rng = _rng(11)
    x, A, B, Wg, Wu, Wd = _layer(rng, d=36, d_i=128, r=4)
    g = x @ Wg.T
    u = x @ Wu.T
    act = g * expit(g) * u
    for bank, k in [(64, 16), (32, 5), (64, 64)]:
        y, m = oracle.dense4x(x, Wg, Wu, Wd, bank, k)
        assert (m == _mask_by_stable_sort(np.abs(act), bank, k)).all()
        keep = oracle.mask_to_bool(m, bank).astype(np.float64)
        assert np.allclose(y, ((Wd.T) @ (keep * act).T).T, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------------ backward
# Reading pinned here ("Executie / Backward Pass" of the same architecture
# section: a sigmoid-like surrogate gradient around the selection threshold):
# tau_b = midpoint of bank b's k-th and (k+1)-th logits, held constant;
# dm_j/dp_j := sigma'((p_j - tau_b) / temp) / temp; the forward mask stays hard.

def _surrogate_grads_torch(x, A, B, Wg, Wu, Wd, dy, bank, k, temp):
    """Gradients by float64 autograd of a straight-through forward whose value
    is the hard-masked layer and whose mask derivative is the surrogate; the
    chain rule is torch's, not the oracle's."""
    import torch
    ts = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (x, A, B, Wg, Wu, Wd)]
    tx, tA, tB, tg, tu, td = ts
    p = (tx @ tA.T) @ tB.T
    T, d_i = p.shape
    pb = p.view(T, d_i // bank, bank)
    order = torch.from_numpy(np.argsort(-pb.detach().numpy(), axis=2, kind="stable"))
    hard = torch.zeros_like(pb).scatter_(2, order[:, :, :k], 1.0)
    if k < bank:
        vals = torch.gather(pb.detach(), 2, order)
        tau = 0.5 * (vals[:, :, k - 1] + vals[:, :, k])
        soft = torch.sigmoid((pb - tau[:, :, None]) / temp)
        m = hard + soft - soft.detach()
    else:
        m = hard
    a = m.reshape(T, d_i) * torch.sigmoid(p) * (tx @ tg.T) * (tx @ tu.T)
    loss = ((a @ td) * torch.tensor(dy, dtype=torch.float64)).sum()
    grads = torch.autograd.grad(loss, ts)
    return dict(zip(["dx", "dA", "dB", "dWg", "dWu", "dWd"], [g.numpy() for g in grads]))


def pin_backward_autograd():
    """Oracle backward = float64 autograd of the straight-through surrogate
    forward (several bank / k / temperature cases, k = bank included)."""
    for seed, (d, d_i, r, bank, k, temp) in enumerate(
            [(12, 32, 6, 8, 3, 0.3), (20, 64, 5, 16, 4, 2.0), (9, 24, 4, 8, 8, 0.5),
             (16, 128, 8, 64, 16, 0.1)]):
        rng = _rng(100 + seed)
        x, A, B, Wg, Wu, Wd = _layer(rng, d, d_i, r, scale=2.0)
        dy = rng.standard_normal(x.shape)
        ref = _surrogate_grads_torch(x, A, B, Wg, Wu, Wd, dy, bank, k, temp)
        got = oracle.backward(x, A, B, Wg, Wu, Wd, dy, bank, k, temp)
        for name, v in ref.items():
            assert np.allclose(got[name], v, rtol=1e-9, atol=1e-12), (name, bank, k)


def pin_backward_finite_differences():
    """With a vanishing temperature the surrogate is zero away from the
    threshold, so the backward must equal central differences of
    L = sum(dy * y) through the oracle's own forward (mask unchanged by the
    perturbation)."""
    rng = _rng(7)
    bank, k, temp, eps = 8, 3, 1e-9, 1e-6
    x, A, B, Wg, Wu, Wd = _layer(rng, 10, 32, 5, scale=2.0)
    dy = rng.standard_normal(x.shape)
    ins = {"dx": x, "dA": A, "dB": B, "dWg": Wg, "dWu": Wu, "dWd": Wd}
    order = ["dx", "dA", "dB", "dWg", "dWu", "dWd"]
    got = oracle.backward(x, A, B, Wg, Wu, Wd, dy, bank, k, temp)
    _, _, m0 = oracle.forward(x, A, B, Wg, Wu, Wd, bank=bank, k=k)

    def loss(args):
        y, _, m = oracle.forward(*args, bank=bank, k=k)
        assert np.array_equal(m, m0), "perturbation flipped the mask"
        return float((y * dy).sum())

    for name in order:
        arr = ins[name]
        for idx in [tuple(rng.integers(0, s) for s in arr.shape) for _ in range(5)]:
            args_p = [ins[n].copy() for n in order]
            args_m = [ins[n].copy() for n in order]
            args_p[order.index(name)][idx] += eps
            args_m[order.index(name)][idx] -= eps
            fd = (loss(args_p) - loss(args_m)) / (2 * eps)
            assert abs(fd - got[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd,
                                                                        got[name][idx])


def pin_backward_closed_form():
    """A one-token layer worked by hand: d = r = 1, two channels in one bank,
    k = 1.  x = 1, A = 1, B = (2, 1) -> h = 1, p = (2, 1): channel 0 kept,
    channel 1 not, tau = 1.5.  g = (0.5, 1.5), u = (2, -1), dy = 1, Wd = (1, 3)
    -> da = (1, 3).  With s_j = sigma(p_j), z_j = (p_j - 1.5) / temp and
    q_j = sigma(z_j)(1 - sigma(z_j)) / temp:
      dp_0 = g0 u0 (s0 (1 - s0) + s0 q0),   dp_1 = 3 g1 u1 s1 q1 (surrogate only),
      dWd = (s0 g0 u0, 0), dWg = (s0 u0, 0), dWu = (s0 g0, 0), dB = (dp_0, dp_1),
      dh = 2 dp_0 + dp_1 = dA,  dx = s0 u0 0.5 + s0 g0 2 + dh."""
    sg = lambda z: 1.0 / (1.0 + math.exp(-z))
    for temp in (0.25, 1.0, 3.0):
        x = np.array([[1.0]]); A = np.array([[1.0]]); B = np.array([[2.0], [1.0]])
        Wg = np.array([[0.5], [1.5]]); Wu = np.array([[2.0], [-1.0]]); Wd = np.array([[1.0], [3.0]])
        dy = np.array([[1.0]])
        g0, g1, u0, u1 = 0.5, 1.5, 2.0, -1.0
        s0, s1 = sg(2.0), sg(1.0)
        q0 = sg(0.5 / temp) * (1 - sg(0.5 / temp)) / temp
        q1 = sg(-0.5 / temp) * (1 - sg(-0.5 / temp)) / temp
        dp0 = g0 * u0 * (s0 * (1 - s0) + s0 * q0)
        dp1 = 3.0 * g1 * u1 * s1 * q1
        dh = 2 * dp0 + dp1
        want = {"dWd": [[s0 * g0 * u0], [0.0]], "dWg": [[s0 * u0], [0.0]],
                "dWu": [[s0 * g0], [0.0]], "dB": [[dp0], [dp1]], "dA": [[dh]],
                "dx": [[s0 * u0 * 0.5 + s0 * g0 * 2.0 + dh]]}
        got = oracle.backward(x, A, B, Wg, Wu, Wd, dy, bank=2, k=1, temp=temp)
        assert int(got["mask"][0, 0]) == 1
        for name, v in want.items():
            assert np.allclose(got[name], np.array(v), rtol=1e-12, atol=1e-15), (name, temp)


ALL_PINS = [
    pin_topk_golden, pin_topk_popcount, pin_topk_stable_sort, pin_topk_brute_force,
    pin_predict_matmul, pin_predict_selector, pin_predict_integer_exact, pin_sigmoid,
    pin_forward_golden, pin_forward_k_equals_bank, pin_forward_masked_dense,
    pin_forward_invariants, pin_forward_bf16_widening, pin_dense4x,
    pin_backward_autograd, pin_backward_finite_differences, pin_backward_closed_form,
]
