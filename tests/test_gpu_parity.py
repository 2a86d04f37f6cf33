"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Inputs come from the seeded generator (predictor_gated_channel_b200.inputs);
expected values come only from the oracle.  Rules in tests/parity.py.
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


@pytest.fixture(scope="module", autouse=True)
def _built():
    sfn_build.build()
    _capi.lib()


def _to_dev(layer):
    return {k: v.to(DEV) for k, v in layer.items()}


@pytest.fixture(scope="module")
def full_layer():
    """The full-width layer (d 4096, d_i 14336, r 448), bf16, seed 0."""
    wl = WORKLOADS["decode"]
    host = make_layer(wl)
    return wl, host, _to_dev(host)


def _run_forward(dev_layer, x_dev, bank, k):
    y, mask = sfn.sparse_ffn_forward(x_dev, dev_layer["A"], dev_layer["B"], dev_layer["Wg"],
                                     dev_layer["Wu"], dev_layer["Wd"], bank=bank, k=k)
    torch.cuda.synchronize()
    return y, mask


def _check_forward(host, x_host, y, mask, bank, k, dtype, rows=None):
    """Oracle on the (sampled) tokens; check mask rule and y error."""
    if rows is None:
        rows = np.arange(x_host.shape[0])
    xs = x_host[torch.as_tensor(rows)]
    logits = oracle.predict(xs, host["A"], host["B"])
    gm = parity.to_u64(mask)[rows]
    n_diff = parity.check_mask(gm, logits, bank, k)
    y_ref = oracle.forward_given_mask(xs, logits, gm, host["Wg"], host["Wu"], host["Wd"], bank)
    err = parity.y_error(y.float().cpu().numpy()[rows], y_ref)
    assert err <= parity.Y_TOL[dtype], f"y error {err:.3g} > {parity.Y_TOL[dtype]}"
    return n_diff, err


# ------------------------------------------------------------------ bank top-k

@pytest.mark.parametrize("bank,k", [(64, 16), (64, 1), (64, 63), (64, 64), (32, 5), (8, 3),
                                    (1, 1), (48, 17)])
def test_bank_topk_bit_exact_random(bank, k):
    rng = np.random.default_rng(bank * 100 + k)
    T, nb = 37, 29
    p = rng.standard_normal((T, nb * bank)).astype(np.float32)
    got = parity.to_u64(sfn.bank_topk(torch.from_numpy(p).to(DEV), bank, k))
    torch.cuda.synchronize()
    assert np.array_equal(got, oracle.bank_topk(p, bank, k))


def test_bank_topk_bit_exact_adversarial():
    rng = np.random.default_rng(7)
    T, bank, k = 64, 64, 16
    p = np.round(rng.standard_normal((T, 224 * bank)) * 2).astype(np.float32) / 2  # many ties
    p[::3, ::5] = -0.0
    p[1::3, ::7] = 0.0
    p[2, :64] = np.nan
    p[3, 5:40] = np.nan
    p[4, :64] = np.inf
    p[5, ::2] = -np.inf
    p[6, :64] = 1.0                        # one value across the bank
    p[7, :64] = np.float32(1e-45)          # denormals
    p[8, 10:20] = np.finfo(np.float32).max
    got = parity.to_u64(sfn.bank_topk(torch.from_numpy(p).to(DEV), bank, k))
    torch.cuda.synchronize()
    assert np.array_equal(got, oracle.bank_topk(p, bank, k))


def test_bank_topk_oracle_logits_full_width(full_layer):
    """Fed the oracle's own logits (rounded to fp32), the GPU mask is
    bit-identical to the oracle's, at the full layer width."""
    wl, host, _ = full_layer
    x = make_tokens(WORKLOADS["prefill"], T=96)
    logits = oracle.predict(x, host["A"], host["B"]).astype(np.float32)
    got = parity.to_u64(sfn.bank_topk(torch.from_numpy(logits).to(DEV), 64, 16))
    torch.cuda.synchronize()
    assert np.array_equal(got, oracle.bank_topk(logits, 64, 16))


# ------------------------------------------------------------------ predictor

@pytest.mark.parametrize("name,T", [("tiny", 8), ("decode", 1), ("decode", 5), ("decode", 64)])
def test_predict_logits(name, T, full_layer):
    wl = WORKLOADS[name]
    host = full_layer[1] if name != "tiny" else make_layer(wl)
    x = make_tokens(wl, T=T)
    got = sfn.predict(x.to(DEV), host["A"].to(DEV), host["B"].to(DEV))
    torch.cuda.synchronize()
    ref = oracle.predict(x, host["A"], host["B"])
    err = np.abs(got.cpu().numpy().astype(np.float64) - ref).max()
    assert err <= 1e-5 * np.abs(ref).max() + 1e-6, err


# ------------------------------------------------------------------ forward

def test_forward_tiny_f32():
    wl = WORKLOADS["tiny"]
    host = make_layer(wl)
    x = make_tokens(wl)
    y, mask = _run_forward(_to_dev(host), x.to(DEV), wl.bank, wl.k)
    assert y.dtype == torch.float32
    n_diff, err = _check_forward(host, x, y, mask, wl.bank, wl.k, "f32")
    assert n_diff == 0


@pytest.mark.parametrize("T", [1, 3, 5, 6, 17, 64])
def test_forward_full_width_bf16(T, full_layer):
    wl, host, dev = full_layer
    x = make_tokens(wl, T=T, seed=T)
    y, mask = _run_forward(dev, x.to(DEV), wl.bank, wl.k)
    assert y.dtype == torch.bfloat16
    _check_forward(host, x, y, mask, wl.bank, wl.k, "bf16")


@pytest.mark.parametrize("bank,k", [(64, 1), (64, 63), (64, 64), (32, 8), (16, 16), (8, 3)])
def test_forward_bank_k_variants_f32(bank, k):
    wl = WORKLOADS["tiny"].with_(bank=bank, k=k)
    host = make_layer(wl, seed=5)
    x = make_tokens(wl, T=11, seed=5)
    y, mask = _run_forward(_to_dev(host), x.to(DEV), bank, k)
    _check_forward(host, x, y, mask, bank, k, "f32")


def test_forward_dense_k64_equals_predictor_gated_dense(full_layer):
    """k = bank keeps every channel (the recipe's predictor-gated dense FFN
    stage): every mask word is all ones and y matches the oracle."""
    wl, host, dev = full_layer
    x = make_tokens(wl, T=2, seed=11)
    y, mask = _run_forward(dev, x.to(DEV), 64, 64)
    assert (parity.to_u64(mask) == np.uint64(2**64 - 1)).all()
    _check_forward(host, x, y, mask, 64, 64, "bf16")


def _prefill_rows(T, tile=128):
    """Rows the oracle checks at a full prefill size.  4096 tokens: every
    token.  More: one whole 128-token tile in the middle of the grid, the
    last tile, and one row of every other tile (a different row in each, so
    every row position inside a tile is covered somewhere)."""
    if T <= 4096:
        return np.arange(T)
    n_tiles = (T + tile - 1) // tile
    mid = n_tiles // 2
    rows = set(range(mid * tile, min(T, (mid + 1) * tile)))
    rows |= set(range((n_tiles - 1) * tile, T))
    for i in range(n_tiles):
        rows.add(min(T - 1, i * tile + (i * 37) % tile))
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", ["prefill", "long_prefill"])
def test_forward_prefill(name, full_layer):
    """Full prefill sizes in one call (the launch configuration the bench
    times).  At 4096 tokens the oracle checks every token; at 32768 it checks
    a whole mid-grid tile, the last tile and one row of every other tile."""
    wl = WORKLOADS[name]
    _, host, dev = full_layer
    x = make_tokens(wl)
    y, mask = _run_forward(dev, x.to(DEV), wl.bank, wl.k)
    rows = _prefill_rows(wl.T)
    _check_forward(host, x, y, mask, wl.bank, wl.k, "bf16", rows=rows)
    assert parity.popcount_ok(parity.to_u64(mask), wl.bank, wl.k)


# ------------------------------------------------------------------ contract

def test_workspace_variant_bit_identical_and_deterministic(full_layer):
    wl, host, dev = full_layer
    x = make_tokens(wl, T=9, seed=3).to(DEV)
    y1, m1 = _run_forward(dev, x, 64, 16)
    y2, m2 = _run_forward(dev, x, 64, 16)
    nbytes = sfn.workspace_bytes(9, wl.d, wl.d_i, wl.r, 64, 16, torch.bfloat16)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    y3, m3 = sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"], dev["Wd"],
                                    workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(m1, m2)
    assert torch.equal(y1, y3) and torch.equal(m1, m3)


@pytest.mark.parametrize("T", [64, 300, 4096])
def test_tensor_path_bit_identical_reruns(T, full_layer):
    """Every sum on the tensor path has a fixed order (split-K partials
    included), so repeated calls give the same bits; a race between the
    pipelines' stages would show up here.  Back-to-back calls on one stream,
    so each one's kernels overlap the previous one's tail."""
    wl, host, dev = full_layer
    x = make_tokens(WORKLOADS["prefill"], T=T, seed=21).to(DEV)
    outs = [sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"], dev["Wd"],
                                   path="tensor") for _ in range(4)]
    torch.cuda.synchronize()
    for y, m in outs[1:]:
        assert torch.equal(y, outs[0][0]) and torch.equal(m, outs[0][1])


def test_concurrent_streams_match_serial(full_layer):
    """Calls on two streams at once (each with its own stream-ordered
    scratch) give the same bits as the same calls one after the other: the
    library keeps no per-call state outside the caller's buffers."""
    wl, host, dev = full_layer
    args = (dev["A"], dev["B"], dev["Wg"], dev["Wu"], dev["Wd"])
    xs = [make_tokens(WORKLOADS["prefill"], T=T, seed=30 + T).to(DEV) for T in (1, 64, 300)]
    serial = [sfn.sparse_ffn_forward(x, *args) for x in xs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in xs]
    conc = []
    for x, s in zip(xs, streams):
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            conc.append(sfn.sparse_ffn_forward(x, *args))
    torch.cuda.synchronize()
    for (y1, m1), (y2, m2) in zip(serial, conc):
        assert torch.equal(y1, y2) and torch.equal(m1, m2)


def test_outputs_do_not_spill(full_layer):
    """Canary words around y and mask stay untouched; mask may be omitted."""
    wl, host, dev = full_layer
    T = 5
    x = make_tokens(wl, T=T, seed=9).to(DEV)
    pad = 64
    ybuf = torch.full((T * wl.d + 2 * pad,), float("nan"), dtype=torch.bfloat16, device=DEV)
    mbuf = torch.full((T * wl.n_banks + 2 * 8,), -12345, dtype=torch.int64, device=DEV)
    y = ybuf[pad:pad + T * wl.d].view(T, wl.d)
    m = mbuf[8:8 + T * wl.n_banks].view(T, wl.n_banks)
    sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"], dev["Wd"], y=y, mask=m)
    y_nomask, none = sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                            dev["Wd"], want_mask=False)
    torch.cuda.synchronize()
    assert none is None
    assert torch.isnan(ybuf[:pad].float()).all() and torch.isnan(ybuf[-pad:].float()).all()
    assert (mbuf[:8] == -12345).all() and (mbuf[-8:] == -12345).all()
    assert torch.equal(y, y_nomask)


def test_launch_counter_counts_kernels(full_layer):
    """Few tokens: h, logits + top-k, gate/up/down, the sum of the partial
    rows; many: the tensor path (h, its split-K sum, logits + top-k,
    gate/up, down, its split-K sum at 64 tokens -- with one token tile the
    logits and gate/up are one kernel)."""
    wl, host, dev = full_layer
    for T, n in ((1, 4), (2, 4), (64, 5), (300, 6)):
        x = make_tokens(wl, T=T).to(DEV)
        c0 = sfn.kernel_launch_count()
        _run_forward(dev, x, 64, 16)
        assert sfn.kernel_launch_count() - c0 == n, T


def test_zero_tokens(full_layer):
    wl, host, dev = full_layer
    x = torch.empty((0, wl.d), dtype=torch.bfloat16, device=DEV)
    y, mask = _run_forward(dev, x, 64, 16)
    assert y.shape == (0, wl.d) and mask.shape == (0, wl.n_banks)


# ------------------------------------------------------------------ tensor path

@pytest.mark.parametrize("T", [1, 5, 6, 16, 64, 100, 127, 128, 129, 130, 256, 257, 300])
def test_tensor_path_full_width(T, full_layer):
    """The tcgen05 path (forced) against the oracle, every token checked: one
    token tile (T <= 128) and several, with full and ragged last tiles on
    both sides of the tile boundaries."""
    wl, host, dev = full_layer
    x = make_tokens(WORKLOADS["prefill"], T=T, seed=100 + T)
    y, mask = sfn.sparse_ffn_forward(x.to(DEV), dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                     dev["Wd"], path="tensor")
    torch.cuda.synchronize()
    _check_forward(host, x, y, mask, 64, 16, "bf16")


@pytest.mark.parametrize("T", [100, 160])
@pytest.mark.parametrize("k", [1, 16, 63, 64])
def test_tensor_path_k_variants(T, k, full_layer):
    """k below, at and above 16 and k = bank on the tensor path, with one
    token tile (100 tokens: the fused logits + gate/up kernel) and two."""
    wl, host, dev = full_layer
    x = make_tokens(WORKLOADS["prefill"], T=T, seed=200 + k)
    y, mask = sfn.sparse_ffn_forward(x.to(DEV), dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                     dev["Wd"], k=k, path="tensor")
    torch.cuda.synchronize()
    rows = np.arange(0, T, 7)
    _check_forward(host, x, y, mask, 64, k, "bf16", rows=rows)


@pytest.mark.parametrize("T", [64, 130])
@pytest.mark.parametrize("k", [1, 4, 16, 20, 63])
def test_tensor_topk_exact_ties(T, k):
    """One-hot tokens and small-integer A and B make the tensor-core logits
    exact integers; every bank of B holds 16 rows four times each, so exact
    ties are everywhere.  The mask of the top-k fused into the logits GEMM
    equals the oracle's bit for bit (ties to the lower channel), for k below
    16, at 16 and above 16 (the wider-staging variant), with one token tile
    (64 tokens: the single-tile loops) and several (130)."""
    rng = np.random.default_rng(300 + k)
    d, d_i, r = 256, 1024, 64
    x, A, B, W, p = _tie_layer(rng, d, d_i, r, 64, T)
    _, mask = sfn.sparse_ffn_forward(_bf16_dev(x), _bf16_dev(A), _bf16_dev(B), _bf16_dev(W),
                                     _bf16_dev(W), _bf16_dev(W), bank=64, k=k, path="tensor")
    torch.cuda.synchronize()
    assert np.array_equal(parity.to_u64(mask), oracle.bank_topk(p, 64, k))


def _tie_layer(rng, d, d_i, r, bank, T):
    """One-hot tokens and small-integer A and B, so that the logits are exact
    integers on either kernel path; inside every bank of B, each of bank/4
    rows appears four times, so exact ties sit at every threshold."""
    x = np.zeros((T, d), np.float32)
    x[np.arange(T), rng.integers(0, d, T)] = 1.0
    A = rng.integers(-3, 4, (r, d)).astype(np.float32)
    B = rng.integers(-2, 3, (d_i, r)).astype(np.float32)
    q = bank // 4
    for b in range(d_i // bank):
        blk = B[b * bank:b * bank + q]
        B[b * bank:(b + 1) * bank] = np.tile(blk, (4, 1))[rng.permutation(bank)]
    W = (rng.standard_normal((d_i, d)) * 0.05).astype(np.float32)
    p = (x.astype(np.int64) @ A.T.astype(np.int64)) @ B.T.astype(np.int64)
    assert np.abs(p).max() < 2 ** 24  # exact in float32
    return x, A, B, W, p.astype(np.float32)


def _bf16_dev(a):
    return torch.from_numpy(a).to(torch.bfloat16).to(DEV)


@pytest.mark.parametrize("T,path", [(1, "cuda_core"), (3, "cuda_core"), (5, "cuda_core")])
@pytest.mark.parametrize("bank,k", [(64, 1), (64, 4), (64, 16), (64, 20), (64, 63), (48, 17),
                                    (32, 5)])
def test_cuda_core_topk_exact_ties(T, path, bank, k):
    """The few-token kernels rank each bank inside their logits kernel (a
    third top-k, beside the standalone one and the tensor-core epilogue).  Fed
    exact-integer logits with ties everywhere, the mask equals the oracle's
    bit for bit (ties to the lower channel), for k below, at and above 16,
    and for banks narrower than 64 (whose order-key rows are padded)."""
    rng = np.random.default_rng(1000 * bank + 10 * k + T)
    d, r = 256, 64
    d_i = (1024 // bank) * bank
    x, A, B, W, p = _tie_layer(rng, d, d_i, r, bank, T)
    _, mask = sfn.sparse_ffn_forward(_bf16_dev(x), _bf16_dev(A), _bf16_dev(B), _bf16_dev(W),
                                     _bf16_dev(W), _bf16_dev(W), bank=bank, k=k, path=path)
    torch.cuda.synchronize()
    assert np.array_equal(parity.to_u64(mask), oracle.bank_topk(p, bank, k))


@pytest.mark.parametrize("T,k", [(1, 16), (1, 1), (1, 63), (1, 64), (2, 16), (4, 16), (5, 16)])
def test_few_token_path_k_variants(T, k, full_layer):
    """The few-token kernels on the full-width layer against the oracle, for
    k below, at and above 16, k = bank, and 1 to 5 tokens."""
    wl, host, dev = full_layer
    x = make_tokens(wl, T=T, seed=500 + 10 * T + k)
    y, mask = sfn.sparse_ffn_forward(x.to(DEV), dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                     dev["Wd"], k=k, path="cuda_core")
    torch.cuda.synchronize()
    _check_forward(host, x, y, mask, 64, k, "bf16")


def test_decode_many_calls_bit_identical(full_layer):
    """Sixty one-token calls in a row on one stream (each call's first kernel
    starts during the previous call's last one) reproduce the first results
    bit for bit; a one-token bank shard (float32 partial y) sums to the
    layer."""
    wl, host, dev = full_layer
    xs = [make_tokens(wl, T=1, seed=600 + i).to(DEV) for i in range(3)]
    first = [_run_forward(dev, x, 64, 16) for x in xs]
    c0 = sfn.kernel_launch_count()
    outs = [sfn.sparse_ffn_forward(xs[i % 3], dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                   dev["Wd"]) for i in range(60)]
    torch.cuda.synchronize()
    assert sfn.kernel_launch_count() - c0 == 4 * 60  # h, logits + top-k, gate/up/down, sum
    for i, (y, m) in enumerate(outs):
        assert torch.equal(y, first[i % 3][0]) and torch.equal(m, first[i % 3][1]), i
    total = torch.zeros((1, wl.d), dtype=torch.float32, device=DEV)
    for rank in range(2):
        b0, b1 = sfn.bank_shard(wl.n_banks, rank, 2)
        rows = slice(b0 * wl.bank, b1 * wl.bank)
        yp, _ = sfn.sparse_ffn_forward_partial(xs[0], dev["A"], dev["B"][rows],
                                               dev["Wg"][rows], dev["Wu"][rows],
                                               dev["Wd"][rows])
        total += yp
    torch.cuda.synchronize()
    ref = first[0][0].float()
    assert (total - ref).abs().max().item() <= 2e-2 * ref.abs().max().item()


def test_one_tile_kernel_several_units_per_cta():
    """With more 128-channel units than SMs (here 304), each CTA of the fused
    one-tile logits + gate/up kernel takes several units in turn, reusing its
    single logits and gate/up accumulators; every token checked."""
    import math
    from predictor_gated_channel_b200.inputs import Workload
    wl = Workload("wide", 64, 256, 38912, 64, 64, 16, "bf16", "rmsnorm", 1.0 / math.sqrt(9728))
    host = make_layer(wl, seed=9)
    dev = {n: v.to(DEV) for n, v in host.items()}
    x = make_tokens(wl, seed=9)
    y, mask = sfn.sparse_ffn_forward(x.to(DEV), dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                     dev["Wd"], path="tensor")
    torch.cuda.synchronize()
    _check_forward(host, x, y, mask, wl.bank, wl.k, "bf16")


@pytest.mark.parametrize("T", [64, 200])
def test_tensor_path_uneven_k_splits(T):
    """Split-K counts that do not divide the K-block count: d = 1280 gives the
    h GEMM 20 K blocks over 8 splits at one token tile, d_i = 2816 the down
    GEMM 44 over 8.  Each split must get a non-empty range; every token is
    checked."""
    wl = Workload("uneven", T, 1280, 2816, 64, 64, 16, "bf16", "rmsnorm",
                  1.0 / math.sqrt(704))
    host = make_layer(wl, seed=13)
    dev = {n: v.to(DEV) for n, v in host.items()}
    x = make_tokens(wl, seed=13)
    y, mask = sfn.sparse_ffn_forward(x.to(DEV), dev["A"], dev["B"], dev["Wg"], dev["Wu"],
                                     dev["Wd"], path="tensor")
    torch.cuda.synchronize()
    _check_forward(host, x, y, mask, wl.bank, wl.k, "bf16")


def test_paths_agree(full_layer):
    """CUDA-core and tensor paths on the same 96 tokens: masks differ only at
    allowed near-ties, outputs within the bf16 tolerance of each other."""
    wl, host, dev = full_layer
    x = make_tokens(WORKLOADS["prefill"], T=96, seed=7).to(DEV)
    y1, m1 = sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"], dev["Wd"],
                                    path="cuda_core")
    y2, m2 = sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"], dev["Wd"],
                                    path="tensor")
    torch.cuda.synchronize()
    same = (m1 == m2).float().mean().item()
    assert same > 0.99, same
    rows = torch.nonzero((m1 == m2).all(dim=1)).flatten()
    err = parity.y_error(y2[rows].float().cpu().numpy(), y1[rows].float().cpu().numpy().astype(np.float64))
    assert err <= parity.Y_TOL["bf16"], err


def test_tensor_predict_logits(full_layer):
    """sfn_predict at T >= 1024 runs on the tensor cores (split-h logits)."""
    wl, host, dev = full_layer
    x = make_tokens(WORKLOADS["prefill"], T=1100, seed=5)
    got = sfn.predict(x.to(DEV), dev["A"], dev["B"])
    torch.cuda.synchronize()
    rows = np.arange(0, 1100, 37)
    ref = oracle.predict(x[torch.as_tensor(rows)], host["A"], host["B"])
    err = np.abs(got.cpu().numpy()[rows].astype(np.float64) - ref).max()
    assert err <= 2e-5 * np.abs(ref).max() + 1e-6, err


def test_tensor_path_rejects_unsupported(full_layer):
    wl, host, dev = full_layer
    x = make_tokens(wl, T=4).to(DEV)
    with pytest.raises(sfn.SfnError):
        sfn.sparse_ffn_forward(x, dev["A"], dev["B"], dev["Wg"], dev["Wu"], dev["Wd"],
                               bank=32, k=8, path="tensor")


# ------------------------------------------------------------------ Dense-4x

@pytest.mark.parametrize("T", [1, 64, 300])
def test_dense4x_against_oracle(T, full_layer):
    """The Dense-4x comparison on the tensor cores: the mask may differ from
    the oracle's only at near-ties of the amplitude |silu(g) u|; y matches the
    oracle applied with the GPU's own mask."""
    wl, host, dev = full_layer
    x = make_tokens(wl, T=T, seed=300 + T)
    y, mask = sfn.dense4x_forward(x.to(DEV), dev["Wg"], dev["Wu"], dev["Wd"])
    torch.cuda.synchronize()
    rows = np.arange(T) if T <= 64 else np.arange(0, T, 11)
    xs = x[torch.as_tensor(rows)]
    _, _, act = oracle.dense4x(xs, host["Wg"], host["Wu"], host["Wd"], 64, 16, want_act=True)
    gm = parity.to_u64(mask)[rows]
    parity.check_mask(gm, np.abs(act), 64, 16)
    y_ref, _ = oracle.dense4x(xs, host["Wg"], host["Wu"], host["Wd"], 64, 16, mask=gm)
    err = parity.y_error(y.float().cpu().numpy()[rows], y_ref)
    assert err <= parity.Y_TOL["bf16"], err


@pytest.mark.parametrize("T,world", [(1, 2), (64, 2), (3, 3)])
def test_bank_shards_sum_to_the_layer(T, world, full_layer):
    """Bank-sharded layer on one device: every shard's float32 partial y from
    its own rows, summed, equals the layer (oracle on the concatenated GPU
    masks); the shard masks concatenate to a valid mask of the whole layer."""
    wl, host, dev = full_layer
    x = make_tokens(wl, T=T, seed=11)
    xd = x.to(DEV)
    total = torch.zeros((T, wl.d), dtype=torch.float32, device=DEV)
    masks = []
    for rank in range(world):
        b0, b1 = sfn.bank_shard(wl.n_banks, rank, world)
        rows = slice(b0 * wl.bank, b1 * wl.bank)
        yp, m = sfn.sparse_ffn_forward_partial(xd, dev["A"], dev["B"][rows], dev["Wg"][rows],
                                               dev["Wu"][rows], dev["Wd"][rows], bank=wl.bank,
                                               k=wl.k)
        total += yp
        masks.append(m)
    torch.cuda.synchronize()
    gm = parity.to_u64(torch.cat(masks, dim=1))
    logits = oracle.predict(x, host["A"], host["B"])
    parity.check_mask(gm, logits, wl.bank, wl.k)
    ref = oracle.forward_given_mask(x, logits, gm, host["Wg"], host["Wu"], host["Wd"], wl.bank)
    got = total.cpu().numpy().astype(np.float64)
    err = max(np.abs(got[t] - ref[t]).max() / np.abs(ref[t]).max() for t in range(T))
    assert err <= parity.Y_TOL["bf16"], err
