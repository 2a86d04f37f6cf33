"""Host logic of bench.py on CPU: the multi-rank parts (gloo, world size 2),
the traffic digests and the roofline accounting.

The path shards by tokens with no collective on the data path; the only
cross-rank step is the max over ranks of the timed region (the slowest rank
sets the job's time) and rank 0 alone printing.  These run as two spawned
processes over gloo on 127.0.0.1.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, world, rank)
        mx = bench.aggregate_max(10.0 + rank * 5.0, world)
        # the reference arm runs on rank 0 only; other ranks return at once
        args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "1"])
        ref = bench.run_reference(args, rank, world) if rank != 0 else "skipped"
        out.put((rank, mx, ref))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank0_only_reference():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    assert res[1][2] is None  # rank 1: no reference work, no output


def test_value_is_whole_job_aggregate():
    """value = tokens of all ranks / slowest rank's time (weak scaling)."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_max(3.0, 1) == 3.0


def test_bank_shard_partitions():
    import sys
    sys.path.insert(0, ROOT)
    import predictor_gated_channel_b200 as sfn
    for n_banks in (1, 7, 224):
        for world in range(1, 9):
            if world > n_banks:
                continue
            ranges = [sfn.bank_shard(n_banks, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n_banks
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def _shard_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    import predictor_gated_channel_b200 as sfn
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(5)
        T, d, d_i, r, bank, k = 3, 16, 64, 6, 16, 4
        x = rng.standard_normal((T, d))
        A = rng.standard_normal((r, d)) / 4
        B = rng.standard_normal((d_i, r)) / 2
        Wg, Wu, Wd = (rng.standard_normal((d_i, d)) / 4 for _ in range(3))
        b0, b1 = sfn.bank_shard(d_i // bank, rank, world)
        rows = slice(b0 * bank, b1 * bank)
        y_part, _, m_part = oracle.forward(x, A, B[rows], Wg[rows], Wu[rows], Wd[rows],
                                           bank=bank, k=k)
        t = torch.from_numpy(y_part)
        dist.all_reduce(t)  # the collective a bank-sharded layer needs
        y_full, _, m_full = oracle.forward(x, A, B, Wg, Wu, Wd, bank=bank, k=k)
        out.put((rank, bool(np.allclose(t.numpy(), y_full, rtol=1e-12, atol=1e-14)),
                 bool((m_part == m_full[:, b0:b1]).all())))
    finally:
        dist.destroy_process_group()


def test_bank_sharded_layer_allreduce_gloo():
    """Two ranks hold disjoint bank ranges of one layer; their partial outputs
    summed by an all-reduce equal the whole layer (oracle arithmetic, gloo)."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok and mask_ok for _, ok, mask_ok in res)


def test_traffic_digest_ignores_comments_only():
    """The DRAM-traffic figures in profiles/ stay valid across comment edits
    and lapse with any change to the code they were measured on (bench.py
    then reports the traffic as null)."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    code = 'int f(int a) { return a + 1; } /* tail */ const char *s = "// kept";\n'
    commented = ("// header\nint f(int a) {  // adds one\n  return a + 1;\n}\n"
                 "/* tail */ const char *s = \"// kept\";\n")
    assert bench._code_only(code) == bench._code_only(commented)
    assert bench._code_only(code) != bench._code_only(code.replace("+ 1", "+ 2"))
    assert "// kept" in bench._code_only(commented)


def test_roofline_accounting_matches_the_layer_sizes():
    """bench.py's algorithmic work per step against the totals the layer's
    sizes fix (d 4096, d_i 14336, r 448, bank 64, k 16, bf16): a decode step
    reads A (3.67 MB), B (12.85 MB) and three 8 KB rows per kept channel
    (3584 of them), 104.6 MB in all, and does 104.6 MFLOP of useful work per
    token (368.8 with every channel kept)."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from predictor_gated_channel_b200.inputs import WORKLOADS
    wl = WORKLOADS["decode"]
    w = bench.stage_work(wl, 1, wl.d_s)
    rows = 3 * 3584 * 8192
    assert rows == 88_080_384
    assert w["ffn"]["bytes"] - rows < 64 * 1024          # x, the kept ids and sigmas
    step = sum(w[s]["bytes"] for s in ("pred_h", "logits_topk", "ffn", "reduce"))
    assert abs(step - 104.6e6) < 0.15e6
    assert w["pred_h"]["bytes"] >= 448 * 4096 * 2 and w["logits_topk"]["bytes"] >= 14336 * 448 * 2
    assert abs(bench.useful_flops_per_token(wl) - 104.6e6) < 0.1e6
    dense = bench.useful_flops_per_token(wl.with_(k=64))
    assert abs(dense - 368.8e6) < 0.1e6
    # 64 tokens whose masks cover every channel read every row once
    w64 = bench.stage_work(wl, 64, wl.d_i)
    weights = 3 * 14336 * 4096 * 2
    gu_down = w64["tc_gateup"]["bytes"] + w64["tc_down"]["bytes"]
    assert weights <= gu_down < weights + 8e6
