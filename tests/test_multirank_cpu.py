"""The multi-rank path on CPU: two gloo ranks.

A multi-GPU run shards the token batch across ranks with no exchange of data:
per-token quantisation ("M8.8 - Native Binary and Ternary Transformers"
0x05C) makes every token row independent, so the sharded result must equal
the unsharded one bit for bit.  Each rank runs the oracle on its shard, the
shards are gathered, and rank 0 compares.  The timing reduction bench.py uses
(the slowest rank's time) is checked the same way.
"""
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    import oracle
    from binary_weight_transformer_b200 import workloads as wls

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, K, N = 37, 160, 48
        fmt = oracle.TERNARY2
        w = wls.normal_weights(900, N, K)
        x = wls.normal_activations(901, M, K)
        codes, s_w = oracle.quantize(w, fmt)
        start, stop = bench.shard_range(M, rank, world)
        q, s_x = oracle.act_quant(x[start:stop])
        y, acc = oracle.linear(q, s_x, oracle.pack(codes, fmt), s_w, fmt, K)
        parts = [None] * world
        dist.all_gather_object(parts, (start, stop, y, acc))
        slowest = bench.max_over_ranks(float(rank + 1))
        if rank == 0:
            q_all, sx_all = oracle.act_quant(x)
            y_all, acc_all = oracle.linear(q_all, sx_all, oracle.pack(codes, fmt), s_w, fmt, K)
            ys = np.concatenate([p[2] for p in sorted(parts, key=lambda p: p[0])])
            accs = np.concatenate([p[3] for p in sorted(parts, key=lambda p: p[0])])
            covered = sorted((p[0], p[1]) for p in parts)
            ok = (np.array_equal(accs, acc_all) and np.array_equal(ys.view(np.uint32), y_all.view(np.uint32))
                  and covered[0][0] == 0 and covered[-1][1] == M
                  and all(a[1] == b[0] for a, b in zip(covered, covered[1:]))
                  and slowest == float(world))
            with open(os.path.join(out_dir, "result.txt"), "w") as f:
                f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_shard_range_partitions_rows():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for M in (1, 2, 7, 8192):
        for world in (1, 2, 3, 8):
            spans = [bench.shard_range(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_match_unsharded(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    assert (tmp_path / "result.txt").read_text() == "ok"
