"""Tensor-parallel BitLinear on CPU: two gloo ranks.

binary_weight_transformer_b200.tp partitions a layer by output rows
(column-parallel) or by input features (row-parallel, with the token
statistics and the int32 partial sums all-reduced).  Here every rank runs the
per-rank compute on the CPU -- the oracle for codes, integer dot and rescale,
and a few lines of numpy for the slice statistics -- so that the partitioning,
the slicing of the packed artifact and the order of the collectives are
checked against the unsplit oracle without a GPU.  The GPU kernels behind the
same functions are checked by tests/test_gpu_tp.py.
"""
import os
import socket
from types import SimpleNamespace

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def cpu_ops():
    """Per-rank compute on the CPU (test infrastructure)."""
    import torch
    import oracle

    def rotated(x, g, hb):
        u = x.numpy().astype(np.float32)
        if g is not None:
            u = (u * g.numpy()).astype(np.float32)
        if hb:
            M, K = u.shape
            u = oracle.fwht32(u.reshape(M, K // hb, hb)).reshape(M, K)
        return u

    def row_stats(x, g, hb, with_ss=False):
        u = rotated(x, g, hb)
        row_max = torch.from_numpy(np.abs(u).max(axis=1).astype(np.float32))
        row_ss = torch.from_numpy((x.numpy().astype(np.float64) ** 2).sum(axis=1)) if with_ss else None
        return row_max, row_ss

    def scales(row_max, row_ss, K_total, norm, eps_norm, hb):
        s = row_max.numpy().astype(np.float64)
        if hb:
            s = s / np.sqrt(float(hb))
        if norm:
            s = s / np.sqrt(row_ss.numpy() / K_total + np.float64(np.float32(eps_norm)))
        out = (s / 127.0).astype(np.float32)
        out[row_max.numpy() == 0] = 0
        return torch.from_numpy(out)

    def codes_given_max(x, row_max, g, hb):
        u = rotated(x, g, hb)
        gm = row_max.numpy()[:, None]
        with np.errstate(divide="ignore", invalid="ignore"):
            z = np.rint((u * np.float32(127)).astype(np.float32) / gm).astype(np.float32)
        z = np.where(gm == 0, 0, np.clip(z, -128, 127))
        return torch.from_numpy(z.astype(np.int8))

    def linear_i32(q, s_x, packed, s_w, fmt, N, K):
        codes, st = oracle.unpack(np.ascontiguousarray(packed.numpy()), K, fmt)
        assert st == oracle.OK
        return torch.from_numpy(oracle.int_dot(q.numpy(), codes, fmt).astype(np.int32))

    def rescale(acc, s_x, s_w, fmt, out_dtype):
        return torch.from_numpy(oracle.rescale(acc.numpy().astype(np.int64), s_w.numpy(), s_x.numpy(), "f32"))

    def bitlinear(x, packed, s_w, fmt, N, out_dtype, g, norm, eps_norm, hb):
        q, s_x = oracle.act_prologue(x.numpy(), None if g is None else g.numpy(), bool(norm), eps_norm, hb)
        K = x.shape[1]
        codes, st = oracle.unpack(np.ascontiguousarray(packed.numpy()), K, fmt)
        assert st == oracle.OK
        acc = oracle.int_dot(q, codes, fmt)
        return torch.from_numpy(oracle.rescale(acc, s_w.numpy(), s_x, "f32"))

    return SimpleNamespace(row_stats=row_stats, scales=scales, codes_given_max=codes_given_max,
                           linear_i32=linear_i32, rescale=rescale, bitlinear=bitlinear)


CASES = [(fmt, norm, hb, gain) for fmt in (0, 1, 2) for norm, hb, gain in
         ((0, 0, False), (1, 0, True), (0, 128, False), (1, 256, True))]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import oracle
    from binary_weight_transformer_b200 import tp
    from binary_weight_transformer_b200 import workloads as wls

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ops = cpu_ops()
    results = []
    try:
        M, K, N = 9, 1024, 40
        for fmt, norm, hb, use_g in CASES:
            w = wls.normal_weights(7000 + fmt, N, K)
            x = wls.normal_activations(7001 + fmt, M, K, 0.01, 8.0)
            g = wls.gain_vector(7002, K) if use_g else None
            codes, s_w = oracle.quantize(w, fmt, 1e-5)
            packed = oracle.pack(codes, fmt)
            # the unsplit layer
            q, s_x = oracle.act_prologue(x, g, bool(norm), 1e-5, hb)
            y_ref = oracle.rescale(oracle.int_dot(q, codes, fmt), s_w, s_x, "f32")

            # row-parallel: this rank's features
            k0, k1 = tp.split(K, world, rank, tp.feature_granule(hb))
            xt = torch.from_numpy(x[:, k0:k1].copy())
            gt = None if g is None else torch.from_numpy(g[k0:k1].copy())
            cols = tp.packed_feature_slice(torch.from_numpy(packed), fmt, k0, k1)
            y_row = tp.row_parallel_bitlinear(xt, cols, torch.from_numpy(s_w), fmt, N, K, 0, gt, norm, 1e-5, hb,
                                              ops=ops).numpy()

            # column-parallel: this rank's output rows
            n0, n1 = tp.split(N, world, rank)
            rows = torch.from_numpy(packed[n0:n1].copy())
            y_cols = tp.column_parallel_bitlinear(torch.from_numpy(x), rows,
                                                  tp.row_scales_slice(torch.from_numpy(s_w), fmt, n0, n1), fmt,
                                                  n1 - n0, 0, None if g is None else torch.from_numpy(g), norm,
                                                  1e-5, hb, ops=ops)
            y_col = tp.gather_columns(y_cols).numpy()

            def close(a, b):
                if norm:  # the sums of squares are added across ranks in another order
                    return np.max(np.abs(a - b) / np.maximum(np.abs(b), 1e-30)) <= 1e-6
                return np.array_equal(a.view(np.uint32), b.view(np.uint32))
            results.append((fmt, norm, hb, close(y_row, y_ref), close(y_col, y_ref)))
        if rank == 0:
            with open(os.path.join(out_dir, "result.txt"), "w") as f:
                bad = [r for r in results if not (r[3] and r[4])]
                f.write("ok" if not bad else f"mismatch {bad}")
    finally:
        dist.destroy_process_group()


def test_split_covers_and_balances():
    import sys
    sys.path.insert(0, ROOT)
    from binary_weight_transformer_b200 import tp
    for total, granule in ((1024, 128), (2560, 128), (9728, 512), (40, 1)):
        for world in (1, 2, 4):
            if (total // granule) < world:
                continue
            spans = [tp.split(total, world, r, granule) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert all(a % granule == 0 and b % granule == 0 for a, b in spans)
    with pytest.raises(ValueError):
        tp.split(1000, 2, 0, 128)


def test_two_gloo_ranks_row_and_column_parallel(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    assert (tmp_path / "result.txt").read_text() == "ok"
