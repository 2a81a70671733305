"""Multi-process check of the batch partition (world size 2, gloo, CPU).

Loki decode is independent per (batch, KV head) row, so ranks own contiguous
batch ranges and exchange nothing on the data path.  Each rank computes its
shard with the oracle; the shards gathered on rank 0 must equal the unsharded
result exactly."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_path):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    from sparse_decode_attention_loki_b200.sharding import shard_batches
    from workloads import Workload
    from workloads import generators as gen
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = Workload(name="shard", dtype="bf16", batch=5, n_q_heads=4, n_kv_heads=2, head_dim=64, seq_len=96,
                 d_f=0.25, k_f=0.25, generator="powerlaw", n_calib=512)
    P = np.stack([oracle.pca_basis(gen.calibration_keys(w, g))[0] for g in range(2)]).astype(np.float32)
    b0, b1 = shard_batches(w.batch, world, rank)
    inp = gen.decode_inputs(w, batches=range(b0, b1))
    K_hat = oracle.rotate_keys(inp["keys64"], P.astype(np.float64), "bf16")
    r = oracle.loki_decode(inp["q64"], K_hat, inp["values64"], P.astype(np.float64), w.seq_len, w.d, w.k)
    # pad to the largest shard so that all_gather sees equal shapes
    maxb = shard_batches(w.batch, world, 0)[1] - shard_batches(w.batch, world, 0)[0]
    out = torch.zeros((maxb, 4, 64), dtype=torch.float64)
    idx = torch.full((maxb, 2, w.k), -1, dtype=torch.int64)
    out[: b1 - b0] = torch.from_numpy(r["out"])
    idx[: b1 - b0] = torch.from_numpy(r["idx"])
    outs = [torch.zeros_like(out) for _ in range(world)]
    idxs = [torch.zeros_like(idx) for _ in range(world)]
    dist.all_gather(outs, out)
    dist.all_gather(idxs, idx)
    if rank == 0:
        parts_o, parts_i = [], []
        for rr in range(world):
            a, b = shard_batches(w.batch, world, rr)
            parts_o.append(outs[rr][: b - a])
            parts_i.append(idxs[rr][: b - a])
        full = gen.decode_inputs(w)
        Kf = oracle.rotate_keys(full["keys64"], P.astype(np.float64), "bf16")
        rf = oracle.loki_decode(full["q64"], Kf, full["values64"], P.astype(np.float64), w.seq_len, w.d, w.k)
        ok = (np.array_equal(torch.cat(parts_o).numpy(), rf["out"])
              and np.array_equal(torch.cat(parts_i).numpy(), rf["idx"]))
        with open(result_path, "w") as f:
            f.write("ok" if ok else "mismatch")
    dist.barrier()
    dist.destroy_process_group()


def test_shard_ranges_cover_batch():
    from sparse_decode_attention_loki_b200.sharding import shard_batches
    for B in range(0, 20):
        for world in range(1, 9):
            ranges = [shard_batches(B, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == B
            for (a, b), (c, d) in zip(ranges, ranges[1:]):
                assert b == c
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_batches(4, 2, 2)


def test_two_rank_sharded_decode_equals_unsharded(tmp_path):
    path = str(tmp_path / "result.txt")
    mp.start_processes(_worker, args=(2, _free_port(), path), nprocs=2, join=True, start_method="spawn")
    assert open(path).read() == "ok"
