"""Output-row split of the layer across ranks (sparse_linear_layers_b200.osplit)
on CPU: gloo, world sizes 2 and 3, spawned processes.

Each rank takes its block of output rows (row_block), prepares that block of
latent weights with the CPU oracle and computes its block of y and of the
integer accumulators; gather_rows assembles them over gloo.  The gathered
results must equal the oracle's unsharded layer bit for bit (accumulators,
float64 y, and the block's codes and scales against the rows of the whole
matrix's preparation): the split is exact, not approximate.  The GPU
contraction of each block is sbl_linear, covered by the GPU parity tests.
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

CASES = [  # (O, K, T, n, m)
    (896, 256, 1, 3, 4),
    (896, 256, 5, 2, 4),
    (300, 128, 3, 6, 8),
    (128, 64, 2, 2, 4),   # fewer rows than ranks' blocks: later ranks own none
]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from sparse_linear_layers_b200 import synthetic
        from sparse_linear_layers_b200.osplit import gather_rows, row_block
        results = []
        for O, K, T, n, m in CASES:
            W = synthetic.latent_weights(O, K, seed=1, tag="osplit")
            _, xv = synthetic.activations(T, K, seed=1, tag="osplit-x")
            a, b = row_block(O, world, rank)
            packed_b, scale_b, _, Wt_b = oracle.prepare_weights(W[a:b], n, m) if b > a else (
                np.zeros((0, K // 4), np.uint8), np.zeros(0, np.float32), None, np.zeros((0, K), np.int8))
            y_b, acc_b, _, _ = oracle.linear(xv, Wt_b, scale_b)
            y = gather_rows(torch.from_numpy(np.ascontiguousarray(y_b)), O, world, rank)
            acc = gather_rows(torch.from_numpy(np.ascontiguousarray(acc_b)), O, world, rank)
            packed_full, scale_full, _, Wt_full = oracle.prepare_weights(W, n, m)
            y_ref, acc_ref, _, _ = oracle.linear(xv, Wt_full, scale_full)
            results.append(dict(
                case=(O, K, T, n, m), rows=(a, b),
                prep_ok=bool(np.array_equal(packed_b, packed_full[a:b]) and
                             np.array_equal(scale_b.view(np.uint32), scale_full[a:b].view(np.uint32))),
                acc_ok=bool(np.array_equal(acc.numpy(), acc_ref)),
                y_ok=bool(np.array_equal(y.numpy(), y_ref)),
                shape=tuple(y.shape)))
        q.put((rank, results))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 3])
def test_output_row_split_equals_unsharded_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, results in out:
        for r in results:
            O, K, T, n, m = r["case"]
            assert r["shape"] == (T, O), r
            assert r["prep_ok"] and r["acc_ok"] and r["y_ok"], (rank, r)
    # the blocks tile [0, O) in order
    for i, (O, K, T, n, m) in enumerate(CASES):
        spans = [results[i]["rows"] for _, results in out]
        assert spans[0][0] == 0 and spans[-1][1] == O
        assert all(spans[j][1] == spans[j + 1][0] for j in range(world - 1))


def test_row_blocks():
    from sparse_linear_layers_b200.osplit import block_rows, row_block
    assert [row_block(7168, 8, r) for r in range(8)] == [(896 * r, 896 * (r + 1)) for r in range(8)]
    assert [row_block(300, 2, r) for r in range(2)] == [(0, 256), (256, 300)]
    assert block_rows(128, 8) == 128 and row_block(128, 8, 3) == (128, 128)
    with pytest.raises(ValueError):
        row_block(10, 2, 2)
