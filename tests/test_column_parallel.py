"""Column-parallel layer: the host logic on CPU (block bounds, and the gather
over a world-size-2 gloo group with a stand-in block computation), and on
one GPU the property that makes the split exact: the blocks of the CUDA
layer's Y, computed shard by shard, are the bits of the full call."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from int8_quantized_row_b200 import column_parallel as cp


@pytest.mark.parametrize("N,world", [(16, 1), (1024, 2), (1040, 3), (49152, 8), (12288, 7), (64, 4)])
def test_column_bounds_cover_disjoint_aligned_balanced(N, world):
    spans = [cp.column_bounds(N, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == N
    for (a0, b0), (a1, b1) in zip(spans, spans[1:]):
        assert b0 == a1
    widths = [b - a for a, b in spans]
    assert all(w % 16 == 0 for w in widths)
    assert max(widths) - min(widths) <= 16


def test_column_bounds_reject_bad_splits():
    for N, world, rank in ((1000, 2, 0), (1024, 0, 0), (1024, 2, 2)):
        with pytest.raises(ValueError):
            cp.column_bounds(N, world, rank)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _block_fn(X, Wq, sW, W16, alpha):
    # stand-in for the CUDA layer, exact on integers: Y = X @ (Wq * sW) (+ W16 on the first row)
    Y = X.double() @ (Wq.double() * sW.double()[None, :])
    if W16 is not None:
        Y = Y + W16.double()[:1, :]
    return Y


def _worker(rank, world, port, N, T, K, wq_only, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(1)
        X = torch.randint(-3, 4, (T, K), generator=g).to(torch.int32)
        Wq = torch.randint(-127, 128, (K, N), generator=g).to(torch.int8)
        sW = torch.randint(1, 5, (N,), generator=g).to(torch.float32)
        W16 = None if wq_only else torch.randint(-8, 9, (K, N), generator=g).to(torch.float32)
        shard = cp.shard_columns(Wq, sW, W16, world, rank)
        Y = cp.int8_mixed_linear_column_parallel(X, *shard, N, 6.0, world=world, rank=rank, local_fn=_block_fn)
        full = _block_fn(X, Wq, sW, W16, 6.0)
        out[rank] = bool(torch.equal(Y, full))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N,wq_only", [(1024, False), (1040, True)])
def test_gather_over_gloo_reassembles_the_full_output(N, wq_only):
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), N, 5, 64, wq_only, out), nprocs=world,
                       start_method="spawn", join=True)
    assert dict(out) == {0: True, 1: True}


@pytest.mark.gpu
@pytest.mark.parametrize("T,world,wq_only", [(16, 2, False), (300, 3, False), (16, 4, True)])
def test_column_blocks_are_bit_identical_to_the_full_layer(orc, T, world, wq_only):
    import int8_quantized_row_b200 as i8
    from gpu_helpers import assert_y_close, device_status_clean, outlier_x, to_dev, to_host
    K, N = 2048, 2048 + 16 * world            # uneven blocks
    rng = np.random.default_rng(T + world)
    Xh = outlier_x(rng, T, K, [3, 700, 2000])
    Wh = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    X, W = to_dev(Xh), to_dev(Wh)
    Wq, sW = i8.int8_quantize_weight_colwise(W)
    full = i8.int8_mixed_linear_wq(X, Wq, sW, 6.0) if wq_only else i8.int8_mixed_linear(X, Wq, sW, W, 6.0)
    blocks = [cp.int8_mixed_linear_column_parallel(X, *cp.shard_columns(Wq, sW, None if wq_only else W, world, r), N,
                                                   6.0, world=world, rank=r, gather=False) for r in range(world)]
    torch.cuda.synchronize()
    Y = to_host(torch.cat(blocks, dim=1))
    assert np.array_equal(Y.view(np.uint16), to_host(full).view(np.uint16))
    # and the reassembled layer is the oracle's, on sampled rows
    Wq_o, sW_o = orc.quantize_weight_colwise(Wh)
    rows = np.unique(np.r_[0:T:7, T - 1]).astype(np.int32)
    Y_o, _, _, cnt = orc.mixed_linear(Xh, Wq_o, sW_o, None if wq_only else Wh, 6.0, rows=rows)
    assert cnt == 3
    assert_y_close(Y[rows], Y_o, f"column-parallel x{world} T={T}")
    assert device_status_clean()
