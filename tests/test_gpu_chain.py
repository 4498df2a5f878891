"""int8_mixed_linear_chain: the projections of a decoder layer run in order on
one stream with one shared workspace.

The chain must give exactly what the same layers give called one by one
(the kernels are deterministic), each layer must match the oracle, a layer
that reads an earlier layer's Y must see it, and a CUDA graph of the chain
must replay to the same bits.
"""
import numpy as np
import pytest
import torch

import int8_quantized_row_b200 as i8
from gpu_helpers import assert_y_close, device_status_clean, outlier_x, to_dev, to_host

pytestmark = pytest.mark.gpu

# a decoder layer scaled down: qkv (d -> 3d), out (d -> d), fc1 (d -> 4d), fc2 (4d -> d)
D = 1024
SHAPES = [("qkv", D, 3 * D), ("out", D, D), ("fc1", D, 4 * D), ("fc2", 4 * D, D)]


def make_layers(T, seed, wq_only=()):
    rng = np.random.default_rng(seed)
    layers = []
    for name, K, N in SHAPES:
        cols = sorted(rng.choice(K, size=max(1, K // 200), replace=False).tolist())
        X = outlier_x(rng, T, K, cols)
        W = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
        Wd = to_dev(W)
        Wq, sW = i8.int8_quantize_weight_colwise(Wd)
        layers.append(dict(name=name, X=X, W=W, Xd=to_dev(X), Wd=None if name in wq_only else Wd, Wq=Wq, sW=sW))
    return layers


def run_chain(layers, alpha=6.0):
    return i8.int8_mixed_linear_chain([(l["Xd"], l["Wq"], l["sW"], l["Wd"], alpha, None) for l in layers])


def run_one_by_one(layers, alpha=6.0):
    out = []
    for l in layers:
        if l["Wd"] is None:
            out.append(i8.int8_mixed_linear_wq(l["Xd"], l["Wq"], l["sW"], alpha))
        else:
            out.append(i8.int8_mixed_linear(l["Xd"], l["Wq"], l["sW"], l["Wd"], alpha))
    return out


@pytest.mark.parametrize("T,wq_only", [(16, ()), (1, ("out",)), (300, ("fc2",)), (128, ())])
def test_chain_equals_layer_by_layer_and_oracle(orc, T, wq_only):
    layers = make_layers(T, seed=T, wq_only=wq_only)
    Ys = run_chain(layers)
    Yref = run_one_by_one(layers)
    torch.cuda.synchronize()
    rows = np.unique(np.r_[0:T:7, T - 1]).astype(np.int32)
    for l, Y, Yr in zip(layers, Ys, Yref):
        y = to_host(Y)
        assert np.array_equal(y.view(np.uint16), to_host(Yr).view(np.uint16)), l["name"]
        Wq_o, sW_o = orc.quantize_weight_colwise(l["W"])
        Y_o, _, _, cnt = orc.mixed_linear(l["X"], Wq_o, sW_o, None if l["Wd"] is None else l["W"], 6.0, rows=rows)
        assert cnt >= 1
        assert_y_close(y[rows], Y_o, f"{l['name']} T={T}")
    assert device_status_clean()


def test_chain_layer_reads_the_previous_layers_output(orc):
    # layer 2's X is layer 1's Y: the chain runs in stream order
    T, K1, N1, N2 = 16, 1024, 2048, 1024
    rng = np.random.default_rng(3)
    X1 = outlier_x(rng, T, K1, [5, 700])
    W1 = (rng.standard_normal((K1, N1)) * 0.02).astype(np.float16)
    W2 = (rng.standard_normal((N1, N2)) * 0.02).astype(np.float16)
    W1d, W2d = to_dev(W1), to_dev(W2)
    Wq1, sW1 = i8.int8_quantize_weight_colwise(W1d)
    Wq2, sW2 = i8.int8_quantize_weight_colwise(W2d)
    Y1 = torch.empty((T, N1), dtype=torch.float16, device="cuda")
    Y1.fill_(float("nan"))                       # anything read before layer 1 writes it shows
    # Y1 has std about 0.02 * sqrt(K1) = 0.64, so alpha = 2 leaves a few outlier columns in layer 2
    Y1, Y2 = i8.int8_mixed_linear_chain([(to_dev(X1), Wq1, sW1, W1d, 6.0, Y1), (Y1, Wq2, sW2, W2d, 2.0, None)])
    torch.cuda.synchronize()
    y1, y2 = to_host(Y1), to_host(Y2)
    assert np.all(np.isfinite(y1.astype(np.float32))) and np.all(np.isfinite(y2.astype(np.float32)))
    # layer 2 against the oracle on the Y layer 1 produced
    Wq2_o, sW2_o = orc.quantize_weight_colwise(W2)
    Y2_o, _, _, cnt = orc.mixed_linear(y1, Wq2_o, sW2_o, W2, 2.0)
    assert cnt >= 1
    assert_y_close(y2, Y2_o, "dependent layer")
    assert device_status_clean()


def test_chain_replays_from_a_cuda_graph():
    T = 16
    layers = make_layers(T, seed=11)
    args = [(l["Xd"], l["Wq"], l["sW"], l["Wd"], 6.0, None) for l in layers]
    outs = i8.int8_mixed_linear_chain(args)
    torch.cuda.synchronize()
    want = [to_host(y).copy() for y in outs]
    need = i8.int8_mixed_linear_chain_workspace_size(args)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    Ys = [torch.empty_like(y) for y in outs]
    graph_args = [(a[0], a[1], a[2], a[3], a[4], y) for a, y in zip(args, Ys)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        i8.int8_mixed_linear_chain(graph_args, workspace_buf=ws, stream=s)   # warm the stream once
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            i8.int8_mixed_linear_chain(graph_args, workspace_buf=ws, stream=s)
    for y in Ys:
        y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for w, y in zip(want, Ys):
        assert np.array_equal(w.view(np.uint16), to_host(y).view(np.uint16))
    del g
    assert device_status_clean()
