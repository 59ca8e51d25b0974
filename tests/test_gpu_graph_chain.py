"""Dependent GEMVs in one CUDA graph, as the decode bench replays a model pass.

Each layer's x is the previous layer's y. The layers run with
AWQ_FLAG_WEIGHTS_STATIC, so inside the graph every launch is a programmatic
dependent of the one before: it may start streaming its weights early and
must still read x only after the previous layer has finished writing it. Two
replays must give the eager chain's bits, and every layer must match the
oracle's own chain (float64 products, each layer's output rounded to fp16
before it feeds the next layer), computed from the seeded input alone."""

import numpy as np
import pytest
import torch

import weight_only_int4_gemv_b200 as awq
from oracle import awq_oracle as O
from parity_util import activations, assert_close, bits, dev, host, oracle_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,layers", [(2, 1024, 6), (1, 4096, 4), (16, 2048, 3)])
def test_dependent_chain_in_one_graph(M, N, layers):
    # square layers, so y of one layer is x of the next; N = 1024 / 2048 / 4096 all cut K into
    # slices (fewer tiles than CTAs), so the replays also reuse the arrival counters
    ls = [oracle_layer(N, N, 0.02, 0.01, True, seed=40 + i) for i in range(layers)]
    packed = [(dev(q), dev(s), dev(z)) for (_, q, s, z, _) in ls]
    ws = [awq.alloc_workspace(M, N, N, True) for _ in ls]
    x0 = dev(activations(M, N, seed=M))
    ys = [torch.empty((M, N), dtype=torch.float16, device="cuda") for _ in ls]

    def chain():
        x = x0
        for i in range(layers):
            awq.awq_gemv(x, *packed[i], workspace=ws[i], out=ys[i], weights_static=True)
            x = ys[i]

    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        chain()                      # eager (also fills the plan caches before capture)
    torch.cuda.synchronize()
    eager = [bits(y).copy() for y in ys]

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        chain()
    for _ in range(2):
        with torch.cuda.stream(stream):
            for y in ys:
                y.zero_()
            g.replay()
        torch.cuda.synchronize()
        for i, y in enumerate(ys):
            assert np.array_equal(bits(y), eager[i]), f"layer {i} differs from the eager chain"
    assert awq.awq_device_error() == 0

    xin = host(x0)
    for i, (_, _, _, _, Wd) in enumerate(ls):
        ref = O.matmul_f64(xin, Wd)
        assert_close(host(ys[i]), ref, f"graph chain layer {i}")
        xin = ref.astype(np.float16)     # the oracle's own fp16 output feeds its next layer
