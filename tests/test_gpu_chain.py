"""awq_gemv_chain on the GPU: several decode products in one launch, where a
layer's input may be an earlier layer's output ("AutoAWQ" code tour, "The big
picture": the GEMV kernel for decoding; "AutoAWQ" capability page: fused
blocks save launches).

Every layer is compared with the oracle's own chain: float64 products over
the oracle's dequantized weights, each layer's output rounded to fp16 before
it feeds the next, all from the seeded inputs alone. Where a layer's K split
matches that of a lone awq_gemv call, its bits must equal that call's on the
same input."""

import numpy as np
import pytest
import torch

import weight_only_int4_gemv_b200 as awq
from oracle import awq_oracle as O
from parity_util import activations, assert_close, bits, dev, host, oracle_layer

pytestmark = pytest.mark.gpu


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _packed(layer, zp, packed_zeros=False):
    _, q, s, z, _ = layer
    z = dev(z) if zp else None
    if packed_zeros:
        z = awq.awq_pack_zeros(z)
    return dev(q), dev(s), z


def _oracle_chain(x0, specs):
    """specs: [(Wd or (Wg, Wu) for silu, x_from)] -> list of float64 outputs."""
    outs, ins = [], []
    for Wd, x_from in specs:
        xin = x0 if x_from < 0 else outs[x_from].astype(np.float16)
        if isinstance(Wd, tuple):
            y = O.gate_up_silu_f64(xin, *Wd)
        else:
            y = O.matmul_f64(xin, Wd)
        outs.append(y)
        ins.append(xin)
    return outs


@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 16])
@pytest.mark.parametrize("N,K", [(4096, 4096), (1000, 1024), (14336 // 2, 512)])
def test_chain_one_layer_matches_oracle_and_gemv(M, N, K):
    layer = oracle_layer(N, K, 0.02, 0.01, True, seed=N + K)
    q, s, z = _packed(layer, True)
    xh = activations(M, K, seed=M)
    x = dev(xh)
    y = awq.awq_gemv_chain(M, [dict(x=x, qweight=q, scales=s, zeros=z)])[0]
    torch.cuda.synchronize()
    assert_close(host(y), O.matmul_f64(xh, layer[4]), f"chain M={M} N={N} K={K}")
    if (N + 15) // 16 >= 2 * _sms():
        # whole tiles, no K split in either entry point: same sums in the same order
        ref = awq.awq_gemv(x, q, s, z, workspace=awq.alloc_workspace(M, N, K, True))
        assert np.array_equal(bits(y), bits(ref))
    assert awq.awq_device_error() == 0


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("zp,packed", [(True, False), (False, False), (True, True)])
def test_chain_decode_layer_with_dependencies(M, zp, packed):
    """A Llama-3-8B-shaped decode layer in one launch: q_proj (4096 x 4096) on
    x; gate_proj and up_proj (14336 x 4096) on q_proj's output; down_proj
    (4096 x 14336) on up_proj's output."""
    shapes = [(4096, 4096, -1), (14336, 4096, 0), (14336, 4096, 0), (4096, 14336, 2)]
    ls = [oracle_layer(N, K, 0.02, 0.01, zp, seed=60 + i) for i, (N, K, _) in enumerate(shapes)]
    xh = activations(M, 4096, seed=5)
    specs = []
    for i, ((N, K, xf), layer) in enumerate(zip(shapes, ls)):
        q, s, z = _packed(layer, zp, packed)
        specs.append(dict(x=dev(xh) if xf < 0 else None, x_from=xf, qweight=q, scales=s, zeros=z))
    chain = awq.GemvChain(M, specs, weights_static=True)
    ys = chain()
    torch.cuda.synchronize()
    refs = _oracle_chain(xh, [(layer[4], xf) for layer, (_, _, xf) in zip(ls, shapes)])
    for i, (y, ref) in enumerate(zip(ys, refs)):
        assert_close(host(y), ref, f"layer {i} M={M} zp={zp} packed={packed}")
    # each layer against a lone awq_gemv on the chain's own input for it (GPU vs GPU)
    for i, (N, K, xf) in enumerate(shapes):
        if (N + 15) // 16 >= 2 * _sms():
            xin = dev(xh) if xf < 0 else ys[xf]
            ref = awq.awq_gemv(xin, specs[i]["qweight"], specs[i]["scales"], specs[i]["zeros"],
                               workspace=awq.alloc_workspace(M, N, K, zp, packed_zeros=packed))
            assert np.array_equal(bits(ys[i]), bits(ref)), f"layer {i}"
    assert awq.awq_device_error() == 0


@pytest.mark.parametrize("M", [1, 3, 16])
def test_chain_fused_mlp(M):
    """q_proj -> fused gate/up with silu(gate) * up -> down_proj on its output,
    the MLP of a decode step as the fuser builds it."""
    D, F = 2048, 5632
    lq = oracle_layer(D, D, 0.02, 0.01, True, seed=70)
    lg = oracle_layer(F, D, 0.02, 0.01, True, seed=71)
    lu = oracle_layer(F, D, 0.02, 0.01, True, seed=72)
    ld = oracle_layer(D, F, 0.02, 0.01, True, seed=73)
    qg, sg, zg = _packed(lg, True)
    qu, su, zu = _packed(lu, True)
    q2, s2, z2 = awq.awq_interleave_gate_up(qg, sg, zg, qu, su, zu)
    xh = activations(M, D, seed=6)
    specs = [dict(x=dev(xh), **dict(zip(("qweight", "scales", "zeros"), _packed(lq, True)))),
             dict(x_from=0, qweight=q2, scales=s2, zeros=z2, silu_mul=True),
             dict(x_from=1, **dict(zip(("qweight", "scales", "zeros"), _packed(ld, True))))]
    ys = awq.awq_gemv_chain(M, specs, weights_static=True)
    torch.cuda.synchronize()
    assert ys[1].shape == (M, F)
    refs = _oracle_chain(xh, [(lq[4], -1), ((lg[4], lu[4]), 0), (ld[4], 1)])
    for i, (y, ref) in enumerate(zip(ys, refs)):
        assert_close(host(y), ref, f"fused chain layer {i} M={M}")


def test_chain_every_batch_size_small_layers():
    """M = 1 .. 16 on a chain of small layers (fewer tiles than CTAs: K is
    split over CTAs and summed through the workspace), K = 128 (one group,
    a stage with fewer groups than consumer warps) and a ragged N (1000: the
    last tile holds 8 rows)."""
    shapes = [(256, 128, -1), (1000, 256, 0), (384, 256, 0), (640, 384, 2)]
    ls = [oracle_layer(N, K, 0.02, 0.01, True, seed=80 + i) for i, (N, K, _) in enumerate(shapes)]
    for M in range(1, 17):
        xh = activations(M, 128, seed=M)
        specs = []
        for (N, K, xf), layer in zip(shapes, ls):
            q, s, z = _packed(layer, True)
            specs.append(dict(x=dev(xh) if xf < 0 else None, x_from=xf, qweight=q, scales=s, zeros=z))
        ys = awq.awq_gemv_chain(M, specs)
        torch.cuda.synchronize()
        refs = _oracle_chain(xh, [(layer[4], xf) for layer, (_, _, xf) in zip(ls, shapes)])
        for i, (y, ref) in enumerate(zip(ys, refs)):
            assert_close(host(y), ref, f"small chain layer {i} M={M}")
    assert awq.awq_device_error() == 0


def test_chain_repeated_calls_and_graph_replay():
    """The workspace is left ready for the next call: repeated calls,
    and a CUDA graph of two chained launches replayed twice, give the eager
    bits (a counter left over would skip or repeat a K-slice sum; an output
    copy left from the previous call would be read as this call's input)."""
    shapes = [(2048, 2048, -1), (2048, 2048, 0), (8192, 2048, 1), (2048, 8192, 2)]
    ls = [oracle_layer(N, K, 0.02, 0.01, True, seed=90 + i) for i, (N, K, _) in enumerate(shapes)]
    M = 2
    xh = activations(M, 2048, seed=9)
    x = dev(xh)
    specs = []
    for (N, K, xf), layer in zip(shapes, ls):
        q, s, z = _packed(layer, True)
        specs.append(dict(x=x if xf < 0 else None, x_from=xf, qweight=q, scales=s, zeros=z))
    a = awq.GemvChain(M, specs, weights_static=True)
    # a second chain whose input is the first chain's last output
    specs2 = [dict(specs[0], x=a.outputs[3])] + [dict(sp) for sp in specs[1:]]
    b = awq.GemvChain(M, specs2, weights_static=True)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        a()
        b()
    torch.cuda.synchronize()
    eager = [bits(y).copy() for y in a.outputs + b.outputs]
    for _ in range(2):
        with torch.cuda.stream(stream):
            a()
            b()
        torch.cuda.synchronize()
        assert all(np.array_equal(bits(y), e) for y, e in zip(a.outputs + b.outputs, eager))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        a()
        b()
    for _ in range(2):
        with torch.cuda.stream(stream):
            for y in a.outputs + b.outputs:
                y.zero_()
            g.replay()
        torch.cuda.synchronize()
        assert all(np.array_equal(bits(y), e) for y, e in zip(a.outputs + b.outputs, eager))
    refs = _oracle_chain(xh, [(layer[4], xf) for layer, (_, _, xf) in zip(ls, shapes)])
    for i, (y, ref) in enumerate(zip(a.outputs, refs)):
        assert_close(host(y), ref, f"graph chain layer {i}")
    refs2 = _oracle_chain(refs[3].astype(np.float16), [(layer[4], xf) for layer, (_, _, xf) in zip(ls, shapes)])
    for i, (y, ref) in enumerate(zip(b.outputs, refs2)):
        assert_close(host(y), ref, f"second chain layer {i}")
    assert awq.awq_device_error() == 0


def test_chain_wait_gives_up_and_recovers():
    """The bounded-wait give-up path, made to run out without a fault: with
    the pipeline-wait limit cut to 1 ns the first wait that does not complete
    at once (a stage whose copies are still in flight, or the second layer's
    wait for the first) gives up, the call records bit 2 of the device error
    word, lets its copies in flight land and returns. With the limit restored the same chain, on the same workspace,
    matches the oracle again: the abandoned call still brought every counter
    back to zero."""
    shapes = [(14336, 4096, -1), (4096, 14336, 0)]
    ls = [oracle_layer(N, K, 0.02, 0.01, True, seed=100 + i) for i, (N, K, _) in enumerate(shapes)]
    xh = activations(1, 4096, seed=10)
    specs = []
    for (N, K, xf), layer in zip(shapes, ls):
        q, s, z = _packed(layer, True)
        specs.append(dict(x=dev(xh) if xf < 0 else None, x_from=xf, qweight=q, scales=s, zeros=z))
    chain = awq.GemvChain(1, specs)
    assert awq.awq_device_error() == 0
    try:
        awq.awq_debug_set_wait_limit_ns(1)
        chain()
        torch.cuda.synchronize()
        err = awq.awq_device_error()
    finally:
        awq.awq_debug_set_wait_limit_ns(0)
    assert err & 4, f"error word {err:#x}: no wait gave up"
    ys = chain()
    torch.cuda.synchronize()
    assert awq.awq_device_error() == 0
    refs = _oracle_chain(xh, [(layer[4], xf) for layer, (_, _, xf) in zip(ls, shapes)])
    for i, (y, ref) in enumerate(zip(ys, refs)):
        assert_close(host(y), ref, f"after recovery layer {i}")


def test_chains_taking_turns_on_one_workspace():
    """Two chains of different layers on one workspace, each call after the
    first of a chain made on a freshly zeroed workspace (the contract when
    the layers change), and a chain called twice in a row on it: every call
    gives the bits of the same chain on a workspace of its own."""
    M = 1
    shapes_a = [(4096, 2048, -1), (2048, 4096, 0), (4096, 2048, 1)]
    shapes_b = [(1024, 4096, -1), (8192, 1024, 0), (4096, 8192, 1), (4096, 4096, 2)]
    chains = []
    for shapes, seed in ((shapes_a, 120), (shapes_b, 130)):
        specs = []
        for i, (N, K, xf) in enumerate(shapes):
            q, s_, z = _packed(oracle_layer(N, K, 0.02, 0.01, True, seed=seed + i), True)
            specs.append(dict(x=dev(activations(M, K, seed=seed)) if xf < 0 else None, x_from=xf,
                              qweight=q, scales=s_, zeros=z))
        chains.append(specs)
    own = [awq.GemvChain(M, sp, weights_static=True) for sp in chains]
    for c in own:
        c()
    torch.cuda.synchronize()
    ref = [[bits(y).copy() for y in c.outputs] for c in own]
    need = max(c.workspace.numel() for c in own)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    shared = [awq.GemvChain(M, sp, weights_static=True, workspace=ws) for sp in chains]
    for k, which in enumerate([0, 0, 1, 1, 1, 0, 1]):
        if k > 0 and which != [0, 0, 1, 1, 1, 0, 1][k - 1]:
            ws.zero_()
        c = shared[which]
        c()
        torch.cuda.synchronize()
        for i, y in enumerate(c.outputs):
            assert np.array_equal(bits(y), ref[which][i]), f"call {k} (chain {which}) layer {i}"
    assert awq.awq_device_error() == 0
