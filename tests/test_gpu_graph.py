"""The layer chained through several calls, replayed from one CUDA graph.

The library launches its kernels with programmatic dependent launch, so a graph
captured from them carries programmatic edges between consecutive kernels.  Three
layers called back to back (each layer's output is the next one's input) must give,
from a graph replay, exactly the bytes the same calls give eagerly, for the GEMV
and the tensor-core FFN paths and all three weight formats; and the eager result
itself must match the oracle (checked on the first layer).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
import moe_router_softmax_b200 as moe
from gpu_support import FFN_TOL, oracle_layer_for, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layers(fmt, E, H, I, n):
    out = []
    for l in range(n):
        w13, w2 = syn.expert_weights(E, H, I, seed=5, layer=l)
        d13 = torch.from_numpy(w13.view(np.int16)).to(DEV).view(torch.bfloat16)
        d2 = torch.from_numpy(w2.view(np.int16)).to(DEV).view(torch.bfloat16)
        out.append((moe.make_layer(fmt, d13, d2), w13, w2))
    return out


@pytest.mark.parametrize("fmt", ["bf16", "int8", "int4"])
@pytest.mark.parametrize("T", [1, 3, 40])  # 1: the routing and the combine inside the FFN's launches
def test_graph_replay_equals_eager_and_oracle(fmt, T):
    E, H, I, k, n = 16, 256, 128, 4, 3
    layers = _layers(moe.FMT[fmt], E, H, I, n)
    x0 = torch.from_numpy(syn.activations(T, H, seed=T).view(np.int16)).to(DEV).view(torch.bfloat16)
    logits = [torch.from_numpy(syn.router_logits(T, E, "normal", seed=T, layer=l)).to(DEV) for l in range(n)]
    ws = [torch.empty(moe.moe_layer_forward_workspace(lay, T, k), dtype=torch.uint8, device=DEV)
          for lay, _, _ in layers]
    ys = [torch.empty((T, H), dtype=torch.bfloat16, device=DEV) for _ in range(n)]

    def chain():
        x = x0
        for l, (lay, _, _) in enumerate(layers):
            moe.moe_layer_forward(lay, logits[l], x, k, y=ys[l], ws=ws[l])
            x = ys[l]

    chain()
    torch.cuda.synchronize()
    eager = [y.clone() for y in ys]
    for y in ys:
        y.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        chain()
    for _ in range(3):
        for y in ys:
            y.zero_()
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(ys, eager):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # the first layer against the oracle
    lay, w13, w2 = layers[0]
    olayer = oracle_layer_for(oracle.FMT_NAMES[fmt], w13, w2)
    _, _, _, y_ref = oracle.moe_layer(olayer, logits[0].cpu().numpy(), x0.view(torch.int16).cpu().numpy().view(np.uint16), k)
    assert rel_err(eager[0].float().cpu().numpy(), y_ref) <= FFN_TOL
    del g
