"""The usage sequence of the design notes, end to end on small shapes: build a
layer, run it in one call and step by step (same output), put experts in cache
slots by a device refresh and run the slotted layer (same output again)."""
import numpy as np
import pytest
import torch

import synthetic as syn
import moe_router_softmax_b200 as moe

pytestmark = pytest.mark.gpu


def test_usage_sequence():
    E, H, I, k, T = 16, 256, 128, 4, 24
    w13, w2 = syn.torch_expert_weights(E, H, I, seed=1, layer=0, device="cuda")
    layer = moe.make_layer(moe.MOE_W_INT4, w13, w2)
    x = torch.from_numpy(syn.activations(T, H, seed=2).view(np.int16)).cuda().view(torch.bfloat16)
    w_router = torch.from_numpy(syn.router_weights(E, H, seed=3)).cuda()

    ids, w, logits = moe.moe_router_topk(x, w_router, k, logits=True)
    y1 = moe.moe_layer_forward(layer, logits, x, k)

    hits = torch.zeros(E, dtype=torch.int32, device="cuda")
    counts, offsets, sorted_route, route_pos = moe.moe_permute(ids, layer.E, hits=hits)
    rows = moe.moe_grouped_ffn(layer, x, k, counts, offsets, sorted_route)
    y2 = moe.moe_combine(rows, route_pos, w)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))

    pool = torch.empty(6 * layer.expert_bytes, dtype=torch.uint8, device="cuda")
    table = torch.full((layer.E,), -1, dtype=torch.int32, device="cuda")
    slotted = moe.MoeLayer(layer.fmt, layer.E, layer.H, layer.I, layer.home, pool=pool, slot_table=table)
    promo, status = moe.moe_refresh_device(hits, 6, table, 6)
    moe.moe_promote_copies(layer.home, pool, layer.expert_bytes, promo, status, 6)
    torch.cuda.synchronize()
    assert int(status[0]) == min(6, int((hits > 0).sum())) and int((table >= 0).sum()) == int(status[0])
    y3 = moe.moe_layer_forward(slotted, logits, x, k)
    assert torch.equal(y1.view(torch.int16), y3.view(torch.int16))
