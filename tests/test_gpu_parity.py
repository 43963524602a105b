"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Routing ids and weights, the permutation, hit counts and the int8/int4 codes are
compared bit for bit; the FFN rows and the combined output by
max|gpu - oracle| / max|oracle| <= 1e-2.  Small cases compare every element and
span several work items and a ragged tail; the full Gemma-shaped layer (128
experts, hidden 2816, intermediate 704, top-8) compares sampled routes and
tokens that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
import moe_router_softmax_b200 as moe
from gpu_support import (FFN_TOL, bf16_dev_to_f64, device_weights_from_host, host_bits, oracle_blob,
                         oracle_layer_for, rel_err)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits_equal(a: np.ndarray, b: np.ndarray) -> bool:
    return np.array_equal(np.ascontiguousarray(a).view(np.uint32), np.ascontiguousarray(b).view(np.uint32))


# ---------------------------------------------------------------------- routing

@pytest.mark.parametrize("T,E,k,kind", [
    (1, 128, 8, "normal"), (8, 128, 8, "normal"), (64, 128, 8, "biased"), (1024, 128, 8, "normal"),
    (16, 8, 2, "normal"), (37, 1000, 32, "normal"), (5, 3, 3, "normal"), (33, 1024, 1, "zipf"),
    (300, 64, 64 // 2, "zipf"), (7, 33, 5, "biased"),
])
def test_route_topk_bit_exact(T, E, k, kind):
    lg = syn.router_logits(T, E, kind, seed=T + E)
    ids, w = moe.moe_route_topk(torch.from_numpy(lg).to(DEV), k)
    oi, ow = oracle.route_topk(lg, k)
    assert np.array_equal(ids.cpu().numpy(), oi)
    assert bits_equal(w.cpu().numpy(), ow)


def test_route_topk_ties_nan_inf():
    rng = np.random.default_rng(3)
    lg = rng.integers(-2, 3, size=(100, 40)).astype(np.float32)
    lg[0, :] = 0.0
    lg[1, 5] = np.nan
    lg[2, [1, 7]] = np.inf
    lg[3, :] = -np.inf
    lg[3, 9] = 1.0
    lg[4, ::3] = -0.0
    ids, w = moe.moe_route_topk(torch.from_numpy(lg).to(DEV), 6)
    oi, ow = oracle.route_topk(lg, 6)
    assert np.array_equal(ids.cpu().numpy(), oi)
    g = w.cpu().numpy()
    assert np.array_equal(np.isnan(g), np.isnan(ow))
    fin = ~np.isnan(ow)
    assert bits_equal(np.where(fin, g, 0), np.where(fin, ow, 0))


# ---------------------------------------------------------------------- permute

@pytest.mark.parametrize("T,k,E", [(1, 8, 128), (64, 8, 128), (1024, 8, 128), (16, 2, 8), (37, 3, 11),
                                   (5000, 8, 1024), (3, 1, 1), (700, 32, 64)])
def test_permute_and_hits_bit_exact(T, k, E):
    rng = np.random.default_rng(T * k + E)
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    bad = rng.random((T, k)) < 0.03
    ids[bad] = rng.choice([-1, E, E + 5, -100], size=int(bad.sum()))
    hits0 = rng.integers(0, 50, size=E).astype(np.uint32)
    hits = torch.from_numpy(hits0.view(np.int32)).to(DEV)
    out = moe.moe_permute(torch.from_numpy(ids).to(DEV), E, hits=hits)
    ref = oracle.permute(ids, E)
    for g, r in zip(out, ref):
        assert np.array_equal(g.cpu().numpy(), r)
    assert np.array_equal(hits.cpu().numpy().view(np.uint32), oracle.hits(ids, E, hits0))


# moe_route_permute: one warp for T*k <= 32 (the one-token cases, (3, 11, 5) and
# the boundary cases with 30 or 32 routes), one CTA for T <= 16 (including
# T*k = 33 and the boundary T = 16, E = 1024, T*k = 512), the two kernels beyond
@pytest.mark.parametrize("T,E,k,kind", [(1, 128, 8, "normal"), (8, 128, 8, "biased"), (16, 128, 8, "normal"),
                                        (1, 1024, 32, "normal"), (3, 11, 5, "normal"), (16, 8, 4, "biased"),
                                        (16, 1024, 32, "normal"), (17, 128, 8, "normal"), (64, 128, 8, "biased"),
                                        (1024, 128, 8, "biased"), (4, 128, 8, "biased"), (2, 40, 16, "normal"),
                                        (5, 1000, 6, "normal"), (1, 1, 1, "normal"), (3, 64, 11, "normal")])
def test_route_permute_matches_the_oracle_and_the_two_calls(T, E, k, kind):
    lg = syn.router_logits(T, E, kind, seed=7 * T + E)
    rng = np.random.default_rng(T + k)
    hits0 = rng.integers(0, 50, size=E).astype(np.uint32)
    h_one = torch.from_numpy(hits0.view(np.int32)).to(DEV)
    h_two = torch.from_numpy(hits0.view(np.int32)).to(DEV)
    d_lg = torch.from_numpy(lg).to(DEV)
    one = moe.moe_route_permute(d_lg, k, hits=h_one)
    ids, w = moe.moe_route_topk(d_lg, k)
    two = (ids, w) + tuple(moe.moe_permute(ids, E, hits=h_two))
    for a, b in zip(one, two):
        assert np.array_equal(a.cpu().numpy().view(np.uint32), b.cpu().numpy().view(np.uint32))
    assert np.array_equal(h_one.cpu().numpy(), h_two.cpu().numpy())
    oi, ow = oracle.route_topk(lg, k)
    assert np.array_equal(one[0].cpu().numpy(), oi)
    assert bits_equal(one[1].cpu().numpy(), ow)
    for g, r in zip(one[2:], oracle.permute(oi, E)):
        assert np.array_equal(g.cpu().numpy(), r)
    assert np.array_equal(h_one.cpu().numpy().view(np.uint32), oracle.hits(oi, E, hits0))


# moe_route_ffn: one token with E <= 128 routes inside the one-token FFN launches
# (the first six cases, E up to 128, k up to 8); E = 200 and T = 5 take the two calls
@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("T,E,H,I,k", [(1, 128, 256, 128, 8), (1, 8, 256, 128, 6), (1, 12, 2816, 704, 8),
                                       (1, 6, 1024, 320, 4), (1, 4, 64, 64, 1), (1, 33, 512, 192, 32),
                                       (1, 200, 256, 128, 8), (5, 16, 512, 192, 3)])
def test_route_ffn_matches_the_two_calls_and_the_oracle(fmt, T, E, H, I, k):
    w13, w2 = syn.expert_weights(E, H, I, seed=E + H + k)
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    x = syn.activations(T, H, seed=H + 1)
    lg = syn.router_logits(T, E, "normal", seed=E * 3 + k)
    rng = np.random.default_rng(E + k)
    hits0 = rng.integers(0, 50, size=E).astype(np.uint32)
    h_one = torch.from_numpy(hits0.view(np.int32)).to(DEV)
    h_two = torch.from_numpy(hits0.view(np.int32)).to(DEV)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    d_lg = torch.from_numpy(lg).to(DEV)
    one = moe.moe_route_ffn(L, d_lg, xd, k, hits=h_one)
    two = moe.moe_route_permute(d_lg, k, hits=h_two)
    rows2 = moe.moe_grouped_ffn(L, xd, k, two[2], two[3], two[4])
    assert moe.moe_take_device_errors() == (0, 0)
    for a, b in zip(one[:6], two):
        assert np.array_equal(a.cpu().numpy().view(np.uint32), b.cpu().numpy().view(np.uint32))
    assert np.array_equal(h_one.cpu().numpy(), h_two.cpu().numpy())
    R = T * k
    assert np.array_equal(one[6][:R].cpu().numpy().view(np.uint32), rows2[:R].cpu().numpy().view(np.uint32))
    oi, ow = oracle.route_topk(lg, k)
    assert np.array_equal(one[0].cpu().numpy(), oi)
    assert bits_equal(one[1].cpu().numpy(), ow)
    for g, r in zip(one[2:6], oracle.permute(oi, E)):
        assert np.array_equal(g.cpu().numpy(), r)
    assert np.array_equal(h_one.cpu().numpy().view(np.uint32), oracle.hits(oi, E, hits0))
    orows = oracle.ffn_routes(oracle_layer_for(fmt, w13, w2), x, oi)
    assert rel_err(one[6].cpu().numpy()[one[5].cpu().numpy().ravel()], orows) <= FFN_TOL


@pytest.mark.parametrize("fmt", [0, 2])
def test_route_ffn_one_token_on_a_slot_table(fmt):
    """The one-token kernels that route for themselves resolve experts through
    the slot table (a pool of 24 slots behind 8 experts) like the other paths."""
    E, H, I, k = 8, 512, 192, 3
    w13, w2 = syn.expert_weights(E, H, I, seed=77)
    slot_of = np.array([23, -1, 17, 5, -1, 20, 0, 11], np.int32)
    Ld, OL = _pool_layers(fmt, E, H, I, w13, w2, slot_of, 24)
    x = syn.activations(1, H, seed=78)
    lg = syn.router_logits(1, E, "normal", seed=91)
    lg[0, 1] += 4.0                          # a home expert as well as pooled ones
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    ids, w, counts, offsets, sr, rp, rows = moe.moe_route_ffn(Ld, torch.from_numpy(lg).to(DEV), xd, k)
    assert moe.moe_take_device_errors() == (0, 0)
    oi, ow, orows, oy = oracle.moe_layer(OL, lg, x, k)
    assert np.array_equal(ids.cpu().numpy(), oi)
    assert (slot_of[oi] >= 0).any() and (slot_of[oi] < 0).any()
    assert rel_err(rows.cpu().numpy()[rp.cpu().numpy().ravel()], orows) <= FFN_TOL


@pytest.mark.parametrize("T", [30, 5])  # 5 tokens x 6 = 30 routes: the one-warp kernel
def test_route_permute_ties_nan_inf(T):
    rng = np.random.default_rng(4)
    lg = rng.integers(-2, 3, size=(30, 40)).astype(np.float32)
    lg[0, :] = 0.0
    lg[1, 5] = np.nan
    lg[2, [1, 7]] = np.inf
    lg[3, :] = -np.inf
    lg[3, 9] = 1.0
    lg[4, ::3] = -0.0
    lg = np.ascontiguousarray(lg[:T])
    ids, w, counts, offsets, sr, rp = moe.moe_route_permute(torch.from_numpy(lg).to(DEV), 6)
    oi, ow = oracle.route_topk(lg, 6)
    assert np.array_equal(ids.cpu().numpy(), oi)
    g = w.cpu().numpy()
    assert np.array_equal(np.isnan(g), np.isnan(ow))
    fin = ~np.isnan(ow)
    assert bits_equal(np.where(fin, g, 0), np.where(fin, ow, 0))
    for a, r in zip((counts, offsets, sr, rp), oracle.permute(oi, 40)):
        assert np.array_equal(a.cpu().numpy(), r)


@pytest.mark.parametrize("n,E", [(1, 4), (5, 4), (100000, 128), (33333, 1024)])
def test_expert_hits_bit_exact(n, E):
    rng = np.random.default_rng(n)
    ids = rng.integers(-3, E + 3, size=n).astype(np.int32)
    h = torch.zeros(E, dtype=torch.int32, device=DEV)
    moe.moe_expert_hits(torch.from_numpy(ids).to(DEV), E, h)
    moe.moe_expert_hits(torch.from_numpy(ids).to(DEV), E, h)
    assert np.array_equal(h.cpu().numpy().view(np.uint32), 2 * oracle.hits(ids, E))


def test_hits_page_vector_on_gpu():
    h = torch.zeros(4, dtype=torch.int32, device=DEV)
    moe.moe_expert_hits(torch.tensor([1, 0, 1, 2, 1], dtype=torch.int32, device=DEV), 4, h)
    assert h.cpu().tolist() == [1, 3, 1, 0]


# ------------------------------------------------------------------- quantisers

def _special_matrix(rows, K, seed):
    w = syn.normal_bf16((rows, K), 0.02, seed, 9)
    w[0] = 0                                         # all-zero row / groups
    w[1, :64] = syn.bf16_bits(np.float32(np.arange(64) - 32) * np.float32(2.0 ** -8))
    w[2, 5] = syn.bf16_bits(np.float32([0.9]))[0]     # outlier
    if rows > 3 and K >= 128:
        w[3, 64:128] = syn.bf16_bits(np.float32([1e-3] * 63 + [-0.5]))
    return w


@pytest.mark.parametrize("rows,K", [(1408, 2816), (2816, 704), (64, 256), (3, 64), (5, 100), (3, 4104)])
def test_quantize_int8_bit_exact(rows, K):
    """(5, 100) and (3, 4104) take the element-loop kernel (K not a multiple of 8,
    or more than 16 chunks per lane); the others the register-resident one."""
    w = _special_matrix(rows, K, rows)
    q, s = moe.moe_quantize_int8(torch.from_numpy(w.view(np.int16)).to(DEV))
    oq, os_ = oracle.quantize_int8(w)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert bits_equal(s.cpu().numpy(), os_)


@pytest.mark.parametrize("rows,K", [(1408, 2816), (2816, 704), (64, 256), (3, 64)])
def test_quantize_int4_bit_exact(rows, K):
    w = _special_matrix(rows, K, rows + 1)
    q, s = moe.moe_quantize_int4(torch.from_numpy(w.view(np.int16)).to(DEV))
    oq, os_ = oracle.quantize_int4(w)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(host_bits(s), os_)


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_packed_blobs_bit_exact(fmt):
    E, H, I = 3, 512, 192
    w13, w2 = syn.expert_weights(E, H, I, seed=5)
    d13, d2 = device_weights_from_host(w13, w2)
    L = moe.make_layer(fmt, d13, d2)
    home = L.home.cpu().numpy()
    eb = L.expert_bytes
    for e in range(E):
        assert np.array_equal(home[e * eb:(e + 1) * eb], oracle_blob(fmt, w13[e], w2[e], H, I))


# ------------------------------------------------------------------ FFN, small

def _run_layer(L, logits, x, k, path=moe.MOE_FFN_AUTO):
    ids, w = moe.moe_route_topk(logits, k)
    counts, offsets, sr, rp = moe.moe_permute(ids, L.E)
    rows = moe.moe_grouped_ffn(L, x, k, counts, offsets, sr, path=path)
    y = moe.moe_combine(rows, rp, w)
    torch.cuda.synchronize()
    return ids, w, counts, offsets, sr, rp, rows, y


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("E,H,I,k,T", [(8, 256, 128, 2, 16), (8, 512, 192, 3, 37), (6, 1024, 320, 2, 61),
                                       (4, 256, 64, 4, 9)])
def test_layer_small_every_element(fmt, E, H, I, k, T):
    w13, w2 = syn.expert_weights(E, H, I, seed=E + H)
    x = syn.activations(T, H, seed=7)
    lg = syn.router_logits(T, E, "normal", seed=11)
    d13, d2 = device_weights_from_host(w13, w2)
    L = moe.make_layer(fmt, d13, d2)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    ids, w, counts, offsets, sr, rp, rows, y = _run_layer(L, torch.from_numpy(lg).to(DEV), xd, k)
    OL = oracle_layer_for(fmt, w13, w2)
    oi, ow, orows, oy = oracle.moe_layer(OL, lg, x, k)
    assert np.array_equal(ids.cpu().numpy(), oi)
    assert bits_equal(w.cpu().numpy(), ow)
    rp_h = rp.cpu().numpy()
    g_rows = rows.cpu().numpy()[rp_h]       # back to flat route order
    assert rel_err(g_rows, orows) <= FFN_TOL
    assert rel_err(bf16_dev_to_f64(y), oy) <= FFN_TOL


def test_layer_forward_single_call_matches_steps():
    E, H, I, k, T = 8, 256, 128, 2, 16  # the tiny layer
    w13, w2 = syn.expert_weights(E, H, I, seed=0)
    x = syn.activations(T, H, seed=0)
    lg = syn.router_logits(T, E, "normal", seed=0)
    L = moe.make_layer(0, *device_weights_from_host(w13, w2))
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    lgd = torch.from_numpy(lg).to(DEV)
    hits = torch.zeros(E, dtype=torch.int32, device=DEV)
    y1 = moe.moe_layer_forward(L, lgd, xd, k, hits=hits)
    y2 = _run_layer(L, lgd, xd, k)[-1]
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    oi, ow, orows, oy = oracle.moe_layer(oracle_layer_for(0, w13, w2), lg, x, k)
    assert rel_err(bf16_dev_to_f64(y1), oy) <= FFN_TOL
    assert np.array_equal(hits.cpu().numpy().view(np.uint32), oracle.hits(oi, E))


def test_slot_table_changes_where_not_what():
    """Router logits and ids are unchanged by placement (expert_pool.rs, module
    doc): the same layer served partly from cache slots gives bit-identical ids,
    weights, rows and output."""
    E, H, I, k, T = 16, 512, 128, 4, 40
    w13, w2 = syn.expert_weights(E, H, I, seed=2)
    L = moe.make_layer(2, *device_weights_from_host(w13, w2))
    eb = L.expert_bytes
    slot_of = np.full(E, -1, np.int32)
    slot_of[[3, 9, 0, 15, 7]] = [4, 0, 2, 1, 3]
    pool = torch.zeros(5 * eb, dtype=torch.uint8, device=DEV)
    moe.moe_copy_to_slots(L.home, pool, eb, np.nonzero(slot_of >= 0)[0], slot_of[slot_of >= 0])
    L2 = moe.MoeLayer(2, E, H, I, L.home, pool=pool, slot_table=torch.from_numpy(slot_of).to(DEV))
    x = torch.from_numpy(syn.activations(T, H, seed=1).view(np.int16)).to(DEV).view(torch.bfloat16)
    lg = torch.from_numpy(syn.router_logits(T, E, "zipf", seed=1)).to(DEV)
    a = _run_layer(L, lg, x, k)
    b = _run_layer(L2, lg, x, k)
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.int32) if u.dtype == torch.float32 else u, v.view(torch.int32) if v.dtype == torch.float32 else v)
    # the pool really is what is read: wipe the home blobs of slotted experts
    home2 = L.home.clone()
    for e in np.nonzero(slot_of >= 0)[0]:
        home2[e * eb:(e + 1) * eb] = 0
    L3 = moe.MoeLayer(2, E, H, I, home2, pool=pool, slot_table=torch.from_numpy(slot_of).to(DEV))
    c = _run_layer(L3, lg, x, k)
    assert torch.equal(a[-1].view(torch.int16), c[-1].view(torch.int16))


def test_empty_batch_and_dropped_routes():
    E, H, I, k = 8, 256, 128, 2
    w13, w2 = syn.expert_weights(E, H, I, seed=4)
    L = moe.make_layer(0, *device_weights_from_host(w13, w2))
    # T == 0 is a no-op everywhere
    x0 = torch.empty((0, H), dtype=torch.bfloat16, device=DEV)
    y0 = moe.moe_layer_forward(L, torch.empty((0, E), device=DEV), x0, k)
    assert y0.shape == (0, H)
    # routes with ids outside [0, E) are dropped from the groups and from the sum
    T = 6
    x = syn.activations(T, H, seed=4)
    ids = np.array([[0, 3], [9, 1], [2, -1], [5, 5 + 8], [7, 6], [-4, 4]], np.int32)
    w = np.full((T, k), 0.5, np.float32)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    counts, offsets, sr, rp = moe.moe_permute(torch.from_numpy(ids).to(DEV), E)
    rows = moe.moe_grouped_ffn(L, xd, k, counts, offsets, sr)
    y = moe.moe_combine(rows, rp, torch.from_numpy(w).to(DEV))
    OL = oracle_layer_for(0, w13, w2)
    orows = oracle.ffn_routes(OL, x, ids)
    oy = oracle.combine(orows, ids, w, E)
    assert rel_err(bf16_dev_to_f64(y), oy) <= FFN_TOL
    assert int(offsets[-1]) == int((ids >= 0).sum() - ((ids >= E).sum()))


def test_one_expert_takes_every_token():
    """Degenerate routing: every token routes to the same k experts (k = E)."""
    E, H, I, T = 4, 256, 128, 70
    w13, w2 = syn.expert_weights(E, H, I, seed=8)
    for fmt in (0, 2):
        L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
        x = syn.activations(T, H, seed=8)
        lg = syn.router_logits(T, E, "normal", seed=8)
        ids, w, counts, offsets, sr, rp, rows, y = _run_layer(
            L, torch.from_numpy(lg).to(DEV), torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16), E)
        assert counts.cpu().tolist() == [T] * E
        oi, ow, orows, oy = oracle.moe_layer(oracle_layer_for(fmt, w13, w2), lg, x, E)
        assert rel_err(bf16_dev_to_f64(y), oy) <= FFN_TOL


# ------------------------------------------------------- FFN, Gemma-shaped layer

_FULL = {}


def _full_layer(fmt):
    """128 experts, hidden 2816, intermediate 704: weights drawn on the device by a
    seeded torch generator; the oracle reads the bf16 bytes back per expert."""
    if fmt not in _FULL:
        E, H, I = 128, 2816, 704
        w13, w2 = syn.torch_expert_weights(E, H, I, seed=0, layer=0, device=DEV)
        L = moe.make_layer(fmt, w13, w2)
        _FULL.clear()
        _FULL[fmt] = (w13, w2, L)
    return _FULL[fmt]


@pytest.mark.parametrize("fmt,kind", [(0, "normal"), (1, "biased"), (2, "normal")])
@pytest.mark.parametrize("T", [1, 8, 64])
def test_gemma_layer_decode_sampled(fmt, kind, T):
    E, H, I, k = 128, 2816, 704, 8
    w13, w2, L = _full_layer(fmt)
    x = syn.activations(T, H, seed=100 + T)
    lg = syn.router_logits(T, E, kind, seed=200 + T)
    ids, w, counts, offsets, sr, rp, rows, y = _run_layer(
        L, torch.from_numpy(lg).to(DEV), torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16), k)
    oi, ow = oracle.route_topk(lg, k)
    assert np.array_equal(ids.cpu().numpy(), oi) and bits_equal(w.cpu().numpy(), ow)
    for g, r in zip((counts, offsets, sr, rp), oracle.permute(oi, E)):
        assert np.array_equal(g.cpu().numpy(), r)
    # sample tokens (all their k routes) for the oracle
    rng = np.random.default_rng(T)
    toks = np.unique(np.r_[0, T - 1, rng.integers(0, T, size=min(T, 3))])
    routes = np.concatenate([np.arange(t * k, (t + 1) * k) for t in toks]).astype(np.int32)
    experts = oi.ravel()[routes]
    h13 = {e: host_bits(w13[e]) for e in set(experts.tolist())}
    h2 = {e: host_bits(w2[e]) for e in set(experts.tolist())}
    w13h = np.zeros((E, 2, H), np.uint16)  # placeholder shape; only sampled experts are packed
    OL = _sparse_oracle_layer(fmt, E, H, I, h13, h2)
    orows = oracle.ffn_some_routes(OL, x, oi, routes)
    g_rows = rows.cpu().numpy()[rp.cpu().numpy()[routes]]
    assert rel_err(g_rows, orows) <= FFN_TOL
    full_rows = np.zeros((T * k, H))
    full_rows[routes] = orows
    oy = oracle.combine(full_rows, oi, ow, E)[toks]
    assert rel_err(bf16_dev_to_f64(y)[toks], oy) <= FFN_TOL
    del w13h


def _sparse_oracle_layer(fmt, E, H, I, h13, h2):
    eb = oracle.expert_bytes(fmt, H, I)
    slot = np.full(E, -1, np.int32)
    ex = sorted(h13)
    pool = np.zeros(len(ex) * eb, np.uint8)
    for i, e in enumerate(ex):
        slot[e] = i
        pool[i * eb:(i + 1) * eb] = oracle_blob(fmt, h13[e], h2[e], H, I)
    return oracle.Layer(fmt, E, H, I, np.zeros(eb, np.uint8), pool=pool, slot_table=slot)


def test_gemma_layer_prefill_sampled():
    """int4 layer, 1024 tokens (the prefill batch): sampled routes and tokens."""
    E, H, I, k, T = 128, 2816, 704, 8, 1024
    w13, w2, L = _full_layer(2)
    x = syn.activations(T, H, seed=5)
    lg = syn.router_logits(T, E, "normal", seed=5)
    ids, w, counts, offsets, sr, rp, rows, y = _run_layer(
        L, torch.from_numpy(lg).to(DEV), torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16), k)
    oi, ow = oracle.route_topk(lg, k)
    assert np.array_equal(ids.cpu().numpy(), oi) and bits_equal(w.cpu().numpy(), ow)
    toks = np.array([0, 1, 511, 1023])
    routes = np.concatenate([np.arange(t * k, (t + 1) * k) for t in toks]).astype(np.int32)
    experts = sorted(set(oi.ravel()[routes].tolist()))
    OL = _sparse_oracle_layer(2, E, H, I, {e: host_bits(w13[e]) for e in experts}, {e: host_bits(w2[e]) for e in experts})
    orows = oracle.ffn_some_routes(OL, x, oi, routes)
    assert rel_err(rows.cpu().numpy()[rp.cpu().numpy()[routes]], orows) <= FFN_TOL
    full_rows = np.zeros((T * k, H))
    full_rows[routes] = orows
    oy = oracle.combine(full_rows, oi, ow, E)[toks]
    assert rel_err(bf16_dev_to_f64(y)[toks], oy) <= FFN_TOL


# ------------------------------------------------------ tensor-core FFN path

def _tc(L, lg, x, k):
    """The layer with the tcgen05 kernels forced (they take every format at every
    H, I that are multiples of 64: the weight maps are 3-D, blob by blob)."""
    return _run_layer(L, lg, x, k, path=moe.MOE_FFN_TC)


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("E,H,I,k,T", [(8, 256, 128, 2, 16), (8, 512, 192, 3, 37), (6, 1024, 320, 2, 61),
                                       (4, 384, 64, 4, 300), (3, 256, 128, 3, 200)])
def test_tc_layer_small_every_element(fmt, E, H, I, k, T):
    """tcgen05 path forced: every row and output against the oracle; shapes with
    several M tiles, a partial last tile (H % 128 != 0), ragged route blocks and
    experts with more than 128 routes (several N blocks)."""
    w13, w2 = syn.expert_weights(E, H, I, seed=E + H + 1)
    x = syn.activations(T, H, seed=8)
    lg = syn.router_logits(T, E, "normal", seed=12)
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    ids, w, counts, offsets, sr, rp, rows, y = _tc(L, torch.from_numpy(lg).to(DEV), xd, k)
    oi, ow, orows, oy = oracle.moe_layer(oracle_layer_for(fmt, w13, w2), lg, x, k)
    assert np.array_equal(ids.cpu().numpy(), oi)
    g_rows = rows.cpu().numpy()[rp.cpu().numpy()]
    assert rel_err(g_rows, orows) <= FFN_TOL
    assert rel_err(bf16_dev_to_f64(y), oy) <= FFN_TOL


@pytest.mark.parametrize("fmt,kind", [(0, "normal"), (1, "biased"), (2, "normal")])
@pytest.mark.parametrize("T", [8, 64])
def test_tc_gemma_layer_decode_sampled(fmt, kind, T):
    E, H, I, k = 128, 2816, 704, 8
    w13, w2, L = _full_layer(fmt)
    x = syn.activations(T, H, seed=300 + T)
    lg = syn.router_logits(T, E, kind, seed=400 + T)
    ids, w, counts, offsets, sr, rp, rows, y = _tc(
        L, torch.from_numpy(lg).to(DEV), torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16), k)
    oi, ow = oracle.route_topk(lg, k)
    toks = np.unique(np.r_[0, T - 1, np.random.default_rng(T).integers(0, T, size=2)])
    routes = np.concatenate([np.arange(t * k, (t + 1) * k) for t in toks]).astype(np.int32)
    experts = sorted(set(oi.ravel()[routes].tolist()))
    OL = _sparse_oracle_layer(fmt, E, H, I, {e: host_bits(w13[e]) for e in experts},
                              {e: host_bits(w2[e]) for e in experts})
    orows = oracle.ffn_some_routes(OL, x, oi, routes)
    assert rel_err(rows.cpu().numpy()[rp.cpu().numpy()[routes]], orows) <= FFN_TOL
    full_rows = np.zeros((T * k, H))
    full_rows[routes] = orows
    oy = oracle.combine(full_rows, oi, ow, E)[toks]
    assert rel_err(bf16_dev_to_f64(y)[toks], oy) <= FFN_TOL


def test_tc_and_gemv_agree_on_the_slot_table():
    """Both kernel paths read experts through the slot table the same way."""
    E, H, I, k, T = 16, 512, 128, 4, 90
    w13, w2 = syn.expert_weights(E, H, I, seed=21)
    L = moe.make_layer(0, *device_weights_from_host(w13, w2))
    eb = L.expert_bytes
    slot_of = np.full(E, -1, np.int32)
    slot_of[[2, 11, 5]] = [1, 0, 2]
    pool = torch.zeros(3 * eb, dtype=torch.uint8, device=DEV)
    moe.moe_copy_to_slots(L.home, pool, eb, np.nonzero(slot_of >= 0)[0], slot_of[slot_of >= 0])
    home2 = L.home.clone()
    for e in np.nonzero(slot_of >= 0)[0]:
        home2[e * eb:(e + 1) * eb] = 0
    L2 = moe.MoeLayer(0, E, H, I, home2, pool=pool, slot_table=torch.from_numpy(slot_of).to(DEV))
    x = torch.from_numpy(syn.activations(T, H, seed=2).view(np.int16)).to(DEV).view(torch.bfloat16)
    lg = torch.from_numpy(syn.router_logits(T, E, "zipf", seed=2)).to(DEV)
    a = _run_layer(L, lg, x, k, path=moe.MOE_FFN_GEMV)[-2]
    b = _tc(L2, lg, x, k)[-2]
    n = a.shape[0]
    assert rel_err(b.cpu().numpy()[:n], a.cpu().numpy()) <= FFN_TOL


def _pool_layers(fmt, E, H, I, w13, w2, slot_of, n_slots):
    """The same slotted layer on both sides: device pool of n_slots blobs filled
    from the device home, oracle pool built by the oracle's own quantiser and
    packer, the same slot table; home of every slotted expert wiped on the device
    so that only the pool can serve it."""
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    eb = L.expert_bytes
    pool = torch.zeros(n_slots * eb, dtype=torch.uint8, device=DEV)
    held = np.nonzero(slot_of >= 0)[0]
    moe.moe_copy_to_slots(L.home, pool, eb, held, slot_of[held])
    home2 = L.home.clone()
    for e in held:
        home2[e * eb:(e + 1) * eb] = 0
    table = torch.from_numpy(slot_of.astype(np.int32)).to(DEV)
    Ld = moe.MoeLayer(fmt, E, H, I, home2, pool=pool, slot_table=table, pool_slots=n_slots)
    oeb = oracle.expert_bytes(fmt, H, I)
    ohome = np.concatenate([oracle_blob(fmt, w13[e], w2[e], H, I) for e in range(E)])
    opool = np.zeros(n_slots * oeb, np.uint8)
    for e in held:
        opool[slot_of[e] * oeb:(slot_of[e] + 1) * oeb] = oracle_blob(fmt, w13[e], w2[e], H, I)
    OL = oracle.Layer(fmt, E, H, I, ohome, pool=opool, slot_table=slot_of.astype(np.int32))
    return Ld, OL


@pytest.mark.parametrize("T", [45, 1])
@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("path", [moe.MOE_FFN_GEMV, moe.MOE_FFN_TC])
def test_pool_with_more_slots_than_experts_matches_the_oracle(fmt, path, T):
    """A pool holds more slots than the layer has experts (prain's 540 cache
    slots are shared by the layers; remote_experts.cpp reads a cached expert from
    its device slot): 8 experts, 24 slots, slot ids up to 23.  Both kernel paths
    (at one token the GEMV path's one-token kernels) against the oracle on the
    same slot table, every row and output element."""
    E, H, I, k = 8, 512, 192, 3
    w13, w2 = syn.expert_weights(E, H, I, seed=77)
    slot_of = np.array([23, -1, 17, 5, -1, 20, 0, 11], np.int32)
    Ld, OL = _pool_layers(fmt, E, H, I, w13, w2, slot_of, 24)
    x = syn.activations(T, H, seed=78)
    lg = syn.router_logits(T, E, "normal", seed=79)
    if T == 1:
        lg[0, 1] += 4.0                      # the token reads a home expert as well as pooled ones
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    ids, w, counts, offsets, sr, rp, rows, y = _run_layer(Ld, torch.from_numpy(lg).to(DEV), xd, k, path=path)
    assert moe.moe_take_device_errors() == (0, 0)
    oi, ow, orows, oy = oracle.moe_layer(OL, lg, x, k)
    assert (slot_of[oi] >= 0).any() and (slot_of[oi] < 0).any()
    assert np.array_equal(ids.cpu().numpy(), oi)
    assert rel_err(rows.cpu().numpy()[rp.cpu().numpy()], orows) <= FFN_TOL
    assert rel_err(bf16_dev_to_f64(y), oy) <= FFN_TOL


@pytest.mark.parametrize("T", [40, 1])
@pytest.mark.parametrize("path", [moe.MOE_FFN_GEMV, moe.MOE_FFN_TC])
def test_slot_past_the_pool_is_refused_and_reported(path, T):
    """A slot table entry at or past pool_slots is refused on the device: that
    expert's routes are skipped (their rows keep what the caller put there), the
    kernels record the bad slot for moe_take_device_errors, and every other
    expert's rows still match the oracle.  The kernels resolve such an expert to
    its home blob for any address they form, so nothing outside the buffers is
    read.  At one token the GEMV path runs its one-token kernels."""
    E, H, I, k = 8, 256, 128, 2
    w13, w2 = syn.expert_weights(E, H, I, seed=81)
    slot_of = np.array([2, -1, 0, -1, 1, -1, -1, -1], np.int32)
    Ld, OL = _pool_layers(2, E, H, I, w13, w2, slot_of, 3)
    bad = slot_of.copy()
    bad[4] = 3                               # == pool_slots: one past the end
    Ld.slot_table.copy_(torch.from_numpy(bad))
    x = syn.activations(T, H, seed=82)
    lg = syn.router_logits(T, E, "normal", seed=83)
    if T == 1:
        lg[0, 4] += 6.0                      # the token routes to the bad slot's expert
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    moe.moe_take_device_errors()             # start from a clear word
    ids, w = moe.moe_route_topk(torch.from_numpy(lg).to(DEV), k)
    counts, offsets, sr, rp = moe.moe_permute(ids, E)
    rows = torch.full((T * k, H), 7.0, dtype=torch.float32, device=DEV)
    moe.moe_grouped_ffn(Ld, xd, k, counts, offsets, sr, rows=rows, path=path)
    code, info = moe.moe_take_device_errors()
    assert code in (0x2005, 0x2006) and info == 3
    oi, _ = oracle.route_topk(lg, k)
    assert int((oi == 4).sum()) > 0
    rp_h = rp.cpu().numpy()
    g = rows.cpu().numpy()[rp_h]
    mine = (oi.ravel() == 4)
    assert np.all(g[mine] == 7.0)            # skipped: untouched
    orows = oracle.ffn_routes(OL, x, oi)
    assert rel_err(g[~mine], orows[~mine]) <= FFN_TOL
    assert moe.moe_take_device_errors() == (0, 0)


# ------------------------------------------------------- [miss] min_weight

@pytest.mark.parametrize("mw", [0.0, 0.3, 0.6, 0.95, 1.0])
def test_route_min_weight_bit_exact(mw):
    T, E, k = 300, 128, 8
    lg = syn.router_logits(T, E, "zipf", seed=31)
    oi, ow = oracle.route_topk(lg, k)
    slot = np.where(np.random.default_rng(4).random(E) < 0.15, np.arange(E), -1).astype(np.int32)
    ids = torch.from_numpy(oi).to(DEV)
    w = torch.from_numpy(ow).to(DEV)
    moe.moe_route_min_weight(ids, w, E, mw, slot_table=torch.from_numpy(slot).to(DEV))
    ri, rw = oracle.route_min_weight(oi, ow, slot, E, mw)
    assert np.array_equal(ids.cpu().numpy(), ri)
    assert bits_equal(w.cpu().numpy(), rw)


def test_layer_with_min_weight_matches_oracle():
    """The whole layer with partial routing: dropped routes join no group and add
    nothing; the kept ones carry the rescaled weights."""
    E, H, I, k, T = 16, 512, 128, 4, 40
    w13, w2 = syn.expert_weights(E, H, I, seed=9)
    L = moe.make_layer(0, *device_weights_from_host(w13, w2))
    x = syn.activations(T, H, seed=9)
    lg = syn.router_logits(T, E, "zipf", seed=9)
    slot = np.where(np.arange(E) % 3 == 0, np.arange(E), -1).astype(np.int32)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    ids, w = moe.moe_route_topk(torch.from_numpy(lg).to(DEV), k)
    moe.moe_route_min_weight(ids, w, E, 0.5, slot_table=torch.from_numpy(slot).to(DEV))
    counts, offsets, sr, rp = moe.moe_permute(ids, E)
    rows = moe.moe_grouped_ffn(L, xd, k, counts, offsets, sr)
    y = moe.moe_combine(rows, rp, w)
    oi, ow = oracle.route_topk(lg, k)
    oi, ow = oracle.route_min_weight(oi, ow, slot, E, 0.5)
    OL = oracle_layer_for(0, w13, w2)
    oy = oracle.combine(oracle.ffn_routes(OL, x, oi), oi, ow, E)
    assert (oi < 0).any()
    assert rel_err(bf16_dev_to_f64(y), oy) <= FFN_TOL


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_one_token_with_repeated_ids(fmt):
    """One-token GEMV calls must be right when a caller's ids repeat an expert
    within the token (here experts 2 and 5 twice each) and when the permutation
    dropped an id (so fewer than k routes have an expert)."""
    E, H, I, k = 8, 256, 128, 6
    w13, w2 = syn.expert_weights(E, H, I, seed=12)
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    x = syn.activations(1, H, seed=12)
    ids = np.array([[2, 5, 2, 7, 5, -1]], np.int32)
    w = np.array([[0.3, 0.2, 0.1, 0.15, 0.15, 0.1]], np.float32)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    counts, offsets, sr, rp = moe.moe_permute(torch.from_numpy(ids).to(DEV), E)
    rows = moe.moe_grouped_ffn(L, xd, k, counts, offsets, sr, path=moe.MOE_FFN_GEMV)
    y = moe.moe_combine(rows, rp, torch.from_numpy(w).to(DEV))
    OL = oracle_layer_for(fmt, w13, w2)
    orows = oracle.ffn_routes(OL, x, ids)
    valid = (ids.ravel() >= 0)
    got = rows.cpu().numpy()[rp.cpu().numpy().ravel()[valid]]
    assert rel_err(got, orows[valid]) <= FFN_TOL
    assert rel_err(bf16_dev_to_f64(y), oracle.combine(orows, ids, w, E)) <= FFN_TOL


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("E,H,I,k", [(8, 256, 128, 2), (6, 1024, 320, 4), (16, 512, 192, 8), (12, 2816, 704, 8),
                                     (4, 64, 64, 1)])
def test_one_token_every_element(fmt, E, H, I, k):
    """One-token batches through the GEMV path's one-token kernels (the k routes'
    rows split evenly over all warps of the grid, each read in passes of a few
    chunks per lane): every row against the oracle, at shapes whose rows split
    unevenly over the warps and lane groups, and rows that take one pass or
    several."""
    w13, w2 = syn.expert_weights(E, H, I, seed=E * 7 + I)
    x = syn.activations(1, H, seed=H)
    lg = syn.router_logits(1, E, "normal", seed=k)
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    ids, w, counts, offsets, sr, rp, rows, y = _run_layer(L, torch.from_numpy(lg).to(DEV), xd, k,
                                                          path=moe.MOE_FFN_GEMV)
    oi, ow, orows, oy = oracle.moe_layer(oracle_layer_for(fmt, w13, w2), lg, x, k)
    assert np.array_equal(ids.cpu().numpy(), oi)
    assert rel_err(rows.cpu().numpy()[rp.cpu().numpy()], orows) <= FFN_TOL
    assert rel_err(bf16_dev_to_f64(y), oy) <= FFN_TOL
    assert moe.moe_take_device_errors() == (0, 0)


# moe_layer_forward at one token: where the FFN's launches route the token, the
# second launch also takes the combine (each CTA sums the k routes of its own
# output rows), so y must be bit-identical to moe_route_ffn + moe_combine; the
# cases cover CTAs without rows (H = 64), k = 32 and E = 200 (two calls, then
# the separate combine)
@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("E,H,I,k", [(128, 256, 128, 8), (8, 256, 128, 6), (128, 2816, 704, 8), (6, 1024, 320, 4),
                                     (4, 64, 64, 1), (33, 512, 192, 32), (200, 256, 128, 8)])
def test_layer_forward_one_token_combine_in_the_ffn(fmt, E, H, I, k):
    w13, w2 = syn.expert_weights(E, H, I, seed=E + 7 * k)
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    x = syn.activations(1, H, seed=H + 3)
    lg = syn.router_logits(1, E, "normal", seed=E * 5 + k)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    d_lg = torch.from_numpy(lg).to(DEV)
    h1 = torch.zeros(E, dtype=torch.int32, device=DEV)
    h2 = torch.zeros(E, dtype=torch.int32, device=DEV)
    ids1 = torch.empty((1, k), dtype=torch.int32, device=DEV)
    w1 = torch.empty((1, k), dtype=torch.float32, device=DEV)
    ys = []
    for _ in range(2):  # twice: the second call finds the previous call's shared memory and y
        ys.append(moe.moe_layer_forward(L, d_lg, xd, k, hits=h1, ids_out=ids1, w_out=w1))
    ids, w, counts, offsets, sr, rp, rows = moe.moe_route_ffn(L, d_lg, xd, k, hits=h2)
    h2 += torch.from_numpy(oracle.hits(oracle.route_topk(lg, k)[0], E).view(np.int32)).to(DEV)
    y2 = moe.moe_combine(rows, rp, w, torch.empty((1, H), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert moe.moe_take_device_errors() == (0, 0)
    for y1 in ys:
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(ids1, ids) and torch.equal(w1.view(torch.int32), w.view(torch.int32))
    assert torch.equal(h1, h2)
    oi, ow, orows, oy = oracle.moe_layer(oracle_layer_for(fmt, w13, w2), lg, x, k)
    assert np.array_equal(ids1.cpu().numpy(), oi)
    assert rel_err(bf16_dev_to_f64(ys[0]), oy) <= FFN_TOL


@pytest.mark.parametrize("fmt", [0, 2])
def test_layer_forward_one_token_combine_on_a_slot_table(fmt):
    """The fused one-token combine reads the rows of pooled and home experts
    alike: y equals the oracle's on a 24-slot pool behind 8 experts."""
    E, H, I, k = 8, 512, 192, 3
    w13, w2 = syn.expert_weights(E, H, I, seed=79)
    slot_of = np.array([23, -1, 17, 5, -1, 20, 0, 11], np.int32)
    Ld, OL = _pool_layers(fmt, E, H, I, w13, w2, slot_of, 24)
    x = syn.activations(1, H, seed=80)
    lg = syn.router_logits(1, E, "normal", seed=93)
    lg[0, 1] += 4.0
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    d_lg = torch.from_numpy(lg).to(DEV)
    y1 = moe.moe_layer_forward(Ld, d_lg, xd, k)
    ids, w, counts, offsets, sr, rp, rows = moe.moe_route_ffn(Ld, d_lg, xd, k)
    y2 = moe.moe_combine(rows, rp, w, torch.empty((1, H), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert moe.moe_take_device_errors() == (0, 0)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    oi, ow, orows, oy = oracle.moe_layer(OL, lg, x, k)
    assert (slot_of[oi] >= 0).any() and (slot_of[oi] < 0).any()
    assert rel_err(bf16_dev_to_f64(y1), oy) <= FFN_TOL


@pytest.mark.parametrize("case", ["ties", "nan", "inf", "neg_inf", "neg_zero"])
def test_layer_forward_one_token_degenerate_logits(case):
    """One token through moe_layer_forward (routing and combine inside the FFN's
    launches) with degenerate router logits: all equal (ties to the lower id),
    a NaN, +inf entries, all -inf but one, -0.0 entries.  ids and weights match
    the oracle's routing bit for bit and y matches the separate calls bit for bit."""
    E, H, I, k = 16, 512, 192, 4
    w13, w2 = syn.expert_weights(E, H, I, seed=101)
    L = moe.make_layer(0, *device_weights_from_host(w13, w2))
    x = syn.activations(1, H, seed=102)
    lg = syn.router_logits(1, E, "normal", seed=103)
    if case == "ties":
        lg[:] = 0.5
    elif case == "nan":
        lg[0, 3] = np.nan
    elif case == "inf":
        lg[0, [2, 9]] = np.inf
    elif case == "neg_inf":
        lg[:] = -np.inf
        lg[0, 7] = 1.0
    else:
        lg[0, ::3] = -0.0
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    d_lg = torch.from_numpy(lg).to(DEV)
    ids1 = torch.empty((1, k), dtype=torch.int32, device=DEV)
    w1 = torch.empty((1, k), dtype=torch.float32, device=DEV)
    y1 = moe.moe_layer_forward(L, d_lg, xd, k, ids_out=ids1, w_out=w1)
    ids, w, counts, offsets, sr, rp, rows = moe.moe_route_ffn(L, d_lg, xd, k)
    y2 = moe.moe_combine(rows, rp, w, torch.empty((1, H), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert moe.moe_take_device_errors() == (0, 0)
    oi, ow = oracle.route_topk(lg, k)
    assert np.array_equal(ids1.cpu().numpy(), oi)
    g = w1.cpu().numpy()
    assert np.array_equal(np.isnan(g), np.isnan(ow))  # NaN weights where the oracle has them
    fin = ~np.isnan(ow)
    assert bits_equal(np.where(fin, g, 0), np.where(fin, ow, 0))
    assert torch.equal(w1.view(torch.int32), w.view(torch.int32))
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
