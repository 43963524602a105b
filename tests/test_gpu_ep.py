"""Expert parallelism on one GPU.

* moe_gather_rows and moe_ep_recv_ids against plain torch / numpy (bit-exact).
* Several ranks driven in lockstep from one process (ExpertParallelLayer's own
  phases, the all-to-alls done as device copies; no kernel waits on another):
  every rank's output against the oracle (tiny layers, every element) and
  against the one-GPU layer (the full-size layer, every element; the oracle on
  sampled routes).
* ExpertParallelLayer.forward over a one-rank NCCL group: the real collectives.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import synthetic as syn
import moe_router_softmax_b200 as moe
from moe_router_softmax_b200.ep import ExpertParallelLayer, TorchExchange, local_layer_of
from ep_support import lockstep
from gpu_support import (FFN_TOL, bf16_dev_to_f64, device_weights_from_host, host_bits, oracle_blob,
                         oracle_layer_for, rel_err)

pytestmark = pytest.mark.gpu
DEV = "cuda"


# ------------------------------------------------------------ the kernels

@pytest.mark.parametrize("dtype,cols,n,src_rows,divisor", [(torch.bfloat16, 2816, 517, 70, 8),
                                                          (torch.float32, 2816, 300, 300, 1),
                                                          (torch.float32, 4, 9, 5, 1),
                                                          (torch.bfloat16, 256, 1, 1, 2)])
def test_gather_rows_bit_exact(dtype, cols, n, src_rows, divisor):
    g = torch.Generator().manual_seed(n)
    src = torch.randn(src_rows, cols, generator=g).to(dtype).to(DEV)
    idx = torch.randint(-3, src_rows * divisor + 5, (n,), generator=g, dtype=torch.int32)
    dst0 = torch.full((n, cols), 7.0, dtype=dtype)
    dst = moe.moe_gather_rows(src, idx.to(DEV), divisor, dst=dst0.clone().to(DEV))
    want = dst0.clone()
    il = idx.long()
    ok = (il >= 0) & (il // divisor < src_rows)
    want[ok] = src.cpu()[il[ok] // divisor]
    assert torch.equal(dst.cpu().view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                       want.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))


@pytest.mark.parametrize("N,El,n_extra", [(2, 4, 0), (4, 32, 5), (8, 16, -3), (1, 1, 0), (8, 128, 0)])
def test_ep_recv_ids_bit_exact(N, El, n_extra):
    rng = np.random.default_rng(N * El)
    counts = rng.integers(0, 40, size=(N, El)).astype(np.int32)
    counts[rng.random((N, El)) < 0.3] = 0              # absent experts
    if N * El >= 4:
        counts.ravel()[2] = 3000                        # one heavy expert
    total = int(counts.sum())
    n = max(total + n_extra, 0)
    got = moe.moe_ep_recv_ids(torch.from_numpy(counts).to(DEV), n).cpu().numpy()
    lab = np.repeat(np.tile(np.arange(El, dtype=np.int32), N), counts.ravel())
    want = np.full(n, -1, np.int32)
    want[:min(n, total)] = lab[:n]
    assert np.array_equal(got, want)


def test_permute_of_no_tokens_is_the_empty_grouping():
    E = 16
    out = (torch.full((E,), 5, dtype=torch.int32, device=DEV), torch.full((E + 1,), 5, dtype=torch.int32, device=DEV),
           torch.empty(0, dtype=torch.int32, device=DEV), torch.empty(0, dtype=torch.int32, device=DEV))
    counts, offsets, _, _ = moe.moe_permute(torch.empty((0, 4), dtype=torch.int32, device=DEV), E, out=out)
    assert int(counts.abs().sum()) == 0 and int(offsets.abs().sum()) == 0


# ------------------------------------------------------ lockstep ranks

def _dev_bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("N,E,H,I,k", [(2, 8, 256, 128, 2), (4, 8, 256, 128, 2), (4, 16, 512, 192, 3)])
def test_lockstep_ranks_match_oracle(fmt, N, E, H, I, k):
    w13, w2 = syn.expert_weights(E, H, I, seed=E + H + N)
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    OL = oracle_layer_for(fmt, w13, w2)
    Ts = [5 + 7 * r for r in range(N)]
    Ts[-1] = 0 if N > 2 else Ts[-1]                     # a rank with no tokens
    xs = [syn.activations(T, H, seed=40 + r) for r, T in enumerate(Ts)]
    lgs = [syn.router_logits(T, E, "normal", seed=60 + r) for r, T in enumerate(Ts)]
    eps = [ExpertParallelLayer(local_layer_of(L, r, N), E, r, N) for r in range(N)]
    hits = [torch.zeros(E // N, dtype=torch.int32, device=DEV) for _ in range(N)]
    ys, _ = lockstep(eps, [torch.from_numpy(g).to(DEV) for g in lgs], [_dev_bf16(x) for x in xs], k, hits)
    torch.cuda.synchronize()
    all_ids = []
    for r in range(N):
        oi, ow, orows, oy = oracle.moe_layer(OL, lgs[r], xs[r], k)
        all_ids.append(oi.ravel())
        assert ys[r].shape == (Ts[r], H)
        if Ts[r]:
            assert rel_err(bf16_dev_to_f64(ys[r]), oy) <= FFN_TOL, r
    want_hits = np.bincount(np.concatenate(all_ids), minlength=E)
    got_hits = np.concatenate([h.cpu().numpy() for h in hits])
    assert np.array_equal(got_hits, want_hits)
    assert moe.moe_take_device_errors() == (0, 0)


def test_lockstep_all_routes_to_one_rank():
    """Every token of every rank picks rank 0's experts: the other ranks receive
    nothing and run no FFN."""
    fmt, N, E, H, I, k, T = 2, 4, 16, 256, 128, 4, 23
    w13, w2 = syn.expert_weights(E, H, I, seed=3)
    L = moe.make_layer(fmt, *device_weights_from_host(w13, w2))
    OL = oracle_layer_for(fmt, w13, w2)
    xs = [syn.activations(T, H, seed=80 + r) for r in range(N)]
    lgs = []
    for r in range(N):
        g = syn.router_logits(T, E, "normal", seed=90 + r)
        g[:, E // N:] -= 100.0
        lgs.append(np.ascontiguousarray(g))
    eps = [ExpertParallelLayer(local_layer_of(L, r, N), E, r, N) for r in range(N)]
    ys, sts = lockstep(eps, [torch.from_numpy(g).to(DEV) for g in lgs], [_dev_bf16(x) for x in xs], k)
    torch.cuda.synchronize()
    assert [sum(st.recv_rows) for st in sts] == [N * T * k, 0, 0, 0]
    for r in range(N):
        oy = oracle.moe_layer(OL, lgs[r], xs[r], k)[3]
        assert rel_err(bf16_dev_to_f64(ys[r]), oy) <= FFN_TOL


def _sparse_oracle_layer(fmt, E, H, I, w13, w2, experts):
    eb = oracle.expert_bytes(fmt, H, I)
    slot = np.full(E, -1, np.int32)
    pool = np.zeros(len(experts) * eb, np.uint8)
    for i, e in enumerate(experts):
        slot[e] = i
        pool[i * eb:(i + 1) * eb] = oracle_blob(fmt, host_bits(w13[e]), host_bits(w2[e]), H, I)
    return oracle.Layer(fmt, E, H, I, np.zeros(eb, np.uint8), pool=pool, slot_table=slot)


@pytest.mark.parametrize("fmt,N", [(0, 4), (2, 8)])
def test_lockstep_full_size_matches_one_gpu(fmt, N):
    E, H, I, k, T = 128, 2816, 704, 8, 64
    w13, w2 = syn.torch_expert_weights(E, H, I, seed=0, layer=0, device=DEV)
    L = moe.make_layer(fmt, w13, w2)
    xs = [syn.activations(T, H, seed=300 + r) for r in range(N)]
    lgs = [syn.router_logits(T, E, "normal", seed=400 + r) for r in range(N)]
    eps = [ExpertParallelLayer(local_layer_of(L, r, N), E, r, N) for r in range(N)]
    ys, sts = lockstep(eps, [torch.from_numpy(g).to(DEV) for g in lgs], [_dev_bf16(x) for x in xs], k)
    for r in range(N):
        lg, xd = torch.from_numpy(lgs[r]).to(DEV), _dev_bf16(xs[r])
        ids, w = moe.moe_route_topk(lg, k)
        c, o, sr, rp = moe.moe_permute(ids, E)
        rows1 = moe.moe_grouped_ffn(L, xd, k, c, o, sr)
        y1 = moe.moe_combine(rows1, rp, w)
        torch.cuda.synchronize()
        # the two calls group the routes differently (El experts over N*T tokens
        # against E over T), so the grouped FFN may take another kernel path and
        # sum in another order; h's bf16 rounding then flips by an ulp in places
        # (measured 1.2e-3 for int4 at N = 8).  A row sent to the wrong expert
        # or back to the wrong route is off by O(1).
        assert rel_err(sts[r].rows_back.cpu().numpy(), rows1.cpu().numpy()) <= FFN_TOL
        assert rel_err(bf16_dev_to_f64(ys[r]), bf16_dev_to_f64(y1)) <= FFN_TOL
    # oracle on sampled routes of rank 1 (in the rows each one came back to)
    oi, ow = oracle.route_topk(lgs[1], k)
    routes = np.array([0, 5, 8 * 31 + 2, T * k - 1], np.int32)
    experts = sorted(set(oi.ravel()[routes].tolist()))
    OL = _sparse_oracle_layer(fmt, E, H, I, w13, w2, experts)
    orows = oracle.ffn_some_routes(OL, xs[1], oi, routes)
    got = sts[1].rows_back.cpu().numpy()[sts[1].route_pos.cpu().numpy()[routes]]
    assert rel_err(got, orows) <= FFN_TOL
    assert moe.moe_take_device_errors() == (0, 0)


# --------------------------------------------------------- real NCCL

def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_forward_over_one_rank_nccl_group():
    fmt, E, H, I, k, T = 0, 128, 2816, 704, 8, 64
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device(DEV, 0))
    try:
        w13, w2 = syn.torch_expert_weights(E, H, I, seed=1, layer=0, device=DEV)
        L = moe.make_layer(fmt, w13, w2)
        ep = ExpertParallelLayer(local_layer_of(L, 0, 1), E, 0, 1, TorchExchange())
        x = _dev_bf16(syn.activations(T, H, seed=500))
        lg = torch.from_numpy(syn.router_logits(T, E, "normal", seed=501)).to(DEV)
        hits = torch.zeros(E, dtype=torch.int32, device=DEV)
        y = ep.forward(lg, x, k, hits=hits)
        y1 = moe.moe_layer_forward(L, lg, x, k)
        ids, _ = moe.moe_route_topk(lg, k)
        torch.cuda.synchronize()
        assert rel_err(bf16_dev_to_f64(y), bf16_dev_to_f64(y1)) <= FFN_TOL
        assert np.array_equal(hits.cpu().numpy(), np.bincount(ids.cpu().numpy().ravel(), minlength=E))
    finally:
        dist.destroy_process_group()
