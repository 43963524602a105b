"""Expert parallelism on the host (no GPU).

* moe_ep_splits (host C) against a brute-force count of where every route goes,
  and its argument checks.
* The whole expert-parallel layer call (ExpertParallelLayer.forward) across 2 and
  4 processes over gloo: the exchange plan, the three all-to-alls and the buffer
  offsets are the product's; the kernels are replaced by host stand-ins built on
  the oracle (route, permute, per-route FFN, combine), so each rank's output must
  equal, bit for bit, the oracle's one-process layer on that rank's tokens -- a
  row sent to the wrong owner, or returned to the wrong place, changes it.
* The same phases for random partitions (1 to 8 ranks) driven in lockstep from
  one process, with the same host stand-ins and the same bit-exact bar.
"""
import os
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import oracle  # noqa: E402
import synthetic as syn  # noqa: E402
import moe_router_softmax_b200 as moe  # noqa: E402
from ep_support import _bits, host_ops, lockstep  # noqa: E402


# ------------------------------------------------------------------ splits

def _splits_brute(ids_per_rank, E, N):
    """send[s][d] = routes of rank s's tokens whose expert rank d owns."""
    El = E // N
    send = np.zeros((N, N), np.int64)
    for s, ids in enumerate(ids_per_rank):
        for e in np.ravel(ids):
            if 0 <= e < E:
                send[s, e // El] += 1
    return send


@pytest.mark.parametrize("E,N", [(8, 2), (8, 4), (128, 8), (6, 3), (5, 1)])
def test_ep_splits_match_brute_force(E, N):
    rng = np.random.default_rng(E * 31 + N)
    El = E // N
    k = min(E, 3)
    ids_per_rank = []
    for _ in range(N):
        n = int(rng.integers(0, 9))
        ids_per_rank.append(np.array([rng.permutation(E)[:k] for _ in range(n)], np.int32).reshape(n, k))
    counts = [np.bincount(i.ravel(), minlength=E).astype(np.int32) for i in ids_per_rank]
    brute = _splits_brute(ids_per_rank, E, N)
    for r in range(N):
        recv_counts = np.stack([counts[s][r * El:(r + 1) * El] for s in range(N)])
        send, recv = moe.moe_ep_splits(counts[r], recv_counts)
        assert send.tolist() == brute[r].tolist()
        assert recv.tolist() == brute[:, r].tolist()


def test_ep_splits_reject_bad_input():
    c = np.zeros(8, np.int32)
    with pytest.raises(moe.MoeError, match="negative"):
        moe.moe_ep_splits(np.array([0, 0, -1, 0], np.int32), np.zeros((2, 2), np.int32))
    with pytest.raises(ValueError):
        moe.moe_ep_splits(c, np.zeros((2, 3), np.int32))
    L = moe._lib
    assert L.moe_ep_splits(None, 8, 256, 2, 256, 256) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ep_splits(256, 8, 256, 3, 256, 256) == moe.MOE_ERR_INVALID_ARG   # 8 % 3
    big = np.full(4, 2 ** 30, np.int32)
    with pytest.raises(moe.MoeError, match="int32"):
        moe.moe_ep_splits(big, big.reshape(2, 2))


def test_ep_device_calls_reject_bad_arguments_before_launch():
    L = moe._lib
    assert L.moe_gather_rows(256, 4, 100, 256, 4, 1, 256, None) == moe.MOE_ERR_INVALID_ARG    # row_bytes % 16
    assert L.moe_gather_rows(264, 4, 128, 256, 4, 1, 256, None) == moe.MOE_ERR_INVALID_ARG    # unaligned src
    assert L.moe_gather_rows(256, 4, 128, 256, 4, 0, 256, None) == moe.MOE_ERR_INVALID_ARG    # divisor 0
    assert L.moe_gather_rows(None, 4, 128, 256, 4, 1, 256, None) == moe.MOE_ERR_INVALID_ARG   # NULL src
    assert L.moe_gather_rows(None, 4, 128, None, 0, 1, None, None) == moe.MOE_OK              # n == 0
    assert L.moe_ep_recv_ids(256, 4, 512, 256, 8, None) == moe.MOE_ERR_INVALID_ARG            # N*El > 1024
    assert L.moe_ep_recv_ids(256, 0, 4, 256, 8, None) == moe.MOE_ERR_INVALID_ARG             # N == 0
    assert L.moe_ep_recv_ids(None, 2, 4, 256, 8, None) == moe.MOE_ERR_INVALID_ARG            # NULL counts
    assert L.moe_ep_recv_ids(None, 2, 4, None, 0, None) == moe.MOE_OK                        # n == 0


def test_ep_layer_checks_the_partition():
    from moe_router_softmax_b200.ep import ExpertParallelLayer

    local = SimpleNamespace(E=4, H=256)
    with pytest.raises(ValueError, match="multiple"):
        ExpertParallelLayer(local, 10, 0, 4)
    with pytest.raises(ValueError, match="expected"):
        ExpertParallelLayer(local, 16, 0, 2)
    with pytest.raises(ValueError, match="rank"):
        ExpertParallelLayer(local, 8, 2, 2)
    with pytest.raises(RuntimeError, match="exchange"):
        ExpertParallelLayer(local, 8, 0, 2).forward(None, None, 2)


def _host_local_layer(full, fmt, rank, El, H, I):
    eb = full.expert_bytes
    return oracle.Layer(fmt, El, H, I, full.home[rank * El * eb:(rank + 1) * El * eb].copy())


@pytest.mark.parametrize("seed", range(8))
def test_ep_lockstep_on_host_equals_one_process_oracle(seed):
    """Random partitions (N in 1..8, El in 1..3), token counts (0 included), k and
    skewed logits, every rank in one process: each rank's output equals the
    one-process oracle bit for bit, and the owners' hits add up to the global
    histogram."""
    import gpu_support as gs
    from moe_router_softmax_b200.ep import ExpertParallelLayer

    rng = np.random.default_rng(seed)
    N = [1, 2, 3, 4, 8, 2, 5, 3][seed]
    El = int(rng.integers(1, 4))
    E, H, I = N * El, 64, 64
    k = int(rng.integers(1, min(E, 4) + 1))
    fmt = [oracle.BF16, oracle.INT8, oracle.INT4][seed % 3]
    w13, w2 = syn.expert_weights(E, H, I, seed=seed)
    full = gs.oracle_layer_for(fmt, w13, w2)
    eps = [ExpertParallelLayer(_host_local_layer(full, fmt, d, El, H, I), E, d, N, ops=host_ops()) for d in range(N)]
    Ts = [int(t) for t in rng.integers(0, 7, size=N)]
    bias = rng.normal(0.0, 2.0, size=E).astype(np.float32)       # some experts, and so some owners, favoured
    xs = [torch.from_numpy(syn.activations(T, H, seed=10 * seed + d).view(np.int16)).view(torch.bfloat16)
          for d, T in enumerate(Ts)]
    lgs = [np.ascontiguousarray(syn.router_logits(T, E, "normal", seed=20 * seed + d) + bias) for d, T in enumerate(Ts)]
    hits = [torch.zeros(El, dtype=torch.int64) for _ in range(N)]
    ys, sts = lockstep(eps, [torch.from_numpy(g) for g in lgs], xs, k, hits)
    all_ids = []
    for d in range(N):
        ids, w = oracle.route_topk(lgs[d], k)
        all_ids.append(ids.ravel())
        rows = oracle.ffn_routes(full, _bits(xs[d]), ids).astype(np.float32).astype(np.float64)
        assert np.array_equal(ys[d].numpy(), oracle.combine(rows, ids, w, E)), d
        assert sum(sts[d].send_rows) == Ts[d] * k
    assert sum(sum(st.recv_rows) for st in sts) == sum(Ts) * k
    want = np.bincount(np.concatenate(all_ids + [np.zeros(0, np.int64)]).astype(np.int64), minlength=E)
    assert np.concatenate([h.numpy() for h in hits]).tolist() == want.tolist()


def _case(fmt, E, H, I, rank, T, kind):
    w13, w2 = syn.expert_weights(E, H, I, seed=5)
    x = torch.from_numpy(syn.activations(T, H, seed=100 + rank).view(np.int16)).view(torch.bfloat16)
    logits = syn.router_logits(T, E, "normal", seed=200 + rank).astype(np.float32)
    if kind == "to-rank-0":            # every route lands on rank 0's experts
        logits[:, E // 2:] -= 100.0
    return w13, w2, x, torch.from_numpy(np.ascontiguousarray(logits))


def _ep_worker(rank, world, port, fmt, kind, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import gpu_support as gs
    from moe_router_softmax_b200.ep import ExpertParallelLayer, TorchExchange

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        E, H, I, k = 8, 256, 128, 2
        T = 0 if (kind == "empty-rank" and rank == 1) else 6 + 3 * rank
        w13, w2, x, logits = _case(fmt, E, H, I, rank, max(T, 1), kind)
        x, logits = x[:T], logits[:T]
        full = gs.oracle_layer_for(fmt, w13, w2)
        El = E // world
        eb = full.expert_bytes
        local = oracle.Layer(fmt, El, H, I, full.home[rank * El * eb:(rank + 1) * El * eb].copy())
        ep = ExpertParallelLayer(local, E, rank, world, TorchExchange(), ops=host_ops())
        hits = torch.zeros(El, dtype=torch.int64)
        y = ep.forward(logits, x, k, hits=hits).numpy()
        ids, w = oracle.route_topk(logits.numpy(), k)
        ref_rows = oracle.ffn_routes(full, _bits(x), ids).astype(np.float32).astype(np.float64)
        y_ref = oracle.combine(ref_rows, ids, w, E)
        # the hits of this rank's experts, summed over every rank's tokens
        all_ids = [None] * world
        dist.all_gather_object(all_ids, ids.ravel().tolist())
        want_hits = np.bincount(np.concatenate([np.asarray(a, np.int64) for a in all_ids] + [np.zeros(0, np.int64)]),
                                minlength=E)[rank * El:(rank + 1) * El]
        q.put((rank, bool(np.array_equal(y, y_ref)), float(np.abs(y - y_ref).max()) if y.size else 0.0,
               hits.tolist() == want_hits.tolist(), y.shape))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,fmt,kind", [(2, oracle.BF16, "normal"), (2, oracle.INT4, "to-rank-0"),
                                            (4, oracle.BF16, "normal"), (2, oracle.INT8, "empty-rank")])
def test_ep_forward_over_gloo_equals_one_process_oracle(world, fmt, kind):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + (os.getpid() * 7 + world * 13 + fmt * 3 + len(kind)) % 900
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, fmt, kind, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, same, err, hits_ok, shape in sorted(out):
        assert same, (rank, err)
        assert hits_ok, rank
        want_T = 0 if (kind == "empty-rank" and rank == 1) else 6 + 3 * rank
        assert shape == (want_T, 256)
