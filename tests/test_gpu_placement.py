"""The placement refresh on the device (moe_refresh_device) and its promotion
copies (moe_promote_copies) vs the CPU oracle's refresh target and paired
promote/demote, bit for bit: the new slot table, the promotion list in order,
and the promotion / demotion counts."""
import json
import os

import numpy as np
import pytest
import torch

import oracle

import moe_router_softmax_b200 as moe

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _random_table(rng, E, n_slots, n_res):
    so = np.full(E, -1, np.int32)
    ex = rng.choice(E, size=n_res, replace=False)
    sl = rng.choice(n_slots, size=n_res, replace=False)
    so[ex] = sl
    return so


def _device_refresh(hits, so, budget, n_slots):
    table = torch.from_numpy(so.copy()).to(DEV)
    promo, status = moe.moe_refresh_device(torch.from_numpy(hits.astype(np.int32)).to(DEV), budget, table, n_slots)
    torch.cuda.synchronize()
    st = status.cpu().numpy()
    return table.cpu().numpy(), promo.cpu().numpy()[: st[0]], st


def _oracle_refresh(hits, so, budget, n_slots):
    target = oracle.refresh_target(hits.astype(np.uint32), budget)
    new, prom, dem = oracle.apply_placement(so, n_slots, target)
    return new, prom, dem


@pytest.mark.parametrize("E,n_slots,budget,hit_range,n_res", [
    (128, 18, 18, 6, 18), (128, 18, 18, 3, 10), (128, 18, 12, 40, 18), (8, 4, 4, 2, 4), (8, 8, 3, 5, 0),
    (1000, 300, 300, 4, 250), (1024, 1024, 1024, 3, 512), (128, 18, 18, 1, 18), (64, 64, 0, 5, 30),
])
def test_device_refresh_matches_oracle(E, n_slots, budget, hit_range, n_res):
    rng = np.random.default_rng(E + n_slots + budget + hit_range)
    for trial in range(6):
        hits = rng.integers(0, hit_range + 1, size=E).astype(np.uint32)
        if trial == 0:
            hits[:] = 0
        so = _random_table(rng, E, n_slots, min(n_res, n_slots))
        table, promo, st = _device_refresh(hits, so, budget, n_slots)
        new, prom, dem = _oracle_refresh(hits, so, budget, n_slots)
        assert st[2] == 0
        assert np.array_equal(table, new)
        assert st[0] == len(prom) and st[1] == len(dem)
        assert np.array_equal(promo[:, 0], prom)
        assert np.array_equal(promo[:, 1], new[prom])


def test_device_refresh_page_vectors(golden_dir):
    """expert_pool.rs tests: the paired swap limits demotions and keeps extra residents."""
    v = json.load(open(os.path.join(golden_dir, "expert_pool_vectors.json")))
    c = v["paired_swap_limits_demotions"]
    E, budget = c["E"], c["budget"]
    so = np.full(E, -1, np.int32)
    so[c["resident"]] = np.arange(len(c["resident"]))
    hits = np.zeros(E, np.uint32)
    hits[c["target"]] = [5, 4]
    table, promo, st = _device_refresh(hits, so, budget, budget)
    assert st[0] == c["promotions"] and st[1] == c["demotions"]
    assert sorted(np.nonzero(table >= 0)[0].tolist()) == c["resident_after"]
    c = v["paired_swap_keeps_extra_residents"]
    E, budget = c["E"], c["budget"]
    so = np.full(E, -1, np.int32)
    so[c["resident"]] = np.arange(len(c["resident"]))
    hits = np.zeros(E, np.uint32)
    hits[c["target"]] = [9, 8, 7, 6]
    table, promo, st = _device_refresh(hits, so, budget, budget)
    assert st[0] == c["promotions"] and st[1] == c["demotions"]
    assert int((table >= 0).sum()) == c["resident_count_after"]
    assert all(table[e] >= 0 for e in c["must_be_resident"])
    assert all(table[e] < 0 for e in c["must_not_be_resident"])


def test_device_refresh_rejects_an_inconsistent_table():
    E, n_slots = 16, 4
    so = np.full(E, -1, np.int32)
    so[[1, 2]] = 3                     # one slot held twice
    hits = np.arange(E, dtype=np.uint32)
    table, promo, st = _device_refresh(hits, so, n_slots, n_slots)
    assert st[2] == 1 and st[0] == 0
    assert np.array_equal(table, so)
    so = np.full(E, -1, np.int32)
    so[5] = 7                          # slot out of range
    table, promo, st = _device_refresh(hits, so, n_slots, n_slots)
    assert st[2] == 1 and np.array_equal(table, so)


def test_chained_refreshes_match_the_oracle_chain():
    """Thirty refreshes of one layer (Zipf-like hits), the device table carried
    from one to the next, against the oracle carrying its own."""
    rng = np.random.default_rng(7)
    E, n_slots = 128, 18
    so_dev = np.full(E, -1, np.int32)
    so_dev[:n_slots] = np.arange(n_slots)
    so_orc = so_dev.copy()
    table = torch.from_numpy(so_dev).to(DEV)
    pop = 1.0 / np.arange(1, E + 1) ** 1.1
    for r in range(30):
        perm = rng.permutation(E)
        hits = np.zeros(E, np.uint32)
        for e in rng.choice(E, size=(64, 8), p=pop / pop.sum()).ravel():
            hits[perm[e]] += 1
        promo, status = moe.moe_refresh_device(torch.from_numpy(hits.astype(np.int32)).to(DEV), n_slots, table, n_slots)
        so_orc, prom, dem = _oracle_refresh(hits, so_orc, n_slots, n_slots)
        st = status.cpu().numpy()
        assert np.array_equal(table.cpu().numpy(), so_orc)
        assert st[0] == len(prom) and np.array_equal(promo.cpu().numpy()[: st[0], 0], prom)


def test_promote_copies_move_exactly_the_listed_blobs():
    E, n_slots, eb = 32, 6, 4096 + 256
    g = torch.Generator(device=DEV)
    g.manual_seed(3)
    home = torch.randint(0, 256, (E * eb,), dtype=torch.uint8, device=DEV, generator=g)
    pool = torch.zeros(n_slots * eb, dtype=torch.uint8, device=DEV)
    so = np.full(E, -1, np.int32)
    so[[3, 9]] = [0, 4]
    hits = np.zeros(E, np.uint32)
    hits[[3, 11, 20, 9, 30]] = [9, 8, 7, 6, 5]
    table = torch.from_numpy(so).to(DEV)
    promo, status = moe.moe_refresh_device(torch.from_numpy(hits.astype(np.int32)).to(DEV), 5, table, n_slots)
    moe.moe_promote_copies(home, pool, eb, promo, status, n_slots)
    torch.cuda.synchronize()
    st = status.cpu().numpy()
    pr = promo.cpu().numpy()[: st[0]]
    assert st[0] == 3 and sorted(pr[:, 0].tolist()) == [11, 20, 30]
    h = home.cpu().numpy().reshape(E, eb)
    p = pool.cpu().numpy().reshape(n_slots, eb)
    for e, s in pr:
        assert np.array_equal(p[s], h[e])
    untouched = set(range(n_slots)) - set(pr[:, 1].tolist())
    for s in untouched:
        assert not p[s].any()
